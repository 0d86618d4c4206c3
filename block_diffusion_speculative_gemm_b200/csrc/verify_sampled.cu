// Sampled (temperature) verify of a drafted block.
//
// Sources: "DFlash: Block Diffusion for Flash Speculative Decoding" (study
// notes), §消融实验结论 (drafting holds up under high-temperature sampling) and
// §与 Speculative Decoding 系列的关系 (the speculative-decoding line of Leviathan
// et al., 2023); blog "DFlash：用“块扩散”魔法", §2 Flash Verification (the
// target's probabilities are compared with the draft's).  The pages give no
// acceptance rule; this is standard speculative sampling:
//
//   p_i = softmax(Z_i / tau) (target row i: the token after block position i),
//   q_j = softmax(Y_j / tau) (draft distribution at block position j);
//   for i = 0..B-2 in order, d_{i+1} is accepted while
//     log U_i < log p_i(d_{i+1}) - log q_{i+1}(d_{i+1});
//   the first rejection at i draws the last token from max(0, p_i - q_{i+1}),
//   no rejection draws it from p_{B-1}; emit d_1..d_a and the drawn token.
//
// Draws are Gumbel-max, argmax_v (log w_v - log(-log U'_v)), ties to the lower
// index.  Uniforms come from Philox4x64-10 (Salmon, Moraes, Dror and Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011) under key (seed, 0)
// with counter (offset, request, stream, n / 4), word n % 4: stream 0 gives
// U_i (n = i), stream 1 gives U'_v (n = v).  A word w gives
// U = (w >> 11) 2^-53 in [0, 1) and U' = ((w >> 11) + 1/2) 2^-53 in (0, 1).
//
// Two kernels chained by programmatic dependent launch:
//   sv_stats_kernel  one CTA per (row chunk, row) of the target and the draft
//                    logits, as many chunks as fill the resident slots once:
//                    (max, sum of 2^(x log2e / tau - max)) per chunk, eight
//                    16-byte loads in flight per thread.  The last CTA of a
//                    request merges its rows (one warp, lane i = row i), takes
//                    the accept decisions in the log domain and records the
//                    accept length and the normalisers of the row(s) the draw
//                    needs.
//   sv_draw_kernel   one CTA per (vocabulary chunk, request), four per SM over
//                    the batch, reads target row a (and draft row a+1) once
//                    more, adds the Gumbel terms, keeps the best perturbed
//                    log-weight; the last CTA of a request merges the chunks in
//                    order, writes d_1..d_a and the drawn token behind out_len
//                    and advances the lengths.
// Counters count arrivals per request and are set back to zero by the CTA
// that completes them, so the workspace stays reusable.
#include "common.cuh"
#include "internal.h"
#include "philox.cuh"

namespace dflash {

namespace {

constexpr int kSvThreads = 256;
constexpr float kLn2 = 0.69314718055994531f;
constexpr float kLog2e = 1.44269504088896341f;

enum SvMode : int { SV_SKIP = 0, SV_RESIDUAL = 1, SV_BONUS = 2 };

struct SvPart {  // per (tensor row, chunk): max and sum of 2^(x c - max), c = log2e / tau
  float m, s;
};

struct SvRec {  // per request, written by the stats kernel for the draw kernel
  int a, mode;
  float offp;  // target row a: log2 p_a(v) = z_v c + offp, c = log2 e / tau
  float offq;  // draft row a+1 (residual mode): log2 q_{a+1}(v) = y_v c + offq
  int pad[4];
};

struct SvDraw {  // per (request, chunk): best residual and best target-only draw
  float sr;
  int ir;
  float sp;
  int ip;
};

__device__ __forceinline__ void stat_merge(float& m, float& s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float M = fmaxf(m, m2);
  s = s * exp2f(m - M) + s2 * exp2f(m2 - M);
  m = M;
}

// The 16 bytes of u as floats: bf16 pairs widen by a shift / mask of each word.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& u, float (&x)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(wd[k] << 16);
      x[2 * k + 1] = __uint_as_float(wd[k] & 0xffff0000u);
    }
  } else {
    x[0] = __uint_as_float(u.x);
    x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z);
    x[3] = __uint_as_float(u.w);
  }
}

// Adds the 16 bytes of u to the running (m, s0 + s1): the maximum is taken
// on the raw values (c > 0 keeps the order) and the exponents are
// fused multiply-adds x c - m; two partial sums halve the add chain.
template <typename T>
__device__ __forceinline__ void stat_add16_lean(const uint4& u, float c, float& m, float& s0,
                                                float& s1) {
  constexpr int W = 16 / sizeof(T);
  float x[W];
  unpack16<T>(u, x);
  float mb = x[0];
#pragma unroll
  for (int k = 1; k < W; ++k) mb = fmaxf(mb, x[k]);
  mb *= c;
  if (mb > m) {
    const float sc = ex2_ftz(m - mb);  // 0 while m is -inf
    s0 *= sc;
    s1 *= sc;
    m = mb;
  }
  if (m == -INFINITY) return;  // nothing finite yet: every x is -inf
  const float nm = -m;
#pragma unroll
  for (int k = 0; k < W; k += 2) {
    s0 += ex2_ftz(fmaf(x[k], c, nm));
    s1 += ex2_ftz(fmaf(x[k + 1], c, nm));
  }
}

// (m, s) of the whole CTA, in warp order, returned to thread 0.  Every thread
// of the CTA calls it; it ends with the CTA synchronised.
__device__ __forceinline__ SvPart block_stat(float m, float s, float* s_m, float* s_s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float sv2 = __shfl_xor_sync(0xffffffffu, s, o);
    stat_merge(m, s, m2, sv2);
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) {
    s_m[w] = m;
    s_s[w] = s;
  }
  __syncthreads();
  SvPart r{s_m[0], s_s[0]};
  if (threadIdx.x == 0)
    for (int k = 1; k < kSvThreads / 32; ++k) stat_merge(r.m, r.s, s_m[k], s_s[k]);
  __syncthreads();  // s_m / s_s free for the next call
  return r;
}

// The accept decisions of request r, by one warp (lane i = block row i).
// stat(y) returns the merged statistics of tensor row y: target row y for
// y < rows, draft row y - rows otherwise.  Writes rec[r] and sets cnt[r] back
// to zero for the draw kernel.
template <typename T, typename StatFn>
__device__ void sv_accept(int r, const T* __restrict__ target, const T* __restrict__ drafted,
                          int rows, int B, int V, float c2, const int32_t* __restrict__ draft,
                          const int32_t* __restrict__ out_len, int out_cap, uint64_t seed,
                          uint64_t offset, SvRec* __restrict__ rec, unsigned* __restrict__ cnt,
                          int32_t* err, StatFn stat) {
  const int lane = threadIdx.x & 31;
  SvPart st{-INFINITY, 0.f}, sd{-INFINITY, 0.f};
  int d = 0;
  if (lane < B) {
    st = stat(r * B + lane);
    if (lane > 0) sd = stat(rows + r * B + lane);
    d = draft[(size_t)r * B + lane];
  }
  const unsigned bad = __ballot_sync(0xffffffffu, lane < B && (d < 0 || d >= V));
  const int d_next = __shfl_down_sync(0xffffffffu, d, 1);
  const float md_next = __shfl_down_sync(0xffffffffu, sd.m, 1);
  const float sd_next = __shfl_down_sync(0xffffffffu, sd.s, 1);
  bool reject = false;
  if (!bad && lane < B - 1) {
    const float z = to_f(target[((size_t)r * B + lane) * V + d_next]) * c2;
    const float yv = to_f(drafted[((size_t)r * B + lane + 1) * V + d_next]) * c2;
    // log2 p_i(x) - log2 q_{i+1}(x), then natural units
    const float l2rho = (z - st.m - log2f(st.s)) - (yv - md_next - log2f(sd_next));
    uint64_t wds[4];
    philox_block(seed, offset, r, 0, (uint64_t)(lane >> 2), wds);
    const int q = lane & 3;
    const uint64_t wsel = q == 0 ? wds[0] : q == 1 ? wds[1] : q == 2 ? wds[2] : wds[3];
    const float lu = log_u_closed_open(wsel);
    reject = !(lu < l2rho * kLn2);
  }
  const unsigned rej = __ballot_sync(0xffffffffu, reject);
  const int a = rej ? (__ffs(rej) - 1) : (B - 1);
  int mode = SV_SKIP;
  if (bad) {
    if (lane == 0) set_error(err, DFLASH_DEV_TOKEN_RANGE);
  } else {
    const int ol = out_len[r];
    if (ol < 0 || (long long)ol + a + 1 > out_cap) {
      if (lane == 0) set_error(err, DFLASH_DEV_OUT_CAP);
    } else {
      mode = a < B - 1 ? SV_RESIDUAL : SV_BONUS;
    }
  }
  if (lane == a) {
    SvRec q;
    q.a = a;
    q.mode = mode;
    q.offp = -(st.m + log2f(st.s));
    q.offq = mode == SV_RESIDUAL ? -(md_next + log2f(sd_next)) : 0.f;
    q.pad[0] = q.pad[1] = q.pad[2] = q.pad[3] = 0;
    rec[r] = q;
  }
  if (lane == 0) cnt[r] = 0;  // ready for the draw kernel and the next call
}

// One thread's share of the n 16-byte units at p (units t, t + 256, ...),
// eight loads in flight at a time.
template <typename T>
__device__ __forceinline__ void stat_units(const uint4* p, int n, float c, float& m, float& s) {
  constexpr int D = 8;
  float s0 = 0.f, s1 = 0.f;
  m = -INFINITY;
  int t = threadIdx.x;
  for (; t + (D - 1) * kSvThreads < n; t += D * kSvThreads) {
    uint4 u[D];
#pragma unroll
    for (int j = 0; j < D; ++j) u[j] = __ldcs(p + t + j * kSvThreads);
#pragma unroll
    for (int j = 0; j < D; ++j) stat_add16_lean<T>(u[j], c, m, s0, s1);
  }
  for (; t < n; t += kSvThreads) stat_add16_lean<T>(__ldcs(p + t), c, m, s0, s1);
  s = s0 + s1;
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kSvThreads)
    sv_stats_kernel(const T* __restrict__ target, const T* __restrict__ drafted, int rows, int B,
                    int V, float c2, int chunk, int chunks, SvPart* __restrict__ part,
                    unsigned* __restrict__ cnt, const int32_t* __restrict__ draft,
                    const int32_t* __restrict__ out_len, int out_cap, uint64_t seed,
                    uint64_t offset, SvRec* __restrict__ rec, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_m[kSvThreads / 32], s_s[kSvThreads / 32];
  __shared__ int s_last;
  const int y = blockIdx.y, c = blockIdx.x;
  const bool is_draft = y >= rows;
  const int row = is_draft ? y - rows : y;  // r * B + i
  const int r = row / B;
  float m = -INFINITY, s = 0.f;
  if (!(is_draft && row % B == 0)) {  // draft row 0 (the anchor) has no distribution
    const T* x = (is_draft ? drafted : target) + (size_t)row * V;
    const int v0 = c * chunk, v1 = min(V, v0 + chunk);
    if (VEC) {
      constexpr int W = 16 / sizeof(T);
      const int nvec = max(0, v1 - v0) / W;  // v0 is a multiple of 64: 16-byte aligned
      stat_units<T>(reinterpret_cast<const uint4*>(x + v0), nvec, c2, m, s);
      for (int v = v0 + nvec * W + threadIdx.x; v < v1; v += kSvThreads)
        stat_merge(m, s, to_f(x[v]) * c2, 1.f);
    } else {
      for (int v = v0 + threadIdx.x; v < v1; v += kSvThreads) stat_merge(m, s, to_f(x[v]) * c2, 1.f);
    }
  }
  const SvPart b = block_stat(m, s, s_m, s_s);
  if (threadIdx.x == 0) {
    part[(size_t)y * chunks + c] = b;
    __threadfence();  // the partial is visible before this CTA is counted
    s_last = atomicAdd(&cnt[r], 1u) == (unsigned)(2 * B * chunks - 1);
  }
  __syncthreads();
  if (!s_last || threadIdx.x >= 32) return;
  __threadfence();  // every partial of request r counted before the reads below
  auto merged = [&](int yy) {
    const SvPart* p = part + (size_t)yy * chunks;
    float mm = __ldcg(&p[0].m), ss = __ldcg(&p[0].s);
    for (int k = 1; k < chunks; ++k) stat_merge(mm, ss, __ldcg(&p[k].m), __ldcg(&p[k].s));
    return SvPart{mm, ss};
  };
  sv_accept<T>(r, target, drafted, rows, B, V, c2, draft, out_len, out_cap, seed, offset, rec, cnt,
               err, merged);
}

__device__ __forceinline__ void draw_merge(float& s, int& i, float s2, int i2) {
  if (s2 > s || (s2 == s && i2 < i)) {
    s = s2;
    i = i2;
  }
}

template <typename T>
__device__ __forceinline__ void load4(const T* p, bool vec, float (&x)[4], int n) {
  if (vec && n == 4) {
    if (sizeof(T) == 2) {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = to_f(e[k]);
    } else {
      const float4 u = *reinterpret_cast<const float4*>(p);
      x[0] = u.x;
      x[1] = u.y;
      x[2] = u.z;
      x[3] = u.w;
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = k < n ? to_f(p[k]) : 0.f;
}

// The inputs another kernel writes (the logits, the draft tokens and the
// stats pass's records) are read through plain pointers.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kSvThreads, 4)
    sv_draw_kernel(const T* target, const T* drafted, int B, int V, float c2, int chunk,
                   int chunks, const SvRec* rec, SvDraw* part, unsigned* cnt,
                   const int32_t* draft, int32_t* out_tokens, int32_t* out_len, int out_cap,
                   int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor, uint64_t seed,
                   uint64_t offset) {
  __shared__ SvDraw s_d[kSvThreads / 32];
  __shared__ int s_last;
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.y, c = blockIdx.x;
  const SvRec q = rec[r];
  // scores in log2 units: log2 w_v + G_v log2 e, the natural-unit score times
  // log2 e, so the argmax is the same
  float sr = -INFINITY, sp = -INFINITY;
  int ir = 0x7fffffff, ip = 0x7fffffff;
  if (q.mode != SV_SKIP) {
    const bool residual = q.mode == SV_RESIDUAL;
    const T* zr = target + ((size_t)r * B + q.a) * V;
    const T* yr = residual ? drafted + ((size_t)r * B + q.a + 1) * V : zr;  // draft row a+1
    const float dq = q.offq - q.offp;  // log2 q - log2 p = (y - z) c + dq
    const int v0 = c * chunk, v1 = min(V, v0 + chunk);  // chunk is a multiple of 64
    // groups of 4 consecutive entries; each thread visits its groups in
    // increasing order, so '>' keeps the lowest index
    for (int g = v0 / 4 + threadIdx.x; g * 4 < v1; g += kSvThreads) {
      const int vb = g * 4, n = min(4, v1 - vb);
      float z[4], yv[4], gum[4];
      load4<T>(zr + vb, VEC, z, n);
      if (residual) load4<T>(yr + vb, VEC, yv, n);
      uint64_t wds[4];
      philox_block(seed, offset, r, 1, (uint64_t)g, wds);
#pragma unroll
      for (int k = 0; k < 4; ++k) gum[k] = gumbel2_of(wds[k]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k >= n) break;
        const float lp = fmaf(z[k], c2, q.offp);
        const float scp = lp + gum[k];
        if (scp > sp) { sp = scp; ip = vb + k; }
        if (residual) {
          const float d = fmaf(yv[k] - z[k], c2, dq);
          if (d < 0.f) {
            const float scr = lp + log2_one_minus_exp2(d) + gum[k];
            if (scr > sr) { sr = scr; ir = vb + k; }
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    draw_merge(sr, ir, __shfl_xor_sync(0xffffffffu, sr, o), __shfl_xor_sync(0xffffffffu, ir, o));
    draw_merge(sp, ip, __shfl_xor_sync(0xffffffffu, sp, o), __shfl_xor_sync(0xffffffffu, ip, o));
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) s_d[w] = SvDraw{sr, ir, sp, ip};
  __syncthreads();
  if (threadIdx.x == 0) {
    SvDraw b = s_d[0];
    for (int k = 1; k < kSvThreads / 32; ++k) {
      draw_merge(b.sr, b.ir, s_d[k].sr, s_d[k].ir);
      draw_merge(b.sp, b.ip, s_d[k].sp, s_d[k].ip);
    }
    part[(size_t)r * chunks + c] = b;
    __threadfence();
    s_last = atomicAdd(&cnt[r], 1u) == (unsigned)(chunks - 1);
  }
  __syncthreads();
  if (!s_last || threadIdx.x >= 32) return;
  __threadfence();
  if (q.mode != SV_SKIP) {
    // chunks in order; the residual draw unless fp32 left it empty
    float br = -INFINITY, bp = -INFINITY;
    int jr = 0x7fffffff, jp = 0x7fffffff;
    for (int k = lane; k < chunks; k += 32) {
      const SvDraw* p = part + (size_t)r * chunks + k;
      draw_merge(br, jr, __ldcg(&p->sr), __ldcg(&p->ir));
      draw_merge(bp, jp, __ldcg(&p->sp), __ldcg(&p->ip));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      draw_merge(br, jr, __shfl_xor_sync(0xffffffffu, br, o), __shfl_xor_sync(0xffffffffu, jr, o));
      draw_merge(bp, jp, __shfl_xor_sync(0xffffffffu, bp, o), __shfl_xor_sync(0xffffffffu, jp, o));
    }
    const int tok = (q.mode == SV_RESIDUAL && br != -INFINITY) ? jr : jp;
    const int a = q.a, ol = out_len[r];
    int32_t* o = out_tokens + (size_t)r * out_cap + ol;
    if (lane < a) o[lane] = draft[(size_t)r * B + lane + 1];
    if (lane == a) o[a] = tok;
    if (lane == 0) {
      out_len[r] = ol + a + 1;
      seq_lens[r] += a + 1;
      accept_len[r] = a;
      next_anchor[r] = tok;
    }
  }
  if (lane == 0) cnt[r] = 0;
}

// Chunks per row of the gridded stats pass (rows that are not 16-byte
// aligned).  The workspace is sized for the most a B200 can hold at once
// (8 CTAs of 256 threads on each of 148 SMs); a launch takes as many chunks as
// fill the resident slots of its kernel once (`slots`), and at least two where
// the workspace allows: with one row per CTA the SMs hold 3 or 4 rows each and
// the ones with 4 set the time, while half rows let a second wave even them out
// (measured 76.8 -> 74.75 us at 32 x 8 rows; three chunks gave 76.8 us).
int sv_chunks_max(int rows, int V, int min_chunk) {
  int target = (8 * 148 + rows - 1) / rows;
  int max_c = (V + min_chunk - 1) / min_chunk;
  int c = target < max_c ? target : max_c;
  return c < 1 ? 1 : c;
}

int sv_chunks(int rows, int V, int min_chunk, int slots) {
  int c = slots / rows;
  if (c < 2) c = 2;
  const int cap = sv_chunks_max(rows, V, min_chunk);
  if (c > cap) c = cap;
  return c < 1 ? 1 : c;
}

template <typename K>
int resident_slots(K kernel, size_t smem = 0) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kSvThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  return per_sm * num_sms();
}

int chunk_len(int V, int chunks) {
  int chunk = (V + chunks - 1) / chunks;
  return (chunk + 63) / 64 * 64;
}

// Draw chunks per request: four CTAs per SM over the batch, chunks of at
// least 2048 entries (at most ceil(V / 2048) chunks, the workspace bound).
int sv_draw_chunks_max(int V) { return (V + 2047) / 2048; }

int sv_draw_chunks(int batch, int V) {
  int q = 4 * num_sms() / (batch > 0 ? batch : 1);
  if (q > sv_draw_chunks_max(V)) q = sv_draw_chunks_max(V);
  return q < 1 ? 1 : q;
}

__global__ void sample_math_kernel(const uint64_t* __restrict__ w, const float* __restrict__ d,
                                   int n, float* __restrict__ g2, float* __restrict__ l2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  g2[i] = gumbel2_of(w[i]);
  l2[i] = log2_one_minus_exp2(d[i]);
}

}  // namespace

int launch_sample_math(const uint64_t* w, const float* d, int n, float* g2, float* l2,
                       cudaStream_t s) {
  if (n <= 0) return DFLASH_OK;
  sample_math_kernel<<<(n + 255) / 256, 256, 0, s>>>(w, d, n, g2, l2);
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

namespace {

struct SvLayout {
  size_t part1, rec, part2, total;
};

SvLayout sv_layout(int batch, int B, int V) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const int rows = batch * B;
  const size_t p1 = (size_t)2 * rows * sv_chunks_max(2 * rows, V, 4096);
  SvLayout L;
  L.part1 = 0;
  L.rec = al(p1 * sizeof(SvPart));
  L.part2 = L.rec + al((size_t)batch * sizeof(SvRec));
  L.total = L.part2 + al((size_t)batch * sv_draw_chunks_max(V) * sizeof(SvDraw));
  return L;
}

}  // namespace

size_t sampled_verify_bytes(int batch, int B, int V) { return sv_layout(batch, B, V).total; }

int launch_sampled_verify(const void* target, const void* drafted, int dtype, const int32_t* draft,
                          int batch, int B, int V, float tau, uint64_t seed, uint64_t offset,
                          int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                          int32_t* accept_len, int32_t* next_anchor, void* scratch,
                          unsigned* cnt, int32_t* err, cudaStream_t s) {
  const int rows = batch * B;
  const SvLayout L = sv_layout(batch, B, V);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  SvPart* part1 = reinterpret_cast<SvPart*>(base + L.part1);
  SvRec* rec = reinterpret_cast<SvRec*>(base + L.rec);
  SvDraw* part2 = reinterpret_cast<SvDraw*>(base + L.part2);
  const int esz = dtype == DFLASH_BF16 ? 2 : 4;
  const bool vec = ((size_t)V * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(target) % 16) == 0 &&
                   (reinterpret_cast<uintptr_t>(drafted) % 16) == 0;
  const float c2f = kLog2e / tau;
  const int q = sv_draw_chunks(batch, V), kq = chunk_len(V, q);
  TimedScope ts(s, TC_VERIFY);
  auto run = [&](auto tag) -> cudaError_t {
    using T = decltype(tag);
    const T* zt = static_cast<const T*>(target);
    const T* yd = static_cast<const T*>(drafted);
    auto ka = vec ? sv_stats_kernel<T, true> : sv_stats_kernel<T, false>;
    static int slots[2] = {0, 0};  // [vec]
    if (slots[vec] == 0) slots[vec] = resident_slots(ka);
    const int c1 = sv_chunks(2 * rows, V, 4096, slots[vec]);
    const cudaError_t e = launch_pdl(ka, dim3(c1, 2 * rows), dim3(kSvThreads), 0, s, 1, zt, yd,
                                     rows, B, V, c2f, chunk_len(V, c1), c1, part1, cnt, draft,
                                     (const int32_t*)out_len, out_cap, seed, offset, rec, err);
    if (e != cudaSuccess) return e;
    auto kb = vec ? sv_draw_kernel<T, true> : sv_draw_kernel<T, false>;
    return launch_pdl(kb, dim3(q, batch), dim3(kSvThreads), 0, s, 1, zt, yd, B, V, c2f, kq, q,
                      (const SvRec*)rec, part2, cnt, draft, out_tokens, out_len, out_cap,
                      seq_lens, accept_len, next_anchor, seed, offset);
  };
  const cudaError_t e = dtype == DFLASH_BF16 ? run(__nv_bfloat16{}) : run(float{});
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
