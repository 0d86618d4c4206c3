// Greedy verify ("DFlash：用“块扩散”魔法", §2 Flash Verification:
// decide_acceptance(logits, draft_block), read greedily).
//
// One bandwidth-bound kernel.  Every target-logit row is cut into chunks; a
// CTA scans one chunk with 16-byte streaming loads (four in flight per
// thread) and keeps (max, lowest index).  It publishes that partial and counts
// itself in its request's counter; the CTA that completes a request's count
// merges the request's partials with one warp (lane i = row i, chunks in
// order), finds the accept length with one ballot and writes the accepted
// tokens plus the bonus token behind out_len, advances out_len and seq_lens,
// and sets the counter back to zero.  Comparisons are exact on the stored
// logit values, so the result does not depend on the chunking or on which
// CTA finishes last.
#include "common.cuh"
#include "internal.h"

namespace dflash {

constexpr int kVerifyThreads = 256;
constexpr int kVerifyUnroll = 4;

template <typename T>
__device__ __forceinline__ void scan16(const uint4& u, int base, float& best, int& bi) {
  constexpr int W = 16 / sizeof(T);
  const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int k = 0; k < W; ++k) {
    const float f = to_f(e[k]);
    if (f > best) { best = f; bi = base + k; }
  }
}

// Argmax of row `row` from its partials part[row * row_stride + c * chunk_stride],
// c < chunks (ascending columns), written by other CTAs or kernels: read from L2.
__device__ __forceinline__ void merge_row(const ArgPart* part, int64_t row_stride,
                                          int64_t chunk_stride, int chunks, int row,
                                          float& best, int& bi) {
  const ArgPart* p = part + (int64_t)row * row_stride;
  best = __ldcg(&p[0].v);
  bi = __ldcg(&p[0].i);
  for (int c = 1; c < chunks; ++c)
    argmax_merge(best, bi, __ldcg(&p[c * chunk_stride].v), __ldcg(&p[c * chunk_stride].i));
}

// Accept step of request r from its B rows' partials (one warp; see merge_row).
__device__ void verify_accept(const ArgPart* part, int64_t row_stride, int64_t chunk_stride,
                              int chunks, int r, const int32_t* draft, int B, int V,
                              int32_t* out_tokens, int32_t* out_len, int out_cap,
                              int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                              int32_t* err) {
  const int lane = threadIdx.x & 31;
  int g = 0;
  int d = 0;
  if (lane < B) {
    float best;
    int bi;
    merge_row(part, row_stride, chunk_stride, chunks, r * B + lane, best, bi);
    g = bi;
    d = draft[(size_t)r * B + lane];
  }
  const unsigned bad = __ballot_sync(0xffffffffu, lane < B && (d < 0 || d >= V));
  const int d_next = __shfl_down_sync(0xffffffffu, d, 1);
  const unsigned mism = __ballot_sync(0xffffffffu, lane < B - 1 && g != d_next);
  const int a = mism ? (__ffs(mism) - 1) : (B - 1);
  const int bonus = __shfl_sync(0xffffffffu, g, a);
  if (bad) {
    if (lane == 0) set_error(err, DFLASH_DEV_TOKEN_RANGE);
    return;
  }
  const int ol = out_len[r];
  if (ol < 0 || (long long)ol + a + 1 > out_cap) {
    if (lane == 0) set_error(err, DFLASH_DEV_OUT_CAP);
    return;
  }
  int32_t* o = out_tokens + (size_t)r * out_cap + ol;
  if (lane < a) o[lane] = d_next;
  if (lane == a) o[a] = bonus;
  if (lane == 0) {
    out_len[r] = ol + a + 1;
    seq_lens[r] += a + 1;
    accept_len[r] = a;
    next_anchor[r] = bonus;
  }
}

// logits and draft are plain pointers: the L2 prefetch runs before the
// dependency wait, and a const __restrict__ pointer would let the compiler
// move a load of another kernel's output above that wait.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kVerifyThreads)
    verify_kernel(const T* logits, int V, int chunk, int chunks, ArgPart* __restrict__ part,
                  unsigned* __restrict__ cnt, const int32_t* draft, int B, int32_t* out_tokens,
                  int32_t* out_len,
                  int out_cap, int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                  int32_t* err, ArgPart* shard_out, int vocab_offset) {
  pdl_trigger();
  __shared__ float s_v[kVerifyThreads / 32];
  __shared__ int s_i[kVerifyThreads / 32];
  __shared__ int s_last;
  const int row = blockIdx.y, c = blockIdx.x;
  const int v0 = c * chunk;
  const int v1 = min(V, v0 + chunk);
  const T* x = logits + (size_t)row * V;
  if (VEC && (threadIdx.x & 31) == 0 && v1 > v0) {
    // The logits are an input no kernel of the cycle writes: while the
    // predecessor drains, each warp asks L2 for its share of the chunk.  L2 is
    // the point of coherence, so a line prefetched early is never read stale.
    const int nw = kVerifyThreads / 32, w = threadIdx.x >> 5;
    const size_t bytes = (size_t)(v1 - v0) * sizeof(T);       // a multiple of 16
    const size_t per = (bytes / nw + 15) / 16 * 16;
    const size_t b0 = (size_t)w * per;
    if (b0 < bytes) {
      const uint32_t n = (uint32_t)min(per, bytes - b0);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                       reinterpret_cast<const uint8_t*>(x + v0) + b0),
                   "r"(n)
                   : "memory");
    }
  }
  pdl_wait();
  float best = -INFINITY;
  int bi = 0x7fffffff;
  if (VEC) {
    constexpr int W = 16 / sizeof(T);  // elements per 16-byte load (chunk is a multiple)
    const int nvec = (v1 - v0) / W;
    const uint4* p = reinterpret_cast<const uint4*>(x + v0);
    int t = threadIdx.x;
    // each thread visits its elements in increasing index order, so a strict
    // '>' keeps the lowest index among equal maxima
    for (; t + (kVerifyUnroll - 1) * kVerifyThreads < nvec; t += kVerifyUnroll * kVerifyThreads) {
      uint4 u[kVerifyUnroll];
#pragma unroll
      for (int j = 0; j < kVerifyUnroll; ++j) u[j] = __ldcs(p + t + j * kVerifyThreads);
#pragma unroll
      for (int j = 0; j < kVerifyUnroll; ++j)
        scan16<T>(u[j], v0 + (t + j * kVerifyThreads) * W, best, bi);
    }
    for (; t < nvec; t += kVerifyThreads) scan16<T>(__ldcs(p + t), v0 + t * W, best, bi);
    for (int v = v0 + nvec * W + threadIdx.x; v < v1; v += kVerifyThreads) {
      const float f = to_f(x[v]);
      if (f > best || (f == best && v < bi)) { best = f; bi = v; }
    }
  } else {
    for (int v = v0 + threadIdx.x; v < v1; v += kVerifyThreads) {
      const float f = to_f(x[v]);
      if (f > best) { best = f; bi = v; }
    }
  }
  warp_argmax(best, bi);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) { s_v[w] = best; s_i[w] = bi; }
  __syncthreads();
  const int r = row / B;
  if (threadIdx.x == 0) {
    best = s_v[0];
    bi = s_i[0];
    for (int k = 1; k < kVerifyThreads / 32; ++k) argmax_merge(best, bi, s_v[k], s_i[k]);
    part[(size_t)row * chunks + c] = ArgPart{best, bi};
    __threadfence();  // the partial is visible before this CTA is counted
    s_last = atomicAdd(&cnt[r], 1u) == (unsigned)(B * chunks - 1);
  }
  __syncthreads();
  if (!s_last || threadIdx.x >= 32) return;
  __threadfence();  // every partial of request r counted before this CTA's reads
  if (shard_out != nullptr) {
    // a vocabulary shard: publish each row's argmax with its global id
    if (lane < B) {
      float best;
      int bi;
      merge_row(part, chunks, 1, chunks, r * B + lane, best, bi);
      shard_out[r * B + lane] = ArgPart{best, bi + vocab_offset};
    }
  } else {
    verify_accept(part, chunks, 1, chunks, r, draft, B, V, out_tokens, out_len, out_cap,
                  seq_lens, accept_len, next_anchor, err);
  }
  if (lane == 0) cnt[r] = 0;  // ready for the next call
}

int verify_chunks(int rows, int V) {
  // enough CTAs for ~4 per SM, chunks of at least 4096 elements, multiple of 64
  int target = (4 * 148 + rows - 1) / rows;
  int max_c = (V + 4095) / 4096;
  int c = target < max_c ? target : max_c;
  return c < 1 ? 1 : c;
}

int launch_verify(const void* logits, int dtype, const int32_t* draft, int batch, int B, int V,
                  int32_t* out_tokens, int32_t* out_len, int out_cap, int32_t* seq_lens,
                  int32_t* accept_len, int32_t* next_anchor, void* part_v, int chunks,
                  unsigned* cnt, int32_t* err, cudaStream_t s) {
  const int rows = batch * B;
  ArgPart* part = reinterpret_cast<ArgPart*>(part_v);
  int chunk = (V + chunks - 1) / chunks;
  chunk = (chunk + 63) / 64 * 64;
  const int esz = dtype == DFLASH_BF16 ? 2 : 4;
  const bool vec = ((size_t)V * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(logits) % 16) == 0;
  const dim3 grid(chunks, rows), block(kVerifyThreads);
  TimedScope ts(s, TC_VERIFY);
  cudaError_t e;
  if (dtype == DFLASH_BF16) {
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(logits);
    auto k = vec ? verify_kernel<__nv_bfloat16, true> : verify_kernel<__nv_bfloat16, false>;
    e = launch_pdl(k, grid, block, 0, s, 1, x, V, chunk, chunks, part, cnt, draft, B, out_tokens,
                   out_len, out_cap, seq_lens, accept_len, next_anchor, err, (ArgPart*)nullptr, 0);
  } else {
    const float* x = static_cast<const float*>(logits);
    auto k = vec ? verify_kernel<float, true> : verify_kernel<float, false>;
    e = launch_pdl(k, grid, block, 0, s, 1, x, V, chunk, chunks, part, cnt, draft, B, out_tokens,
                   out_len, out_cap, seq_lens, accept_len, next_anchor, err, (ArgPart*)nullptr, 0);
  }
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

int launch_verify_shard(const void* logits, int dtype, int batch, int B, int Vs, int vocab_offset,
                        ArgPart* out, void* part_v, int chunks, unsigned* cnt, cudaStream_t s) {
  const int rows = batch * B;
  ArgPart* part = reinterpret_cast<ArgPart*>(part_v);
  int chunk = (Vs + chunks - 1) / chunks;
  chunk = (chunk + 63) / 64 * 64;
  const int esz = dtype == DFLASH_BF16 ? 2 : 4;
  const bool vec = ((size_t)Vs * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(logits) % 16) == 0;
  const dim3 grid(chunks, rows), block(kVerifyThreads);
  TimedScope ts(s, TC_VERIFY);
  cudaError_t e;
  if (dtype == DFLASH_BF16) {
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(logits);
    auto k = vec ? verify_kernel<__nv_bfloat16, true> : verify_kernel<__nv_bfloat16, false>;
    e = launch_pdl(k, grid, block, 0, s, 1, x, Vs, chunk, chunks, part, cnt,
                   (const int32_t*)nullptr, B, (int32_t*)nullptr, (int32_t*)nullptr, 0,
                   (int32_t*)nullptr, (int32_t*)nullptr, (int32_t*)nullptr, (int32_t*)nullptr, out,
                   vocab_offset);
  } else {
    const float* x = static_cast<const float*>(logits);
    auto k = vec ? verify_kernel<float, true> : verify_kernel<float, false>;
    e = launch_pdl(k, grid, block, 0, s, 1, x, Vs, chunk, chunks, part, cnt,
                   (const int32_t*)nullptr, B, (int32_t*)nullptr, (int32_t*)nullptr, 0,
                   (int32_t*)nullptr, (int32_t*)nullptr, (int32_t*)nullptr, (int32_t*)nullptr, out,
                   vocab_offset);
  }
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

// One warp per request: row i's argmax merged over the shards in order, then the
// accept step.
__global__ void verify_merge_kernel(const ArgPart* __restrict__ parts, int world, int batch,
                                    const int32_t* __restrict__ draft, int B, int V,
                                    int32_t* out_tokens, int32_t* out_len, int out_cap,
                                    int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                                    int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= batch) return;
  verify_accept(parts, 1, (int64_t)batch * B, world, r, draft, B, V, out_tokens, out_len, out_cap,
                seq_lens, accept_len, next_anchor, err);
}

int launch_verify_merge(const ArgPart* parts, int world, const int32_t* draft, int batch, int B,
                        int V, int32_t* out_tokens, int32_t* out_len, int out_cap,
                        int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                        int32_t* err, cudaStream_t s) {
  TimedScope ts(s, TC_VERIFY);
  const int wpb = 4;
  const cudaError_t e =
      launch_pdl(verify_merge_kernel, dim3((batch + wpb - 1) / wpb), dim3(32 * wpb), 0, s, 1,
                 parts, world, batch, draft, B, V, out_tokens, out_len, out_cap, seq_lens,
                 accept_len, next_anchor, err);
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
