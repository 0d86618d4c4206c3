// Token draw of sampled (temperature) drafting.
//
// Sources: "DFlash + Spec V2 深度解析", §2.3 块扩散 (each forward predicts every
// masked position of the block, most confident positions are fixed first) and
// "DFlash: Block Diffusion for Flash Speculative Decoding" (study notes),
// §消融实验结论 (drafting holds up under high-temperature sampling).  The pages
// give no sampling rule for a diffusion draft; the reading taken is the
// sampled counterpart of the greedy commit rule:
//
//   at step t, every still-masked position j of request r draws
//     x_j = argmax_v (Y_jv / tau + G_v),   G_v = -log(-log U'_v),
//   ties to the lowest id, with U'_v from Philox4x64-10 stream 2 under key
//   (seed, 0): draw n = (t B + j) V + v is word n % 4 of counter
//   (offset, r, 2, n / 4), mapped to ((w >> 11) + 1/2) 2^-53;
//   its confidence is the untempered probability softmax(Y_j)(x_j).
// The commit of the ceil(remaining / steps left) most confident positions is
// the greedy path's commit kernel, unchanged.
//
// Y_j is read back from the logits row the LM-head epilogue wrote for
// position j (the caller's draft_logits output): the draw uses exactly the
// stored row, so the token is an exact draw from the distribution that sampled
// verify later reads.  One CTA per (vocabulary chunk, masked row) keeps the
// untempered softmax statistics (max and sum of 2^(y log2 e - max)) and the
// best Gumbel score with its id and logit; the last CTA of a row, found with
// the row's counter (which it sets back to zero), merges the chunks in order.
#include "common.cuh"
#include "internal.h"
#include "philox.cuh"

namespace dflash {

namespace {

constexpr int kSdThreads = 256;
constexpr int kSdMaxChunks = 64;
constexpr int kSdStream = 2;
constexpr float kLog2e = 1.44269504088896341f;

struct SdPart {
  float m, s;   // untempered softmax statistics of the chunk, log2 units
  float gs, gy; // best Gumbel score and the logit of its entry
  int gi;       // id of the best entry (lowest on equal scores)
  int pad[3];
};

__device__ __forceinline__ void sm_merge(float& m, float& s, float m2, float s2) {
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

__device__ __forceinline__ void g_merge(float& gs, int& gi, float& gy, float gs2, int gi2,
                                        float gy2) {
  if (gs2 > gs || (gs2 == gs && gi2 < gi)) {
    gs = gs2;
    gi = gi2;
    gy = gy2;
  }
}

template <typename T>
__device__ __forceinline__ void load4(const T* p, bool vec, float (&x)[4], int n) {
  if (vec && n == 4) {
    if (sizeof(T) == 2) {
      const uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = to_f(e[k]);
    } else {
      const float4 u = __ldcs(reinterpret_cast<const float4*>(p));
      x[0] = u.x;
      x[1] = u.y;
      x[2] = u.z;
      x[3] = u.w;
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = k < n ? to_f(p[k]) : -INFINITY;
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(kSdThreads, 4)
    sd_draw_kernel(const T* __restrict__ q, const int32_t* __restrict__ lm_rows,
                   const int32_t* __restrict__ req_valid, int B, int V, int step, float inv_tau,
                   int chunk, int chunks, SdPart* __restrict__ part, unsigned* __restrict__ cnt,
                   int32_t* __restrict__ tok, float* __restrict__ conf, uint64_t seed,
                   uint64_t offset) {
  pdl_trigger();
  pdl_wait();
  __shared__ SdPart s_p[kSdThreads / 32];
  __shared__ int s_last;
  const int row = blockIdx.y, c = blockIdx.x;
  const int pos = lm_rows[row];  // r * B + j
  const int r = pos / B, j = pos % B;
  float m = -INFINITY, s = 0.f, gs = -INFINITY, gy = 0.f;
  int gi = 0x7fffffff;
  if (req_valid == nullptr || req_valid[r]) {
    const T* y = q + (size_t)pos * V;
    const uint64_t n0 = ((uint64_t)step * B + j) * (uint64_t)V;
    const float c2 = inv_tau * kLog2e;
    const int v0 = c * chunk, v1 = min(V, v0 + chunk);  // chunk is a multiple of 4
    // groups of 4 consecutive entries; their draws n0 + vb .. n0 + vb + 3 lie in
    // one Philox block when n0 % 4 == 0, else in two.  Each thread visits its
    // groups in increasing order, so '>' keeps the lowest id on equal scores.
    for (int g = v0 / 4 + threadIdx.x; g * 4 < v1; g += kSdThreads) {
      const int vb = g * 4, n = min(4, v1 - vb);
      float x[4];
      load4<T>(y + vb, VEC, x, n);
      const uint64_t na = n0 + (uint64_t)vb;
      // VEC launches have V % 4 == 0, so n0 % 4 == 0 and every group is one block
      const int sh = VEC ? 0 : (int)(na & 3u);
      uint64_t wa[4], wb[4] = {0, 0, 0, 0};
      philox_block(seed, offset, r, kSdStream, na >> 2, wa);
      if (!VEC && sh != 0) philox_block(seed, offset, r, kSdStream, (na >> 2) + 1, wb);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k >= n) break;
        // word sh + k of the two blocks, chosen by selects (a register index)
        uint64_t w = wa[k];
        if (!VEC) {
          const uint64_t c1 = k < 3 ? wa[k + 1] : wb[k - 3];
          const uint64_t c2w = k < 2 ? wa[k + 2] : wb[k - 2];
          const uint64_t c3 = k < 1 ? wa[k + 3] : wb[k - 1];
          w = sh == 1 ? c1 : sh == 2 ? c2w : sh == 3 ? c3 : w;
        }
        const float t2 = x[k] * kLog2e;
        if (t2 > m) {
          s = (m == -INFINITY) ? 1.f : s * exp2f(m - t2) + 1.f;
          m = t2;
        } else {
          s += ex2_ftz(t2 - m);
        }
        const float sc = fmaf(x[k], c2, gumbel2_of(w));  // (Y / tau + G) log2 e
        if (sc > gs) {
          gs = sc;
          gi = vb + k;
          gy = x[k];
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sm_merge(m, s, __shfl_xor_sync(0xffffffffu, m, o), __shfl_xor_sync(0xffffffffu, s, o));
    g_merge(gs, gi, gy, __shfl_xor_sync(0xffffffffu, gs, o), __shfl_xor_sync(0xffffffffu, gi, o),
            __shfl_xor_sync(0xffffffffu, gy, o));
  }
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) s_p[w] = SdPart{m, s, gs, gy, gi, {0, 0, 0}};
  __syncthreads();
  if (threadIdx.x == 0) {
    SdPart b = s_p[0];
    for (int k = 1; k < kSdThreads / 32; ++k) {
      sm_merge(b.m, b.s, s_p[k].m, s_p[k].s);
      g_merge(b.gs, b.gi, b.gy, s_p[k].gs, s_p[k].gi, s_p[k].gy);
    }
    part[(size_t)row * chunks + c] = b;
    __threadfence();  // the partial is visible before this CTA is counted
    s_last = atomicAdd(&cnt[row], 1u) == (unsigned)(chunks - 1);
  }
  __syncthreads();
  if (!s_last || threadIdx.x >= 32) return;
  __threadfence();  // every counted partial of the row is visible to the reads below
  float M = -INFINITY, S = 0.f, GS = -INFINITY, GY = 0.f;
  int GI = 0x7fffffff;
  for (int k = lane; k < chunks; k += 32) {
    const SdPart* p = part + (size_t)row * chunks + k;
    sm_merge(M, S, __ldcg(&p->m), __ldcg(&p->s));
    g_merge(GS, GI, GY, __ldcg(&p->gs), __ldcg(&p->gi), __ldcg(&p->gy));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sm_merge(M, S, __shfl_xor_sync(0xffffffffu, M, o), __shfl_xor_sync(0xffffffffu, S, o));
    g_merge(GS, GI, GY, __shfl_xor_sync(0xffffffffu, GS, o), __shfl_xor_sync(0xffffffffu, GI, o),
            __shfl_xor_sync(0xffffffffu, GY, o));
  }
  if (lane == 0) {
    if (GI >= 0 && GI < V) {
      tok[row] = GI;
      conf[row] = exp2f(GY * kLog2e - M) / S;
    } else {  // no finite entry (a request that writes nothing): a valid id, zero confidence
      tok[row] = 0;
      conf[row] = 0.f;
    }
    cnt[row] = 0;  // ready for the next launch
  }
}

}  // namespace

int sampled_draw_chunks(int rows, int V) {
  // about four CTAs per SM over all rows, chunks of at least 4096 entries
  const int target = (4 * 148 + rows - 1) / rows;
  const int max_c = (V + 4095) / 4096;
  int c = target < max_c ? target : max_c;
  if (c > kSdMaxChunks) c = kSdMaxChunks;
  return c < 1 ? 1 : c;
}

size_t sampled_draw_part_bytes(int rows, int chunks) {
  return (size_t)rows * chunks * sizeof(SdPart);
}

int launch_sampled_draw(const void* q, int q_bf16, const int32_t* lm_rows,
                        const int32_t* req_valid, int rows, int B, int V, int step, float tau,
                        uint64_t seed, uint64_t offset, int32_t* tok, float* conf, void* part,
                        int chunks, unsigned* cnt, cudaStream_t s) {
  if (rows <= 0) return DFLASH_OK;
  const int esz = q_bf16 ? 2 : 4;
  const bool vec = V % 4 == 0 && (reinterpret_cast<uintptr_t>(q) % (4 * esz)) == 0;
  const float inv_tau = 1.f / tau;
  SdPart* p = static_cast<SdPart*>(part);
  // `chunks` is what the partials were sized for; a launch takes no more
  // chunks than fill the kernel's resident slots once
  static int slots[2][2] = {};  // [bf16][vec]
  auto fit = [&](auto kernel) {
    int& sl = slots[q_bf16 ? 1 : 0][vec ? 1 : 0];
    if (sl == 0) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kSdThreads, 0) !=
              cudaSuccess || per_sm < 1)
        per_sm = 1;
      sl = per_sm * num_sms();
    }
    const int c = sl / rows;
    return c < 1 ? 1 : (c < chunks ? c : chunks);
  };
  TimedScope ts(s, TC_ROW);
  cudaError_t e;
  auto go = [&](auto kernel, auto x) {
    const int c = fit(kernel);
    int chunk = (V + c - 1) / c;
    chunk = (chunk + 63) / 64 * 64;
    return launch_pdl(kernel, dim3(c, rows), dim3(kSdThreads), 0, s, 1, x, lm_rows, req_valid, B,
                      V, step, inv_tau, chunk, c, p, cnt, tok, conf, seed, offset);
  };
  if (q_bf16) {
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(q);
    e = go(vec ? sd_draw_kernel<__nv_bfloat16, true> : sd_draw_kernel<__nv_bfloat16, false>, x);
  } else {
    const float* x = static_cast<const float*>(q);
    e = go(vec ? sd_draw_kernel<float, true> : sd_draw_kernel<float, false>, x);
  }
  return e == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
