// The split-KV chunk combine shared by the tensor-core attention kernels: the
// last chunk CTA of a (request, kv head) merges every chunk's (m, l, O)
// partial into the output rows, o = sum_c w_c O_c with
// w_c = exp(m_c - M) / sum_c' exp(m_c' - M) l_c', chunks in order.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace dflash {

constexpr int kAttnMaxChunks = 64;  // split-KV chunks per request

// Every thread of the CTA calls it after writing (and fencing) its chunk's
// partial; `scratch` is shared memory of at least 2 * kAttnMaxChunks *
// kAttnMaxRows floats that nothing else uses any more.
template <int HD, int NTH>
__device__ void attn_chunk_combine(float* scratch, int r, int g, int R, int B, int G, int nq,
                                   int nkv, int Tc, int chunk, int n_chunks,
                                   const float* part_o, const float* part_ml, unsigned* cnt,
                                   __half* out) {
  const int tid = threadIdx.x;
  constexpr int kThreads = NTH;
  __shared__ int s_last;
  const int nvc = min(n_chunks, (Tc + B + chunk - 1) / chunk);  // chunks with keys
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&cnt[r * nkv + g], 1u) == (unsigned)(nvc - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();  // every counted chunk's partial is visible to the reads below
  const size_t base = ((size_t)r * nkv + g) * n_chunks * kAttnMaxRows;
  // every chunk's (m, l) of every row, fetched by all threads at once; the
  // chunk weights then replace the m values in place
  float* sml = scratch;  // [nvc][kAttnMaxRows][2]
  for (int idx = tid; idx < nvc * R; idx += kThreads) {
    const int cc = idx / R, row = idx % R;
    const float2 ml =
        __ldcg(reinterpret_cast<const float2*>(part_ml + (base + (size_t)cc * kAttnMaxRows + row) * 2));
    sml[(cc * kAttnMaxRows + row) * 2] = ml.x;
    sml[(cc * kAttnMaxRows + row) * 2 + 1] = ml.y;
  }
  __syncthreads();
  for (int row = tid; row < R; row += kThreads) {
    float M = -INFINITY;
    for (int cc = 0; cc < nvc; ++cc) M = fmaxf(M, sml[(cc * kAttnMaxRows + row) * 2]);
    float Lsum = 0.f;
    for (int cc = 0; cc < nvc; ++cc) {
      float* e = sml + (cc * kAttnMaxRows + row) * 2;
      const float w = expf(e[0] - M);
      e[0] = w;
      Lsum += w * e[1];
    }
    const float inv = 1.f / Lsum;
    for (int cc = 0; cc < nvc; ++cc) sml[(cc * kAttnMaxRows + row) * 2] *= inv;
  }
  __syncthreads();
  // output float4 i4 = (row, col): row = 4 i4 / HD; chunk cc's partial of it
  // sits cc * kAttnMaxRows * HD / 4 float4s after chunk 0's.  Each thread
  // keeps kU outputs and two chunks of loads in flight, so the merge waits
  // for about nvc / 2 memory round trips; chunks are summed in order.
  constexpr int kU = 8;
  const int total = R * HD / 4;
  const size_t cstride = (size_t)kAttnMaxRows * HD / 4;
  const float4* src0 = reinterpret_cast<const float4*>(part_o + base * HD);
  for (int i0 = tid; i0 < total; i0 += kThreads * kU) {
    float4 acc[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int cc = 0; cc < nvc; cc += 2) {
      float4 v[kU][2];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i4 = i0 + u * kThreads;
#pragma unroll
        for (int k = 0; k < 2; ++k)
          v[u][k] = (i4 < total && cc + k < nvc) ? __ldcg(src0 + (size_t)(cc + k) * cstride + i4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int row = ((i0 + u * kThreads) * 4) / HD;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          if (i0 + u * kThreads < total && cc + k < nvc) {
            const float w = sml[((cc + k) * kAttnMaxRows + row) * 2];
            acc[u].x += w * v[u][k].x;
            acc[u].y += w * v[u][k].y;
            acc[u].z += w * v[u][k].z;
            acc[u].w += w * v[u][k].w;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i4 = i0 + u * kThreads;
      if (i4 >= total) break;
      const int row = (i4 * 4) / HD, col = (i4 * 4) % HD;
      __half* dst = out + ((size_t)(r * B + row / G) * nq + g * G + row % G) * HD + col;
      *reinterpret_cast<__half2*>(dst) = __floats2half2_rn(acc[u].x, acc[u].y);
      *reinterpret_cast<__half2*>(dst + 2) = __floats2half2_rn(acc[u].z, acc[u].w);
    }
  }
  if (tid == 0) cnt[r * nkv + g] = 0;  // ready for the next launch
}

}  // namespace dflash
