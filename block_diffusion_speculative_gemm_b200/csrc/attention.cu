// Block-vs-context attention with split-KV.
//
// For request r and kv head g the B*G query rows of the block (G = nq/nkv
// query heads share one kv head) attend, without a mask, to the keys
// [context positions 0..T_r-1 from the cache] ++ [the block's own B keys]
// ("DFlash + Spec V2 深度解析", §2.3: the whole block is predicted in one
// forward).  The key axis is cut into chunks; each CTA (request, kv head,
// chunk) produces an online-softmax partial (row max m, row sum l, unnormalised
// o), merged over the chunks in ascending order.  fp16 models run the
// tensor-core kernel of attention_tc.cu, which merges its chunks itself; fp32
// models run the SIMT kernel below and the combine kernel after it.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace dflash {

constexpr int kAttnThreads = 128;
constexpr int kKeyTile = 32;
constexpr int kMaxRows = kAttnMaxRows;

template <typename T, typename TC, int HD>
__global__ void __launch_bounds__(kAttnThreads)
    attn_partial_kernel(const T* __restrict__ q, const T* __restrict__ kb,
                        const T* __restrict__ vb, const TC* __restrict__ kc,
                        const TC* __restrict__ vc, int layer, int batch, int cap,
                        const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ req_valid,
                        int B, int nq, int nkv, int chunk, int n_chunks,
                        float* __restrict__ part_o, float* __restrict__ part_ml) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPL = HD / 32;  // output elements per lane
  extern __shared__ float sm[];
  const int c = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int G = nq / nkv;
  const int R = B * G;
  const int Tc = req_valid[r] ? ctx_len[r] : 0;
  const int total = Tc + B;
  const int k0 = c * chunk;
  if (k0 >= total) return;
  const int k1 = min(total, k0 + chunk);

  float* q_s = sm;                       // [R][HD], pre-scaled by 1/sqrt(HD)
  float* k_s = q_s + kMaxRows * HD;      // [kKeyTile][HD + 1]
  float* v_s = k_s + kKeyTile * (HD + 1);  // [kKeyTile][HD]

  const float scale = rsqrtf((float)HD);
  for (int idx = threadIdx.x; idx < R * HD; idx += kAttnThreads) {
    const int row = idx / HD, e = idx % HD;
    const int j = row / G, head = g * G + row % G;
    q_s[idx] = to_f(q[((size_t)(r * B + j) * nq + head) * HD + e]) * scale;
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kMaxRowsPerWarp = kMaxRows / (kAttnThreads / 32);
  float m_i[kMaxRowsPerWarp], l_i[kMaxRowsPerWarp], o_i[kMaxRowsPerWarp][EPL];
#pragma unroll
  for (int t = 0; t < kMaxRowsPerWarp; ++t) {
    m_i[t] = -INFINITY;
    l_i[t] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o_i[t][e] = 0.f;
  }

  const size_t cache_base = (((size_t)layer * batch + r) * nkv + g) * (size_t)cap * HD;
  for (int kt = k0; kt < k1; kt += kKeyTile) {
    const int nk = min(kKeyTile, k1 - kt);
    __syncthreads();
    for (int idx = threadIdx.x; idx < kKeyTile * HD; idx += kAttnThreads) {
      const int kk = idx / HD, e = idx % HD;
      float kv = 0.f, vv = 0.f;
      if (kk < nk) {
        const int key = kt + kk;
        if (key < Tc) {
          kv = to_f(kc[cache_base + (size_t)key * HD + e]);
          vv = to_f(vc[cache_base + (size_t)key * HD + e]);
        } else {
          const size_t o = ((size_t)(r * B + key - Tc) * nkv + g) * HD + e;
          kv = to_f(kb[o]);
          vv = to_f(vb[o]);
        }
      }
      k_s[kk * (HD + 1) + e] = kv;
      v_s[kk * HD + e] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kMaxRowsPerWarp; ++t) {
      const int row = warp + 4 * t;
      if (row >= R) break;
      float s = -INFINITY;
      if (lane < nk) {
        const float* qr = q_s + row * HD;
        const float* kr = k_s + lane * (HD + 1);
        float acc = 0.f;
#pragma unroll 16
        for (int e = 0; e < HD; ++e) acc = fmaf(qr[e], kr[e], acc);
        s = acc;
      }
      const float mt = warp_max(s);
      const float mn = fmaxf(m_i[t], mt);
      const float p = (lane < nk) ? expf(s - mn) : 0.f;
      const float corr = expf(m_i[t] - mn);
      l_i[t] = l_i[t] * corr + warp_sum(p);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o_i[t][e] *= corr;
      for (int kk = 0; kk < nk; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
        for (int e = 0; e < EPL; ++e) o_i[t][e] = fmaf(pk, v_s[kk * HD + lane + 32 * e], o_i[t][e]);
      }
      m_i[t] = mn;
    }
  }

  const size_t pbase = (((size_t)r * nkv + g) * n_chunks + c) * kMaxRows;
#pragma unroll
  for (int t = 0; t < kMaxRowsPerWarp; ++t) {
    const int row = warp + 4 * t;
    if (row >= R) break;
#pragma unroll
    for (int e = 0; e < EPL; ++e) part_o[(pbase + row) * HD + lane + 32 * e] = o_i[t][e];
    if (lane == 0) {
      part_ml[(pbase + row) * 2 + 0] = m_i[t];
      part_ml[(pbase + row) * 2 + 1] = l_i[t];
    }
  }
}

// Merge of the split-KV partials of one (kv head, request): for query row i,
// o_i = sum_c exp(m_ci - M_i) o_ci / sum_c exp(m_ci - M_i) l_ci with
// M_i = max_c m_ci, chunks in ascending order.  The per-(chunk, row) weights
// are computed once into shared memory, then the CTA streams the [R][HD]
// partial blocks with 16-byte loads.
constexpr int kCombineThreads = 256;
constexpr int kMaxChunksC = 64;

template <typename T, int HD>
__global__ void __launch_bounds__(kCombineThreads)
    attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                        const int32_t* __restrict__ ctx_len,
                        const int32_t* __restrict__ req_valid, int B, int nq, int nkv, int chunk,
                        int n_chunks, T* __restrict__ o) {
  pdl_trigger();
  pdl_wait();
  __shared__ float wgt[kMaxChunksC * kMaxRows];
  const int g = blockIdx.x, r = blockIdx.y;
  const int G = nq / nkv, R = B * G;
  const int T_r = req_valid[r] ? ctx_len[r] : 0;
  const int nc = min(n_chunks, (T_r + B + chunk - 1) / chunk);
  const size_t base = ((size_t)r * nkv + g) * n_chunks * kMaxRows;
  for (int row = threadIdx.x; row < R; row += blockDim.x) {
    float M = -INFINITY;
    for (int c = 0; c < nc; ++c) M = fmaxf(M, part_ml[(base + (size_t)c * kMaxRows + row) * 2]);
    float L = 0.f;
    for (int c = 0; c < nc; ++c) {
      const size_t pr = base + (size_t)c * kMaxRows + row;
      const float w = expf(part_ml[pr * 2] - M);
      wgt[c * kMaxRows + row] = w;
      L += w * part_ml[pr * 2 + 1];
    }
    const float inv = 1.f / L;
    for (int c = 0; c < nc; ++c) wgt[c * kMaxRows + row] *= inv;
  }
  __syncthreads();
  for (int i4 = threadIdx.x; i4 < R * HD / 4; i4 += blockDim.x) {
    const int row = (i4 * 4) / HD, col = (i4 * 4) % HD;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < nc; ++c) {
      const float w = wgt[c * kMaxRows + row];
      const float4 v = *reinterpret_cast<const float4*>(
          part_o + (base + (size_t)c * kMaxRows + row) * HD + col);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    T* dst = o + ((size_t)(r * B + row / G) * nq + g * G + row % G) * HD + col;
    dst[0] = from_f<T>(acc.x);
    dst[1] = from_f<T>(acc.y);
    dst[2] = from_f<T>(acc.z);
    dst[3] = from_f<T>(acc.w);
  }
}

template <typename T, typename TC>
int launch_block_attention(const T* q, const T* kb, const T* vb, const TC* kc, const TC* vc,
                           const KvPages& pages, int layer, int L, int batch, int cap,
                           const int32_t* ctx_len, const int32_t* req_valid, int B, int nq,
                           int nkv, int hd, float* part_o, float* part_ml, int n_chunks, int chunk,
                           const int32_t* plan_dev, const int32_t* seg_start, T* o,
                           unsigned* cnt, int32_t* err, cudaStream_t s) {
  if (B * (nq / nkv) > kMaxRows) return DFLASH_EUNSUPPORTED;
  dim3 grid(n_chunks, nkv, batch);
  if constexpr (std::is_same<T, __half>::value) {
    // the tensor-core kernel merges its chunks itself
    return launch_attn_tc(q, kb, vb, kc, vc, pages, layer, batch, cap, ctx_len, req_valid, B, nq, nkv,
                          hd, L, chunk, plan_dev, n_chunks, seg_start, part_o, part_ml, cnt, o,
                          err, s);
  } else {
    if (pages.table != nullptr || seg_start != nullptr || plan_dev != nullptr)
      return DFLASH_EUNSUPPORTED;
    {
      TimedScope ts(s, TC_ATTN);
      if (hd == 128) {
        const size_t sm = (kMaxRows * 128 + kKeyTile * 129 + kKeyTile * 128) * sizeof(float);
        cudaFuncSetAttribute(attn_partial_kernel<T, TC, 128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        launch_pdl(attn_partial_kernel<T, TC, 128>, dim3(grid), dim3(kAttnThreads), sm, s, 1, q,
            kb, vb, kc, vc, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, chunk, n_chunks,
            part_o, part_ml);
      } else if (hd == 64) {
        const size_t sm = (kMaxRows * 64 + kKeyTile * 65 + kKeyTile * 64) * sizeof(float);
        launch_pdl(attn_partial_kernel<T, TC, 64>, dim3(grid), dim3(kAttnThreads), sm, s, 1, q,
            kb, vb, kc, vc, layer, batch, cap, ctx_len, req_valid, B, nq, nkv, chunk, n_chunks,
            part_o, part_ml);
      } else {
        return DFLASH_EUNSUPPORTED;
      }
    }
    TimedScope ts(s, TC_ATTN);
    if (n_chunks > kMaxChunksC) return DFLASH_EUNSUPPORTED;
    dim3 g2(nkv, batch);
    if (hd == 128)
      launch_pdl(attn_combine_kernel<T, 128>, dim3(g2), dim3(kCombineThreads), 0, s, 1, part_o,
          part_ml, ctx_len, req_valid, B, nq, nkv, chunk, n_chunks, o);
    else
      launch_pdl(attn_combine_kernel<T, 64>, dim3(g2), dim3(kCombineThreads), 0, s, 1, part_o,
          part_ml, ctx_len, req_valid, B, nq, nkv, chunk, n_chunks, o);
    return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
  }
}

template int launch_block_attention<float, float>(const float*, const float*, const float*,
                                                  const float*, const float*, const KvPages&, int,
                                                  int, int, int, const int32_t*, const int32_t*,
                                                  int, int, int, int, float*, float*, int, int,
                                                  const int32_t*, const int32_t*, float*, unsigned*,
                                                  int32_t*, cudaStream_t);
template int launch_block_attention<__half, __half>(const __half*, const __half*, const __half*,
                                                    const __half*, const __half*, const KvPages&,
                                                    int, int, int, int, const int32_t*,
                                                    const int32_t*, int, int, int, int, float*,
                                                    float*, int, int, const int32_t*,
                                                    const int32_t*, __half*, unsigned*, int32_t*,
                                                    cudaStream_t);

}  // namespace dflash
