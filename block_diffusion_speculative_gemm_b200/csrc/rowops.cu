// Row-wise kernels of the draft hot path: split-K reduction of GEMM partials
// fused with the elementwise step that follows each projection (RMSNorm,
// residual add, RoPE, SwiGLU, K/V cache scatter).  All are memory-bound; one
// CTA per token row (or per row and column block), fp32 arithmetic, splits
// summed in ascending order so results do not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace dflash {

constexpr int kRowThreads = 256;
constexpr int kMaxRowElems = 16;  // d <= 4096 per 256 threads

__device__ __forceinline__ float sum_splits(const float* part, int splits, size_t stride,
                                            size_t idx) {
  float v = part[idx];
  for (int s = 1; s < splits; ++s) v += part[(size_t)s * stride + idx];
  return v;
}

// ---------------------------------------------------------------- embedding + RMSNorm
// x[m] = emb[tokens[m]] (fp32 residual stream); h[m] = RMSNorm(x[m]; g).
template <typename TE, typename T>
__global__ void __launch_bounds__(kRowThreads)
    embed_norm_kernel(const int32_t* __restrict__ tokens, const TE* __restrict__ emb,
                      const float* __restrict__ g, float* __restrict__ x, T* __restrict__ h, int d,
                      float eps) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  const int tok = tokens[m];
  const TE* e = emb + (size_t)tok * d;
  float v[kMaxRowElems];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    v[i] = c < d ? to_f(e[c]) : 0.f;
    ss += v[i] * v[i];
  }
  const float inv = rsqrtf(block_sum(ss, red) / d + eps);
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < d) {
      x[(size_t)m * d + c] = v[i];
      h[(size_t)m * d + c] = from_f<T>(v[i] * inv * g[c]);
    }
  }
}

template <typename TE, typename T>
void launch_embed_norm(const int32_t* tokens, const TE* emb, const float* g, float* x, T* h, int M,
                       int d, float eps, cudaStream_t s) {
  if (M <= 0) return;
  TimedScope ts(s, TC_ROW);
  embed_norm_kernel<TE, T><<<M, kRowThreads, 0, s>>>(tokens, emb, g, x, h, d, eps);
}

// ---------------------------------------------------------------- residual + RMSNorm
// x[m] += sum_s part[s][m]; h[out_row[m]] = RMSNorm(x[m]; g) (all rows when
// out_row is null; rows with out_row < 0 are not written).
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
    residual_norm_kernel(const float* __restrict__ part, int splits, int M, int d,
                         float* __restrict__ x, const float* __restrict__ g, T* __restrict__ h,
                         const int32_t* __restrict__ out_row, float eps) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  const size_t stride = (size_t)M * d;
  float v[kMaxRowElems];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < d) {
      const size_t idx = (size_t)m * d + c;
      v[i] = x[idx] + sum_splits(part, splits, stride, idx);
      x[idx] = v[i];
    } else {
      v[i] = 0.f;
    }
    ss += v[i] * v[i];
  }
  const float inv = rsqrtf(block_sum(ss, red) / d + eps);
  const int orow = out_row ? out_row[m] : m;
  if (orow < 0) return;
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < d) h[(size_t)orow * d + c] = from_f<T>(v[i] * inv * g[c]);
  }
}

template <typename T>
void launch_residual_norm(const float* part, int splits, int M, int d, float* x, const float* g,
                          T* h, const int32_t* out_row, float eps, cudaStream_t s) {
  if (M <= 0) return;
  TimedScope ts(s, TC_ROW);
  residual_norm_kernel<T><<<M, kRowThreads, 0, s>>>(part, splits, M, d, x, g, h, out_row, eps);
}

// ---------------------------------------------------------------- context-feature RMSNorm
// c[n] = RMSNorm(sum_s part[s][n]; g)
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
    ctx_norm_kernel(const float* __restrict__ part, int splits, int n_rows, int d,
                    const float* __restrict__ g, T* __restrict__ c, float eps) {
  __shared__ float red[32];
  const int n = blockIdx.x;
  const size_t stride = (size_t)n_rows * d;
  float v[kMaxRowElems];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int col = threadIdx.x + i * kRowThreads;
    v[i] = col < d ? sum_splits(part, splits, stride, (size_t)n * d + col) : 0.f;
    ss += v[i] * v[i];
  }
  const float inv = rsqrtf(block_sum(ss, red) / d + eps);
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int col = threadIdx.x + i * kRowThreads;
    if (col < d) c[(size_t)n * d + col] = from_f<T>(v[i] * inv * g[col]);
  }
}

template <typename T>
void launch_ctx_norm(const float* part, int splits, int n, int d, const float* g, T* c, float eps,
                     cudaStream_t s) {
  if (n <= 0) return;
  TimedScope ts(s, TC_ROW);
  ctx_norm_kernel<T><<<n, kRowThreads, 0, s>>>(part, splits, n, d, g, c, eps);
}

// ---------------------------------------------------------------- QKV epilogue
// part columns: [q heads | k heads | v heads], each head hd wide.  q and k get
// rotate-half RoPE at position ctx_len[r] + j; v is copied.  One thread per
// (head, rotation pair).
template <typename T>
__global__ void qkv_post_kernel(const float* __restrict__ part, int splits, int M, int B,
                                const int32_t* __restrict__ ctx_len,
                                const int32_t* __restrict__ req_valid, int nq, int nkv, int hd,
                                const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                                T* __restrict__ q, T* __restrict__ kb, T* __restrict__ vb) {
  const int m = blockIdx.y;
  const int half = hd / 2;
  const int nh = nq + 2 * nkv;
  const int N = nh * hd;
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= nh * half) return;
  const int head = p / half, i = p % half;
  const int r = m / B, j = m % B;
  const int pos = (req_valid[r] ? ctx_len[r] : 0) + j;
  const size_t stride = (size_t)M * N;
  const size_t c0 = (size_t)m * N + head * hd + i;
  const float x1 = sum_splits(part, splits, stride, c0);
  const float x2 = sum_splits(part, splits, stride, c0 + half);
  if (head < nq + nkv) {
    const float c = cos_t[(size_t)pos * half + i], s = sin_t[(size_t)pos * half + i];
    const float y1 = x1 * c - x2 * s, y2 = x2 * c + x1 * s;
    T* dst = head < nq ? q + ((size_t)m * nq + head) * hd : kb + ((size_t)m * nkv + head - nq) * hd;
    dst[i] = from_f<T>(y1);
    dst[i + half] = from_f<T>(y2);
  } else {
    T* dst = vb + ((size_t)m * nkv + head - nq - nkv) * hd;
    dst[i] = from_f<T>(x1);
    dst[i + half] = from_f<T>(x2);
  }
}

template <typename T>
void launch_qkv_post(const float* part, int splits, int M, int B, const int32_t* ctx_len,
                     const int32_t* req_valid, int nq, int nkv, int hd, const float* cos_t,
                     const float* sin_t, T* q, T* kb, T* vb, cudaStream_t s) {
  if (M <= 0) return;
  const int pairs = (nq + 2 * nkv) * hd / 2;
  dim3 grid((pairs + 255) / 256, M);
  TimedScope ts(s, TC_ROW);
  qkv_post_kernel<T><<<grid, 256, 0, s>>>(part, splits, M, B, ctx_len, req_valid, nq, nkv, hd,
                                          cos_t, sin_t, q, kb, vb);
}

// ---------------------------------------------------------------- SwiGLU
// part columns: [gate (I) | up (I)]; act = silu(gate) * up.
template <typename T>
__global__ void swiglu_kernel(const float* __restrict__ part, int splits, int M, int I,
                              T* __restrict__ act) {
  const int m = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= I) return;
  const size_t stride = (size_t)M * 2 * I;
  const float g = sum_splits(part, splits, stride, (size_t)m * 2 * I + i);
  const float u = sum_splits(part, splits, stride, (size_t)m * 2 * I + I + i);
  act[(size_t)m * I + i] = from_f<T>(g / (1.f + expf(-g)) * u);
}

template <typename T>
void launch_swiglu(const float* part, int splits, int M, int I, T* act, cudaStream_t s) {
  if (M <= 0) return;
  dim3 grid((I + 255) / 256, M);
  TimedScope ts(s, TC_ROW);
  swiglu_kernel<T><<<grid, 256, 0, s>>>(part, splits, M, I, act);
}

// ---------------------------------------------------------------- K/V cache scatter
// part columns: for each layer l: [K heads (nkv*hd) | V heads (nkv*hd)].
// Row n belongs to request r with cu_rows[r] <= n < cu_rows[r+1]; its position
// is start_pos[r] + n - cu_rows[r].  K gets RoPE at that position.
template <typename T>
__global__ void kv_scatter_kernel(const float* __restrict__ part, int splits, int n_rows,
                                  int row0, int L, int nkv, int hd, const int32_t* __restrict__ cu_rows,
                                  const int32_t* __restrict__ start_pos, int batch, int cap,
                                  const float* __restrict__ cos_t,
                                  const float* __restrict__ sin_t, int max_pos,
                                  T* __restrict__ kc, T* __restrict__ vc, int32_t* err) {
  const int nl = blockIdx.y;       // row inside this chunk (partials)
  const int n = row0 + nl;         // row of the whole call (cu_rows)
  const int half = hd / 2;
  const int per_layer = 2 * nkv * half;  // pairs per layer (K and V)
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= L * per_layer) return;
  // request of row n: last r with cu_rows[r] <= n
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu_rows[mid] <= n) lo = mid; else hi = mid - 1;
  }
  const int r = lo;
  if (n < cu_rows[r] || n >= cu_rows[r + 1]) {
    if (p == 0) set_error(err, DFLASH_DEV_ROWS);
    return;
  }
  const int pos = start_pos[r] + (n - cu_rows[r]);
  if (pos < 0 || pos >= cap || pos >= max_pos) {
    if (p == 0) set_error(err, DFLASH_DEV_CTX_CAP);
    return;
  }
  const int l = p / per_layer;
  const int q = p % per_layer;
  const bool is_v = q >= nkv * half;
  const int qq = is_v ? q - nkv * half : q;
  const int head = qq / half, i = qq % half;
  const int N = L * 2 * nkv * hd;
  const size_t stride = (size_t)n_rows * N;
  const size_t c0 = (size_t)nl * N + (size_t)l * 2 * nkv * hd + (is_v ? nkv * hd : 0) + head * hd + i;
  float x1 = sum_splits(part, splits, stride, c0);
  float x2 = sum_splits(part, splits, stride, c0 + half);
  if (!is_v) {
    const float c = cos_t[(size_t)pos * half + i], s = sin_t[(size_t)pos * half + i];
    const float y1 = x1 * c - x2 * s, y2 = x2 * c + x1 * s;
    x1 = y1;
    x2 = y2;
  }
  T* dst = (is_v ? vc : kc) + ((((size_t)l * batch + r) * nkv + head) * cap + pos) * hd;
  dst[i] = from_f<T>(x1);
  dst[i + half] = from_f<T>(x2);
}

template <typename T>
void launch_kv_scatter(const float* part, int splits, int n_rows, int row0, int L, int nkv,
                       int hd, const int32_t* cu_rows, const int32_t* start_pos, int batch, int cap,
                       const float* cos_t, const float* sin_t, int max_pos, T* kc, T* vc,
                       int32_t* err, cudaStream_t s) {
  if (n_rows <= 0) return;
  const int pairs = L * 2 * nkv * hd / 2;
  dim3 grid((pairs + 255) / 256, n_rows);
  TimedScope ts(s, TC_ROW);
  kv_scatter_kernel<T><<<grid, 256, 0, s>>>(part, splits, n_rows, row0, L, nkv, hd, cu_rows, start_pos,
                                            batch, cap, cos_t, sin_t, max_pos, kc, vc, err);
}

// T: activation type (GEMM operand); TC: K/V cache type; TE: embedding type.
#define DFLASH_INST_A(T)                                                                         \
  template void launch_residual_norm<T>(const float*, int, int, int, float*, const float*, T*,   \
                                        const int32_t*, float, cudaStream_t);                    \
  template void launch_ctx_norm<T>(const float*, int, int, int, const float*, T*, float,         \
                                   cudaStream_t);                                                \
  template void launch_qkv_post<T>(const float*, int, int, int, const int32_t*, const int32_t*,  \
                                   int, int, int, const float*, const float*, T*, T*, T*,        \
                                   cudaStream_t);                                                \
  template void launch_swiglu<T>(const float*, int, int, int, T*, cudaStream_t);
#define DFLASH_INST_C(TC)                                                                        \
  template void launch_kv_scatter<TC>(const float*, int, int, int, int, int, int,                \
                                      const int32_t*, const int32_t*, int, int, const float*,    \
                                      const float*, int, TC*, TC*, int32_t*, cudaStream_t);

DFLASH_INST_A(float)
DFLASH_INST_A(__half)
DFLASH_INST_C(float)
DFLASH_INST_C(__half)
template void launch_embed_norm<float, float>(const int32_t*, const float*, const float*, float*,
                                              float*, int, int, float, cudaStream_t);
template void launch_embed_norm<__nv_bfloat16, __half>(const int32_t*, const __nv_bfloat16*,
                                                       const float*, float*, __half*, int, int,
                                                       float, cudaStream_t);

}  // namespace dflash
