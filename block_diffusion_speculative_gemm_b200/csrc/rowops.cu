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

// Sum of the K-split partials of 4 consecutive fp32 elements (16-byte aligned
// index), in ascending split order.  Partials are dead after this read.  Up to
// four splits, every load is issued before the first add, so a thread waits
// for one memory round trip instead of one per split.
__device__ __forceinline__ float4 sum_splits4(const float* part, int splits, size_t stride,
                                              size_t idx) {
  const float4* p = reinterpret_cast<const float4*>(part + idx);
  const size_t st4 = stride / 4;
  if (splits <= 4) {
    float4 w[4];
#pragma unroll
    for (int s = 0; s < 4; ++s)
      if (s < splits) w[s] = __ldcs(p + s * st4);
    float4 v = w[0];
#pragma unroll
    for (int s = 1; s < 4; ++s)
      if (s < splits) {
        v.x += w[s].x;
        v.y += w[s].y;
        v.z += w[s].z;
        v.w += w[s].w;
      }
    return v;
  }
  float4 v = __ldcs(p);
  for (int s = 1; s < splits; ++s) {
    const float4 w = __ldcs(p + s * st4);
    v.x += w.x;
    v.y += w.y;
    v.z += w.z;
    v.w += w.w;
  }
  return v;
}

// Once a warp has consumed its split sums, the partials are dead: the GEMM
// kept them in L2 (evict-last stores) for this read, and a dirty line left
// there costs a DRAM write when it is evicted later.  The lane whose 16-byte
// unit starts a 128-byte line drops that line of every split without writing
// it back (the next GEMM rewrites every partial it leaves).  Called by every
// lane after the warp's last use of the values; lines that are not 128-byte
// aligned are left alone.
__device__ __forceinline__ void discard_splits(const float* part, int splits, size_t stride,
                                               size_t idx) {
  if ((idx & 31) != 0) return;
  for (int s = 0; s < splits; ++s) {
    const float* line = part + idx + (size_t)s * stride;
    if ((reinterpret_cast<uintptr_t>(line) & 127) == 0)
      asm volatile("discard.global.L2 [%0], 128;" ::"l"(line) : "memory");
  }
}

// Stores four values; returns true when a value does not fit the element type
// (an fp16 store of a value that rounds past the largest finite fp16, or NaN).
template <typename T>
__device__ __forceinline__ bool store4(T* dst, float a, float b, float c, float d) {
  dst[0] = from_f<T>(a);
  dst[1] = from_f<T>(b);
  dst[2] = from_f<T>(c);
  dst[3] = from_f<T>(d);
  return narrow_bad<T>(a) || narrow_bad<T>(b) || narrow_bad<T>(c) || narrow_bad<T>(d);
}
template <>
__device__ __forceinline__ bool store4<__half>(__half* dst, float a, float b, float c, float d) {
  __half2 lo = __floats2half2_rn(a, b), hi = __floats2half2_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = u;
  return narrow_bad<__half>(a) || narrow_bad<__half>(b) || narrow_bad<__half>(c) ||
         narrow_bad<__half>(d);
}
template <>
__device__ __forceinline__ bool store4<float>(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
  return false;
}

// ---------------------------------------------------------------- embedding + RMSNorm
// x[m] = emb[tokens[m]] (fp32 residual stream); h[m] = RMSNorm(x[m]; g).
template <typename TE, typename T>
__global__ void __launch_bounds__(kRowThreads)
    embed_norm_kernel(const int32_t* __restrict__ tokens, const TE* __restrict__ emb,
                      const float* __restrict__ g, float* __restrict__ x, T* __restrict__ h, int d,
                      float eps, int32_t* err) {
  pdl_trigger();
  pdl_wait();
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
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kMaxRowElems; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < d) {
      x[(size_t)m * d + c] = v[i];
      const float y = v[i] * inv * g[c];
      h[(size_t)m * d + c] = from_f<T>(y);
      bad |= narrow_bad<T>(y);
    }
  }
  if (bad) set_error(err, DFLASH_DEV_RANGE);
}

template <typename TE, typename T>
void launch_embed_norm(const int32_t* tokens, const TE* emb, const float* g, float* x, T* h, int M,
                       int d, float eps, int32_t* err, cudaStream_t s) {
  if (M <= 0) return;
  TimedScope ts(s, TC_ROW);
  launch_pdl(embed_norm_kernel<TE, T>, dim3(M), dim3(kRowThreads), 0, s, 1, tokens, emb, g, x, h, d,
      eps, err);
}

// ---------------------------------------------------------------- residual + RMSNorm
// x[m] += sum_s part[s][m] (skipped when part is null); h[out_row[m]] =
// RMSNorm(x[m]; g) (all rows when out_row is null; rows with out_row < 0 are
// not written).
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
    residual_norm_kernel(const float* __restrict__ part, int splits, int M, int d,
                         float* __restrict__ x, const float* __restrict__ g, T* __restrict__ h,
                         const int32_t* __restrict__ out_row, float eps, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int m = blockIdx.x;
  const size_t stride = (size_t)M * d;
  constexpr int kV = kMaxRowElems / 4;  // float4 per thread
  float4 v[kV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kV; ++i) {
    const int c = (threadIdx.x + i * kRowThreads) * 4;
    if (c < d) {
      const size_t idx = (size_t)m * d + c;
      v[i] = *reinterpret_cast<const float4*>(x + idx);
      if (part != nullptr) {
        const float4 p = sum_splits4(part, splits, stride, idx);
        v[i].x += p.x;
        v[i].y += p.y;
        v[i].z += p.z;
        v[i].w += p.w;
        *reinterpret_cast<float4*>(x + idx) = v[i];
      }
    } else {
      v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  }
  const float inv = rsqrtf(block_sum(ss, red) / d + eps);  // every sum consumed
  if (part != nullptr) {
#pragma unroll
    for (int i = 0; i < kV; ++i) {
      const int c = (threadIdx.x + i * kRowThreads) * 4;
      if (c < d) discard_splits(part, splits, stride, (size_t)m * d + c);
    }
  }
  const int orow = out_row ? out_row[m] : m;
  if (orow < 0) return;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kV; ++i) {
    const int c = (threadIdx.x + i * kRowThreads) * 4;
    if (c < d) {
      const float4 gg = *reinterpret_cast<const float4*>(g + c);
      bad |= store4<T>(h + (size_t)orow * d + c, v[i].x * inv * gg.x, v[i].y * inv * gg.y,
                       v[i].z * inv * gg.z, v[i].w * inv * gg.w);
    }
  }
  if (bad) set_error(err, DFLASH_DEV_RANGE);
}

template <typename T>
void launch_residual_norm(const float* part, int splits, int M, int d, float* x, const float* g,
                          T* h, const int32_t* out_row, float eps, int32_t* err, cudaStream_t s) {
  if (M <= 0) return;
  TimedScope ts(s, TC_ROW);
  launch_pdl(residual_norm_kernel<T>, dim3(M), dim3(kRowThreads), 0, s, 1, part, splits, M, d, x, g,
      h, out_row, eps, err);
}

// ---------------------------------------------------------------- context-feature RMSNorm
// c[n] = RMSNorm(sum_s part[s][n]; g)
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
    ctx_norm_kernel(const float* __restrict__ part, int splits, int n_rows, int d,
                    const float* __restrict__ g, T* __restrict__ c, float eps, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int n = blockIdx.x;
  const size_t stride = (size_t)n_rows * d;
  constexpr int kV = kMaxRowElems / 4;
  float4 v[kV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kV; ++i) {
    const int col = (threadIdx.x + i * kRowThreads) * 4;
    v[i] = col < d ? sum_splits4(part, splits, stride, (size_t)n * d + col)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  }
  const float inv = rsqrtf(block_sum(ss, red) / d + eps);
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kV; ++i) {
    const int col = (threadIdx.x + i * kRowThreads) * 4;
    if (col < d) {
      const float4 gg = *reinterpret_cast<const float4*>(g + col);
      bad |= store4<T>(c + (size_t)n * d + col, v[i].x * inv * gg.x, v[i].y * inv * gg.y,
                       v[i].z * inv * gg.z, v[i].w * inv * gg.w);
    }
  }
  if (bad) set_error(err, DFLASH_DEV_RANGE);
}

template <typename T>
void launch_ctx_norm(const float* part, int splits, int n, int d, const float* g, T* c, float eps,
                     int32_t* err, cudaStream_t s) {
  if (n <= 0) return;
  TimedScope ts(s, TC_ROW);
  launch_pdl(ctx_norm_kernel<T>, dim3(n), dim3(kRowThreads), 0, s, 1, part, splits, n, d, g, c, eps,
             err);
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
                                int32_t* err,
                                T* __restrict__ q, T* __restrict__ kb, T* __restrict__ vb) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.y;
  const int half = hd / 2;
  const int nh = nq + 2 * nkv;
  const int N = nh * hd;
  const int p4 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;  // first of 4 pairs
  const bool live = p4 < nh * half;
  const int head = (live ? p4 : 0) / half, i = (live ? p4 : 0) % half;
  const int r = m / B, j = m % B;
  const int pos = (req_valid[r] ? ctx_len[r] : 0) + j;
  const size_t stride = (size_t)M * N;
  const size_t c0 = (size_t)m * N + head * hd + i;
  float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), x2 = x1;
  if (live) {
    x1 = sum_splits4(part, splits, stride, c0);
    x2 = sum_splits4(part, splits, stride, c0 + half);
  }
  T* dst = q;
  if (head < nq + nkv) {
    const float4 c = *reinterpret_cast<const float4*>(cos_t + (size_t)pos * half + i);
    const float4 sn = *reinterpret_cast<const float4*>(sin_t + (size_t)pos * half + i);
    const float4 y1 = make_float4(x1.x * c.x - x2.x * sn.x, x1.y * c.y - x2.y * sn.y,
                                  x1.z * c.z - x2.z * sn.z, x1.w * c.w - x2.w * sn.w);
    const float4 y2 = make_float4(x2.x * c.x + x1.x * sn.x, x2.y * c.y + x1.y * sn.y,
                                  x2.z * c.z + x1.z * sn.z, x2.w * c.w + x1.w * sn.w);
    x1 = y1;
    x2 = y2;
    dst = head < nq ? q + ((size_t)m * nq + head) * hd : kb + ((size_t)m * nkv + head - nq) * hd;
  } else {
    dst = vb + ((size_t)m * nkv + head - nq - nkv) * hd;
  }
  if (live) {
    const bool bad = store4<T>(dst + i, x1.x, x1.y, x1.z, x1.w) |
                     store4<T>(dst + i + half, x2.x, x2.y, x2.z, x2.w);
    if (bad) set_error(err, DFLASH_DEV_RANGE);
  }
  __syncwarp();  // every lane's stores used its loads
  if (live) {
    discard_splits(part, splits, stride, c0);
    discard_splits(part, splits, stride, c0 + half);
  }
}

template <typename T>
void launch_qkv_post(const float* part, int splits, int M, int B, const int32_t* ctx_len,
                     const int32_t* req_valid, int nq, int nkv, int hd, const float* cos_t,
                     const float* sin_t, T* q, T* kb, T* vb, int32_t* err, cudaStream_t s) {
  if (M <= 0) return;
  const int pairs = (nq + 2 * nkv) * hd / 2;
  dim3 grid((pairs / 4 + 255) / 256, M);
  TimedScope ts(s, TC_ROW);
  launch_pdl(qkv_post_kernel<T>, dim3(grid), dim3(256), 0, s, 1, part, splits, M, B, ctx_len,
      req_valid, nq, nkv, hd, cos_t, sin_t, err, q, kb, vb);
}

// ---------------------------------------------------------------- SwiGLU
// part columns: 128-column blocks of 64 gate outputs then the 64 up outputs
// of the same features; act = silu(gate) * up.
template <typename T>
__global__ void swiglu_kernel(const float* __restrict__ part, int splits, int M, int I,
                              T* __restrict__ act, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.y;
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) * 4;  // 4 features in one 64-block
  const bool live = i < I;
  const size_t stride = (size_t)M * 2 * I;
  const size_t gc = (size_t)m * 2 * I + (size_t)((live ? i : 0) >> 6) * 128 + ((live ? i : 0) & 63);
  if (live) {
    const float4 g = sum_splits4(part, splits, stride, gc);
    const float4 u = sum_splits4(part, splits, stride, gc + 64);
    const bool bad = store4<T>(act + (size_t)m * I + i, g.x / (1.f + expf(-g.x)) * u.x,
                               g.y / (1.f + expf(-g.y)) * u.y, g.z / (1.f + expf(-g.z)) * u.z,
                               g.w / (1.f + expf(-g.w)) * u.w);
    if (bad) set_error(err, DFLASH_DEV_RANGE);
  }
  __syncwarp();  // every lane's stores used its loads
  if (live) {
    discard_splits(part, splits, stride, gc);
    discard_splits(part, splits, stride, gc + 64);
  }
}

template <typename T>
void launch_swiglu(const float* part, int splits, int M, int I, T* act, int32_t* err,
                   cudaStream_t s) {
  if (M <= 0) return;
  dim3 grid((I / 4 + 255) / 256, M);
  TimedScope ts(s, TC_ROW);
  launch_pdl(swiglu_kernel<T>, dim3(grid), dim3(256), 0, s, 1, part, splits, M, I, act, err);
}

// ---------------------------------------------------------------- K/V cache scatter
// part columns: for each layer l: [K heads (nkv*hd) | V heads (nkv*hd)].
// Row n belongs to request r with cu_rows[r] <= n < cu_rows[r+1]; its position
// is start_pos[r] + n - cu_rows[r].  K gets RoPE at that position.
template <typename T>
__global__ void kv_scatter_kernel(const float* __restrict__ part, int splits, int n_rows,
                                  int row0, int L, int nkv, int hd, const int32_t* __restrict__ cu_rows,
                                  const int32_t* __restrict__ start_pos, int batch, int cap,
                                  const KvPages pg, const float* __restrict__ cos_t,
                                  const float* __restrict__ sin_t, int max_pos,
                                  T* __restrict__ kc, T* __restrict__ vc, int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int nl = blockIdx.y;       // row inside this chunk (partials)
  const int n = row0 + nl;         // row of the whole call (cu_rows)
  const int half = hd / 2;
  const int per_layer = 2 * nkv * half;  // pairs per layer (K and V)
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) * 4;  // first of 4 pairs
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
  if (pg.table != nullptr && !pg.req_ok[r]) return;  // the page check reported it
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
  float4 x1 = sum_splits4(part, splits, stride, c0);
  float4 x2 = sum_splits4(part, splits, stride, c0 + half);
  if (!is_v) {
    const float4 c = *reinterpret_cast<const float4*>(cos_t + (size_t)pos * half + i);
    const float4 sn = *reinterpret_cast<const float4*>(sin_t + (size_t)pos * half + i);
    const float4 y1 = make_float4(x1.x * c.x - x2.x * sn.x, x1.y * c.y - x2.y * sn.y,
                                  x1.z * c.z - x2.z * sn.z, x1.w * c.w - x2.w * sn.w);
    const float4 y2 = make_float4(x2.x * c.x + x1.x * sn.x, x2.y * c.y + x1.y * sn.y,
                                  x2.z * c.z + x1.z * sn.z, x2.w * c.w + x1.w * sn.w);
    x1 = y1;
    x2 = y2;
  }
  const long long drow = kv_row(pg, l, batch, r, nkv, head, cap, pos);
  [[maybe_unused]] const long long rows = (long long)L * nkv * (pg.table ? (long long)pg.n_pages * pg.page
                                                        : (long long)batch * cap);
  if (!DFLASH_CHECK(drow >= 0 && drow < rows, err)) return;
  T* dst = (is_v ? vc : kc) + (size_t)drow * hd;
  const bool bad = store4<T>(dst + i, x1.x, x1.y, x1.z, x1.w) |
                   store4<T>(dst + i + half, x2.x, x2.y, x2.z, x2.w);
  if (bad) set_error(err, DFLASH_DEV_RANGE);
}

template <typename T>
void launch_kv_scatter(const float* part, int splits, int n_rows, int row0, int L, int nkv,
                       int hd, const int32_t* cu_rows, const int32_t* start_pos, int batch, int cap,
                       const KvPages& pages, const float* cos_t, const float* sin_t, int max_pos,
                       T* kc, T* vc, int32_t* err, cudaStream_t s) {
  if (n_rows <= 0) return;
  const int pairs = L * 2 * nkv * hd / 2;
  dim3 grid((pairs / 4 + 255) / 256, n_rows);
  TimedScope ts(s, TC_ROW);
  launch_pdl(kv_scatter_kernel<T>, dim3(grid), dim3(256), 0, s, 1, part, splits, n_rows, row0, L,
      nkv, hd, cu_rows, start_pos, batch, cap, pages, cos_t, sin_t, max_pos, kc, vc, err);
}

// One warp per request: the pages holding its rows' positions must all be
// mapped (an entry in [0, n_pages) inside the request's table row); a request
// with an unmapped one writes nothing and reports DFLASH_DEV_PAGE.
__global__ void inject_page_check_kernel(const int32_t* __restrict__ cu_rows,
                                         const int32_t* __restrict__ start_pos, int batch,
                                         const KvPages pg, int32_t* __restrict__ req_ok,
                                         int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= batch) return;
  const int n = cu_rows[r + 1] - cu_rows[r];
  const int st = start_pos[r];
  bool bad = false;
  if (n > 0 && st >= 0) {
    const int p0 = st / pg.page;
    const long long last = ((long long)st + n - 1) / pg.page;
    for (long long k = p0 + lane; k <= last; k += 32) {
      const int e = k < pg.max_pages ? pg.table[(long long)r * pg.max_pages + k] : -1;
      bad |= e < 0 || e >= pg.n_pages;
    }
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    req_ok[r] = bad ? 0 : 1;
    if (bad) set_error(err, DFLASH_DEV_PAGE);
  }
}

void launch_inject_page_check(const int32_t* cu_rows, const int32_t* start_pos, int batch,
                              const KvPages& pages, int32_t* req_ok, int32_t* err,
                              cudaStream_t s) {
  TimedScope ts(s, TC_ROW);
  const int wpb = 4;
  launch_pdl(inject_page_check_kernel, dim3((batch + wpb - 1) / wpb), dim3(32 * wpb), 0, s, 1,
             cu_rows, start_pos, batch, pages, req_ok, err);
}

// T: activation type (GEMM operand); TC: K/V cache type; TE: embedding type.
#define DFLASH_INST_A(T)                                                                         \
  template void launch_residual_norm<T>(const float*, int, int, int, float*, const float*, T*,   \
                                        const int32_t*, float, int32_t*, cudaStream_t);          \
  template void launch_ctx_norm<T>(const float*, int, int, int, const float*, T*, float,         \
                                   int32_t*, cudaStream_t);                                      \
  template void launch_qkv_post<T>(const float*, int, int, int, const int32_t*, const int32_t*,  \
                                   int, int, int, const float*, const float*, T*, T*, T*,        \
                                   int32_t*, cudaStream_t);                                      \
  template void launch_swiglu<T>(const float*, int, int, int, T*, int32_t*, cudaStream_t);
#define DFLASH_INST_C(TC)                                                                        \
  template void launch_kv_scatter<TC>(const float*, int, int, int, int, int, int,                \
                                      const int32_t*, const int32_t*, int, int, const KvPages&,  \
                                      const float*, const float*, int, TC*, TC*, int32_t*,       \
                                      cudaStream_t);

DFLASH_INST_A(float)
DFLASH_INST_A(__half)
DFLASH_INST_C(float)
DFLASH_INST_C(__half)
template void launch_embed_norm<float, float>(const int32_t*, const float*, const float*, float*,
                                              float*, int, int, float, int32_t*, cudaStream_t);
template void launch_embed_norm<__nv_bfloat16, __half>(const int32_t*, const __nv_bfloat16*,
                                                       const float*, float*, __half*, int, int,
                                                       float, int32_t*, cudaStream_t);

}  // namespace dflash
