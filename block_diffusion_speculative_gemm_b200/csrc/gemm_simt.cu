// fp32 SIMT GEMM for the fp32 (small, correctness-oriented) model type.
// out[m][n] = sum_k X[m][k] * W[n][k] with X split into K segments; fp32
// accumulation in a fixed order (k ascending), one thread per output.
#include "common.cuh"
#include "internal.h"

namespace dflash {

struct SegPtrs {
  const float* p[kMaxSeg];
};

__global__ void gemm_simt_f32_kernel(const float* __restrict__ W, int N, int K, SegPtrs xs,
                                     int seg_k, int M, float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float xrow[];  // one token row of X (K floats)
  const int m = blockIdx.y;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const int seg = k / seg_k;
    xrow[k] = xs.p[seg][(size_t)m * seg_k + (k - seg * seg_k)];
  }
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const float* w = W + (size_t)n * K;
  float acc = 0.f;
  for (int k = 0; k < K; ++k) acc = fmaf(w[k], xrow[k], acc);
  out[(size_t)m * N + n] = acc;
}

void gemm_simt_f32(const float* W, int N, int K, const float* const* xseg, int n_seg, int seg_k,
                   int M, float* out, cudaStream_t s) {
  if (M <= 0) return;
  SegPtrs xs;
  for (int i = 0; i < kMaxSeg; ++i) xs.p[i] = i < n_seg ? xseg[i] : nullptr;
  dim3 grid((N + 127) / 128, M);
  TimedScope ts(s, TC_GEMM);
  launch_pdl(gemm_simt_f32_kernel, dim3(grid), dim3(128), (size_t)K * sizeof(float), s, 1, W, N, K,
      xs, seg_k, M, out);
}

}  // namespace dflash
