// Greedy verify ("DFlash：用“块扩散”魔法", §2 Flash Verification:
// decide_acceptance(logits, draft_block), read greedily).
//
// Kernel 1 (bandwidth-bound): every target-logit row is cut into chunks; a CTA
// scans one chunk with 16-byte loads and keeps (max, lowest index).  Kernel 2:
// one warp per request merges the chunk partials of its B rows (lane i = row
// i), finds the accept length with one ballot and writes the accepted tokens
// plus the bonus token behind out_len, then advances out_len and seq_lens.
// Comparisons are exact on the stored logit values, so the result does not
// depend on the chunking.
#include "common.cuh"
#include "internal.h"

namespace dflash {

constexpr int kVerifyThreads = 256;

struct ArgPart {
  float v;
  int32_t i;
};

template <typename T, bool VEC>
__global__ void __launch_bounds__(kVerifyThreads)
    verify_argmax_kernel(const T* __restrict__ logits, int V, int chunk, ArgPart* __restrict__ part) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_v[kVerifyThreads / 32];
  __shared__ int s_i[kVerifyThreads / 32];
  const int row = blockIdx.y, c = blockIdx.x;
  const int v0 = c * chunk;
  const int v1 = min(V, v0 + chunk);
  const T* x = logits + (size_t)row * V;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  if (VEC) {
    constexpr int W = 16 / sizeof(T);  // elements per 16-byte load (chunk is a multiple)
    const int nvec = (v1 - v0) / W;
    const uint4* p = reinterpret_cast<const uint4*>(x + v0);
    for (int t = threadIdx.x; t < nvec; t += kVerifyThreads) {
      uint4 u = __ldg(p + t);
      const T* e = reinterpret_cast<const T*>(&u);
      const int base = v0 + t * W;
#pragma unroll
      for (int k = 0; k < W; ++k) {
        const float f = to_f(e[k]);
        if (f > best) { best = f; bi = base + k; }
      }
    }
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
  if (threadIdx.x == 0) {
    best = s_v[0];
    bi = s_i[0];
    for (int k = 1; k < kVerifyThreads / 32; ++k) argmax_merge(best, bi, s_v[k], s_i[k]);
    part[(size_t)row * gridDim.x + c] = ArgPart{best, bi};
  }
}

__global__ void verify_accept_kernel(const ArgPart* __restrict__ part, int chunks,
                                     const int32_t* __restrict__ draft, int batch, int B, int V,
                                     int32_t* out_tokens, int32_t* out_len, int out_cap,
                                     int32_t* seq_lens, int32_t* accept_len, int32_t* next_anchor,
                                     int32_t* err) {
  pdl_trigger();
  pdl_wait();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= batch) return;
  int g = 0;
  int d = 0;
  if (lane < B) {
    const ArgPart* p = part + (size_t)(r * B + lane) * chunks;
    float best = p[0].v;
    int bi = p[0].i;
    for (int c = 1; c < chunks; ++c) argmax_merge(best, bi, p[c].v, p[c].i);
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
                  int32_t* err, cudaStream_t s) {
  const int rows = batch * B;
  ArgPart* part = reinterpret_cast<ArgPart*>(part_v);
  int chunk = (V + chunks - 1) / chunks;
  chunk = (chunk + 63) / 64 * 64;
  const int esz = dtype == DFLASH_BF16 ? 2 : 4;
  const bool vec = ((size_t)V * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(logits) % 16) == 0;
  dim3 grid(chunks, rows);
  {
    TimedScope ts(s, TC_VERIFY);
    if (dtype == DFLASH_BF16) {
      const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(logits);
      if (vec) launch_pdl(verify_argmax_kernel<__nv_bfloat16, true>, dim3(grid),
          dim3(kVerifyThreads), 0, s, 1, x, V, chunk, part);
      else launch_pdl(verify_argmax_kernel<__nv_bfloat16, false>, dim3(grid), dim3(kVerifyThreads),
          0, s, 1, x, V, chunk, part);
    } else {
      const float* x = static_cast<const float*>(logits);
      if (vec) launch_pdl(verify_argmax_kernel<float, true>, dim3(grid), dim3(kVerifyThreads), 0, s,
          1, x, V, chunk, part);
      else launch_pdl(verify_argmax_kernel<float, false>, dim3(grid), dim3(kVerifyThreads), 0, s, 1,
          x, V, chunk, part);
    }
  }
  {
    TimedScope ts(s, TC_VERIFY);
    const int wpb = 4;
    launch_pdl(verify_accept_kernel, dim3((batch + wpb - 1) / wpb), dim3(32 * wpb), 0, s, 1, part,
        chunks, draft, batch, B, V, out_tokens, out_len, out_cap, seq_lens, accept_len, next_anchor,
        err);
  }
  return cudaGetLastError() == cudaSuccess ? DFLASH_OK : DFLASH_ECUDA;
}

}  // namespace dflash
