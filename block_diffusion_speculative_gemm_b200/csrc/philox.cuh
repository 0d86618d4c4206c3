// Counter-based random numbers for the sampled kernels: Philox4x64-10
// (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2,
// 3", SC 2011) and the two maps of a 64-bit output word to a uniform that the
// sampled verify and sampled drafting use.
#pragma once

#include <stdint.h>

namespace dflash {

constexpr float kTwoM53 = 1.1102230246251565e-16f;  // 2^-53

// Philox4x64-10 block function: counter (c0..c3), key (k0, k1).
__device__ __forceinline__ void philox4x64_10(uint64_t (&c)[4], uint64_t k0, uint64_t k1) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint64_t hi0 = __umul64hi(M0, c[0]), lo0 = M0 * c[0];
    const uint64_t hi1 = __umul64hi(M1, c[2]), lo1 = M1 * c[2];
    const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
  }
}

__device__ __forceinline__ void philox_block(uint64_t seed, uint64_t offset, int request,
                                             int stream, uint64_t n4, uint64_t (&w)[4]) {
  w[0] = offset;
  w[1] = (uint64_t)request;
  w[2] = (uint64_t)stream;
  w[3] = n4;
  philox4x64_10(w, seed, 0ull);
}

// log U for U = (w >> 11) 2^-53 in [0, 1) (-inf at 0); the upper half goes
// through log1p(-(1 - U)) with 1 - U formed exactly from the integer.
__device__ __forceinline__ float log_u_closed_open(uint64_t w) {
  const uint64_t k = w >> 11;
  if (k < (1ull << 52)) return k == 0 ? -INFINITY : logf(__ull2float_rn(k) * kTwoM53);
  const uint64_t m = (1ull << 53) - k;  // 1 - U = m 2^-53
  return log1pf(-__ull2float_rn(m) * kTwoM53);
}

// Gumbel variate -log(-log U') for U' = ((w >> 11) + 1/2) 2^-53 in (0, 1).
__device__ __forceinline__ float gumbel_of(uint64_t w) {
  const uint64_t k = w >> 11;
  float e;  // -log U' > 0
  if (k < (1ull << 52)) {
    e = -logf((__ull2float_rn(k) + 0.5f) * kTwoM53);
  } else {
    const uint64_t m = (1ull << 53) - 1 - k;  // 1 - U' = (m + 1/2) 2^-53
    e = -log1pf(-(__ull2float_rn(m) + 0.5f) * kTwoM53);
  }
  return -logf(e);
}

}  // namespace dflash
