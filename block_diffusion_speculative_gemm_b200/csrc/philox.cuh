// Counter-based random numbers for the sampled kernels: Philox4x64-10
// (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2,
// 3", SC 2011) and the two maps of a 64-bit output word to a uniform that the
// sampled verify and sampled drafting use.
#pragma once

#include <stdint.h>

namespace dflash {

constexpr float kTwoM53 = 1.1102230246251565e-16f;  // 2^-53

// Full 64 x 64 -> 128-bit product from four 32 x 32 -> 64 products: with
// a = a1 2^32 + a0 and b = b1 2^32 + b0,
//   t = a0 b1 + hi32(a0 b0),  u = a1 b0 + lo32(t),
//   a b = (a1 b1 + hi32(t) + hi32(u)) 2^64 + lo32(u) 2^32 + lo32(a0 b0);
// none of the partial sums can pass 2^64 - 1.
__device__ __forceinline__ void mul128(uint64_t a, uint64_t b, uint64_t& hi, uint64_t& lo) {
  const uint32_t a0 = (uint32_t)a, a1 = (uint32_t)(a >> 32);
  const uint32_t b0 = (uint32_t)b, b1 = (uint32_t)(b >> 32);
  const uint64_t p00 = (uint64_t)a0 * b0;
  const uint64_t t = (uint64_t)a0 * b1 + (p00 >> 32);
  const uint64_t u = (uint64_t)a1 * b0 + (uint32_t)t;
  hi = (uint64_t)a1 * b1 + (t >> 32) + (u >> 32);
  lo = (u << 32) | (uint32_t)p00;
}

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
    uint64_t hi0, lo0, hi1, lo1;
    mul128(M0, c[0], hi0, lo0);
    mul128(M1, c[2], hi1, lo1);
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
// through log1p(-(1 - U)) with 1 - U formed exactly from the integer.  Used
// for the accept decisions, a few per request, so it keeps the accurate
// library logarithms.
__device__ __forceinline__ float log_u_closed_open(uint64_t w) {
  const uint64_t k = w >> 11;
  if (k < (1ull << 52)) return k == 0 ? -INFINITY : logf(__ull2float_rn(k) * kTwoM53);
  const uint64_t m = (1ull << 53) - k;  // 1 - U = m 2^-53
  return log1pf(-__ull2float_rn(m) * kTwoM53);
}

// Gumbel variate in log2 units, -log2(-ln U') = G log2 e, for
// U' = ((w >> 11) + 1/2) 2^-53 in (0, 1).  One per vocabulary entry of every
// draw, so it is branch-free and uses the hardware base-2 logarithm
// (__log2f: absolute error at most 2^-22 on [1/2, 2], 2 ulp elsewhere):
//
//   E = -ln U' > 0.  For U' < 7/8 (k < 7 2^50), E = -log2(U') ln 2, whose
//   relative error is at most 2^-22 / log2(8/7) < 1.3e-6 (plus 2^-24 from
//   rounding U' to float).  For U' >= 7/8, 1 - U' = m' = (m + 1/2) 2^-53 with
//   m = 2^53 - 1 - k exact, and E = -ln(1 - m') = 2 atanh(s) with
//   s = m' / (2 - m') in (0, 1/15]; the series s (1 + s^2/3 + s^4/5) leaves a
//   relative error below s^6 / 7 < 1.3e-8.
//   The result -log2(E) then carries an absolute error of at most ~1e-5
//   (2 ulp of |log2 E| <= 54), far below fp32 ties that matter in the draw.
__device__ __forceinline__ float gumbel2_of(uint64_t w) {
  const uint64_t k = w >> 11;
  const bool up = k >= 7ull * (1ull << 50);
  const uint64_t sel = up ? (1ull << 53) - 1 - k : k;
  const float f = (__ull2float_rn(sel) + 0.5f) * kTwoM53;  // U' (lower) or m' (upper)
  const float e_lo = -__log2f(f) * 0.69314718055994531f;
  const float s = __fdividef(f, 2.f - f);
  const float t = s * s;
  const float e_up = 2.f * s * fmaf(t, fmaf(t, 0.2f, 0.33333333f), 1.f);
  return -__log2f(up ? e_up : e_lo);
}

// log2(1 - 2^d) for d < 0 in log2 units: the log2 of the residual weight
// max(0, p - q) / p with d = log2 q - log2 p.  For d < -1/4 it is
// log2(1 - exp2(d)), 1 - exp2(d) >= 0.159 and its relative error below
// ~1.3e-6.  For -1/4 <= d < 0, x = d ln 2 in [-0.174, 0) and
// 1 - 2^d = -expm1(x) = -x (1 + x/2 + x^2/6 + x^3/24 + x^4/120 + x^5/720)
// up to a relative x^6/5040 < 6e-9.  d = 0 gives -inf.
__device__ __forceinline__ float log2_one_minus_exp2(float d) {
  const float x = d * 0.69314718055994531f;
  const float p = fmaf(x, fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.f / 720.f, 1.f / 120.f), 1.f / 24.f),
                                       1.f / 6.f), 0.5f), 1.f);
  const float w = d < -0.25f ? 1.f - exp2f(d) : -x * p;
  return __log2f(w);
}

}  // namespace dflash
