// Counter-based random numbers for the sampled kernels: Philox4x64-10
// (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2,
// 3", SC 2011) and the two maps of a 64-bit output word to a uniform that the
// sampled verify and sampled drafting use.
#pragma once

#include <stdint.h>

#include "common.cuh"

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
// through log1p(-(1 - U)) with 1 - U formed exactly from the integer.  Used
// for the accept decisions, a few per request, so it keeps the accurate
// library logarithms.
__device__ __forceinline__ float log_u_closed_open(uint64_t w) {
  const uint64_t k = w >> 11;
  if (k < (1ull << 52)) return k == 0 ? -INFINITY : logf(__ull2float_rn(k) * kTwoM53);
  const uint64_t m = (1ull << 53) - k;  // 1 - U = m 2^-53
  return log1pf(-__ull2float_rn(m) * kTwoM53);
}

// Hardware base-2 logarithm and reciprocal (PTX lg2.approx.ftz.f32: absolute
// error at most about 2^-22 on [1/2, 2] and relative error about 2^-22
// elsewhere; rcp.approx.ftz.f32: about 1 ulp).  Subnormal inputs count as 0.
__device__ __forceinline__ float lg2_ftz(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_ftz(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Gumbel variate in log2 units, -log2(-ln U') = G log2 e, for
// U' = ((w >> 11) + 1/2) 2^-53 in (0, 1).  One per vocabulary entry of every
// draw, so it is branch-free, works on 32-bit halves and uses the hardware
// base-2 logarithm:
//
//   E = -ln U' > 0.  For U' < 7/8 (w < 7 2^61), E = -log2(U') ln 2, whose
//   relative error is at most 2^-22 / log2(8/7) < 1.3e-6 (plus about 2^-23 from
//   forming U' in float).  For U' >= 7/8, 1 - U' = m' = (((~w) >> 11) + 1/2)
//   2^-53 (exact in the integers: (~w) >> 11 = 2^53 - 1 - (w >> 11)), and
//   E = -ln(1 - m') = 2 atanh(s) with s = m' / (2 - m') in (0, 1/15]; the
//   series s (1 + s^2/3 + s^4/5) leaves a relative error below s^6 / 7 < 1.3e-8.
//   Both branches form their float from v = w or ~w the same way:
//   ((v >> 11) + 1/2) 2^-53 = hi32(v) 2^-32 + ((lo32(v) >> 11) + 1/2) 2^-53,
//   the second term exact (a 21-bit integer plus 1/2, made with the 2^23
//   exponent trick), one rounding in the fused multiply-add.
//   The result -log2(E) then carries an absolute error of at most ~1e-5
//   (2^-22 relative of |log2 E| <= 54), far below fp32 ties that matter in the
//   draw.
__device__ __forceinline__ float gumbel2_of(uint64_t w) {
  const bool up = (uint32_t)(w >> 32) >= 0xE0000000u;  // w >= 7 2^61
  const uint64_t v = up ? ~w : w;
  const uint32_t vh = (uint32_t)(v >> 32), vl = (uint32_t)v;
  // (vl >> 11) + 1/2 exactly: 2^23 + n has n in its mantissa (n < 2^21)
  const float low = __uint_as_float(0x4B000000u | (vl >> 11)) - 8388607.5f;
  const float f = fmaf(__uint2float_rn(vh), 2.3283064365386963e-10f, low * kTwoM53);
  const float e_lo = -lg2_ftz(f) * 0.69314718055994531f;
  const float s = f * rcp_ftz(2.f - f);
  const float t = s * s;
  const float e_up = 2.f * s * fmaf(t, fmaf(t, 0.2f, 0.33333333f), 1.f);
  return -lg2_ftz(up ? e_up : e_lo);
}

// log2(1 - 2^d) for d < 0 in log2 units: the log2 of the residual weight
// max(0, p - q) / p with d = log2 q - log2 p.  For d < -1/4 it is
// log2(1 - exp2(d)), 1 - exp2(d) >= 0.159 and its relative error below
// ~1.3e-6.  For -1/4 <= d < 0, x = d ln 2 in [-0.174, 0) and
// 1 - 2^d = -expm1(x) = -x (1 + x/2 + x^2/6 + x^3/24 + x^4/120 + x^5/720)
// up to a relative x^6/5040 < 6e-9.  d = 0 (and |d| below 2^-126) gives -inf.
__device__ __forceinline__ float log2_one_minus_exp2(float d) {
  const float x = d * 0.69314718055994531f;
  const float p = fmaf(x, fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.f / 720.f, 1.f / 120.f), 1.f / 24.f),
                                       1.f / 6.f), 0.5f), 1.f);
  const float w = d < -0.25f ? 1.f - ex2_ftz(d) : -x * p;
  return lg2_ftz(w);
}

}  // namespace dflash
