// FP8 E4M3 quantization of 8-element bf16 / binary16 vectors, shared by the
// row kernels and the QK prologue: the group scale and the division-free codes.
#pragma once
#include "fn_device.cuh"

namespace fn {

// FP8 scale of a group (or row) and the reciprocal pair the codes use.
struct Fp8Scale {
  float s;         // RN(amax / 448), 1 for an all-zero group
  float r, r_lo;   // the float at or just below 1/s (RD or RD - 1 ulp); RN(RN(1 - s r) r) >= 0
  bool exact_div;  // the fast quotient is not proven here: use the IEEE division
};

// RN(amax / 448) without a division: the product with c = RN(1/448),
// corrected by its exact FMA remainder (Markstein's method).  Equal to the
// IEEE quotient for every bf16 and every binary16 amax, subnormals included
// (checked exhaustively by tests/quotient_proof.c).
__device__ __forceinline__ float scale_div448(float amax) {
  constexpr float c = 1.0f / 448.0f;
  const float q0 = __fmul_rn(amax, c);
  const float rem = fmaf(-448.0f, q0, amax);
  return fmaf(rem, c, q0);
}

// 1/s within one ulp of RN(1/s): the hardware approximation (at most one ulp
// from 1/s) refined by one Newton-Raphson step y + y (1 - s y), which leaves a
// relative error below 2^-46 before the final rounding.  The quotient below
// is proven for every r within one ulp of RN(1/s).
__device__ __forceinline__ float recip_near(float s) {
  float y;
  asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(s));
  return fmaf(fmaf(-s, y, 1.0f), y, y);
}

// A reciprocal not above 1/s: recip_near stepped down (at most twice, since it
// is within one ulp of RN(1/s)) while the exact residual 1 - s r is negative.
// The result is RD(1/s) or, when recip_near was already below, RD(1/s) - 1 ulp:
// within one ulp of RN(1/s) either way.  For s >= 2^-120 r is a normal float,
// so one step down is one less in its bit pattern.
__device__ __forceinline__ float recip_down(float s) {
  float r = recip_near(s);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (fmaf(-s, r, 1.0f) < 0.f) r = __int_as_float(__float_as_int(r) - 1);
  return r;
}

// The group's scale and the reciprocal pair of the codes.
__device__ __forceinline__ Fp8Scale fp8_scale_direct(float amax) {
  Fp8Scale c;
  c.s = amax == 0.f ? 1.f : scale_div448(amax);
  c.exact_div = !(c.s >= 0x1p-120f);
  c.r = c.exact_div ? 1.f : recip_down(c.s);
  c.r_lo = __fmul_rn(fmaf(-c.s, c.r, 1.f), c.r);
  return c;
}

// Eight E4M3 codes of fl32(y / s), the IEEE quotient.
//
// Fast path: with r within one ulp of RN(1/s) and r_lo = RN(RN(1 - s r) r)
// (r + r_lo carries 1/s to about 2^-46), q = RN(|y| r + RN(|y| r_lo)) has the
// same E4M3 code as RN(|y| / s) for every bf16 y with |y| <= amax and every
// bf16 amax with s = RN(amax / 448) >= 2^-120, and likewise for every
// binary16 pair (whose scales are all above 2^-120): checked exhaustively over
// all such (amax, y) pairs and all three such r by tests/quotient_proof.c.
// The codes are computed from the signed y: every step rounds to nearest
// even, which is odd-symmetric, so a negative y gets minus the quotient of
// |y| and the conversion writes the sign.  Zeros keep their sign because
// r_lo >= 0 (r is not above 1/s): -0 r_lo = -0 and -0 + -0 = -0 (code 0x80).
// If any lane of the warp needs the IEEE division the whole warp takes it
// (warp-uniform branch; the signed quotient keeps signs there too): `exact`
// must be the same in every lane and true if any lane's scale needs it.
template <class IO = Bf16>
__device__ __forceinline__ uint2 e4m3_codes_uniform(const uint4& y, const Fp8Scale& c, bool exact) {
  uint32_t q8[4];
  if (!exact) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 yf = make_float2(IO::lo(word(y, i)), IO::hi(word(y, i)));
      const float2 t = mul_f32x2(yf, make_float2(c.r_lo, c.r_lo));
      const float2 q = fma_f32x2(yf, make_float2(c.r, c.r), t);
      q8[i] = cvt_e4m3x2(q.x, q.y);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q8[i] = cvt_e4m3x2(__fdiv_rn(IO::lo(word(y, i)), c.s), __fdiv_rn(IO::hi(word(y, i)), c.s));
  }
  return make_uint2(q8[0] | (q8[1] << 16), q8[2] | (q8[3] << 16));
}

// e4m3_codes_uniform with the path voted by the warp.  All 32 lanes must call.
template <class IO = Bf16>
__device__ __forceinline__ uint2 e4m3_codes(const uint4& y, const Fp8Scale& c) {
  return e4m3_codes_uniform<IO>(y, c, __any_sync(0xffffffffu, c.exact_div));
}

}  // namespace fn
