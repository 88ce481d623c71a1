// Device helpers for the sm_100a kernels: 128-bit streaming loads/stores,
// bf16 packing, and the packed E4M3 / E2M1 conversions (PTX `cvt` with
// round-to-nearest-even and saturation to the largest finite value).
#pragma once
#include <cstdint>

namespace fn {

// ---- launch ordering --------------------------------------------------------------

// First statement of every kernel.  Programmatic dependent launch: wait until
// the grids this one depends on have completed and their writes are visible
// (at once for an ordinary launch), then allow the next grid on the stream to
// start launching its blocks (which wait the same way before touching memory).
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- memory -----------------------------------------------------------------

// Read-only input that no output aliases: non-coherent path, no L1 allocation
// (each byte is read once).
__device__ __forceinline__ uint4 ld_stream_nc(const uint4* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// Input that an output may alias in place (the residual): coherent load.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Bulk prefetch of a contiguous global range into L2 (nothing to wait for).
// 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Small, reused operand (the norm weight): normal cached read-only load.
__device__ __forceinline__ uint4 ld_keep(const uint4* p) { return __ldg(p); }

__device__ __forceinline__ void st_stream(uint4* p, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_stream(uint2* p, uint2 v) {
  asm volatile("st.global.L1::no_allocate.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y)
               : "memory");
}

__device__ __forceinline__ void st_stream(uint32_t* p, uint32_t v) {
  asm volatile("st.global.L1::no_allocate.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---- bf16 -------------------------------------------------------------------

// Element 2i of a packed pair lives in the low half (little-endian memory).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 -> packed bf16 pair, each rounded to nearest even (subnormals kept).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Packed bf16 add, one rounding of the exact sum.  For two bf16 operands this
// equals rounding their fp32 sum to bf16: if the fp32 sum is inexact the
// operands' exponents differ by more than 16, so the smaller one moves the
// larger by less than 2^-15 of it, far from any bf16 rounding midpoint.
__device__ __forceinline__ uint32_t add_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Packed max of |a| and |b| per half (exact: max only selects).  The sign
// bit of each result half is the xor of the operands' signs: only the
// magnitude is meaningful, and further absmax calls may take it as is.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void set_word(uint4& v, int i, uint32_t w) {
  if (i == 0) v.x = w;
  else if (i == 1) v.y = w;
  else if (i == 2) v.z = w;
  else v.w = w;
}

// ---- mixed bf16 / fp32 and packed fp32 arithmetic (sm_100) ---------------------

// acc + x, x the low (HI = false) or high bf16 half of w, rounded once to fp32:
// the same value as adding x converted to fp32.
template <bool HI>
__device__ __forceinline__ float add_bf16(uint32_t w, float acc) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %2;\n\t}"
        : "=f"(d) : "r"(w), "f"(acc));
  else
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, l, %2;\n\t}"
        : "=f"(d) : "r"(w), "f"(acc));
  return d;
}

// a * b + c for the low (HI = false) or high bf16 halves of a and b, rounded
// once to fp32.  The product of two bf16 is exact in fp32, so with c = -0 this
// is exactly a * b (and its sign for zeros).
template <bool HI>
__device__ __forceinline__ float fma_bf16(uint32_t a, uint32_t b, float c) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// Element-wise a * b and a * b + c on fp32 pairs, each rounded once.
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// ---- IEEE binary16 -------------------------------------------------------------

__device__ __forceinline__ float f16_lo(uint32_t w) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(d) : "r"(w));
  return d;
}
__device__ __forceinline__ float f16_hi(uint32_t w) {
  float d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(d) : "r"(w));
  return d;
}

// Two fp32 -> packed binary16 pair, each rounded to nearest even (subnormals
// kept, overflow to infinity).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Packed binary16 add, one rounding of the exact sum, subnormals kept.  For
// two binary16 operands this equals rounding their fp32 sum to binary16: the
// fp32 sum is inexact only if the exponents differ by more than 13, and then
// the smaller operand moves the larger by under a quarter of its half-ulp, so
// both roundings return the larger operand.
__device__ __forceinline__ uint32_t add_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

template <bool HI>
__device__ __forceinline__ float add_f16(uint32_t w, float acc) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.f16 %0, h, %2;\n\t}"
        : "=f"(d) : "r"(w), "f"(acc));
  else
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.f16 %0, l, %2;\n\t}"
        : "=f"(d) : "r"(w), "f"(acc));
  return d;
}

// As fma_bf16: the product of two binary16 (11-bit significands) is exact in
// fp32.
template <bool HI>
__device__ __forceinline__ float fma_f16(uint32_t a, uint32_t b, float c) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, ah, bh, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %3;\n\t}"
        : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// ---- element formats ---------------------------------------------------------------
// The row kernels are written once over the format of their 16-bit tensors:
// Bf16, or F16 (IEEE binary16).  Each gives the pair decode, the rounding
// pack, the packed add and |max|, and the mixed fp32 add and fma on one half.

struct Bf16 {
  static constexpr bool kF16 = false;
  static __device__ __forceinline__ float lo(uint32_t w) { return bf_lo(w); }
  static __device__ __forceinline__ float hi(uint32_t w) { return bf_hi(w); }
  static __device__ __forceinline__ uint32_t pack(float l, float h) { return pack_bf16x2(l, h); }
  static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
    return add_bf16x2(a, b);
  }
  static __device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
    return absmax_bf16x2(a, b);
  }
  template <bool HI>
  static __device__ __forceinline__ float add(uint32_t w, float acc) {
    return add_bf16<HI>(w, acc);
  }
  template <bool HI>
  static __device__ __forceinline__ float fma(uint32_t a, uint32_t b, float c) {
    return fma_bf16<HI>(a, b, c);
  }
};

struct F16 {
  static constexpr bool kF16 = true;
  static __device__ __forceinline__ float lo(uint32_t w) { return f16_lo(w); }
  static __device__ __forceinline__ float hi(uint32_t w) { return f16_hi(w); }
  static __device__ __forceinline__ uint32_t pack(float l, float h) { return pack_f16x2(l, h); }
  static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
    return add_f16x2(a, b);
  }
  static __device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
    return absmax_f16x2(a, b);
  }
  template <bool HI>
  static __device__ __forceinline__ float add(uint32_t w, float acc) {
    return add_f16<HI>(w, acc);
  }
  template <bool HI>
  static __device__ __forceinline__ float fma(uint32_t a, uint32_t b, float c) {
    return fma_f16<HI>(a, b, c);
  }
};

// max |y| over the 8 16-bit values of a vector, as fp32.
template <class IO = Bf16>
__device__ __forceinline__ float vec_absmax(const uint4& y) {
  const uint32_t m = IO::absmax2(IO::absmax2(y.x, y.y), IO::absmax2(y.z, y.w));
  return fmaxf(fabsf(IO::lo(m)), fabsf(IO::hi(m)));
}

// ---- FP8 E4M3 -----------------------------------------------------------------

// Two fp32 -> two E4M3 codes (nearest even, saturating to +-448); `lo` lands in
// the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// ---- FP4 E2M1 -----------------------------------------------------------------

// Eight fp32 -> eight E2M1 codes (nearest even, saturating to +-6) packed in a
// 32-bit word: element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t d;
  asm("{\n\t"
      ".reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t"
      "}"
      : "=r"(d)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
        "f"(v[7]));
  return d;
}

// ---- reductions ------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Max of a non-negative value over each 16-lane half of the warp, by two
// hardware warp reductions on the bit patterns (non-negative floats order as
// unsigned integers).  All 32 lanes must call.
__device__ __forceinline__ float half_warp_max(float v) {
  const uint32_t u = __float_as_uint(v);
  const bool lo = (threadIdx.x & 16) == 0;
  uint32_t a, b;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(a) : "r"(lo ? u : 0u));
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(b) : "r"(lo ? 0u : u));
  return __uint_as_float(lo ? a : b);
}

// Max over aligned groups of `G` lanes (G a power of two, <= 32).
template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// MX block exponent from the block amax (a non-negative bf16 or binary16
// value): e = floor(log2 amax) - 2, clamped to [-127, 127]; zero and bf16
// subnormals (binary32 exponent field 0) give -127.  Returns the E8M0 code e + 127, and
// 2^-e (always a normal binary32, since e <= 125) in `inv`.  A NaN or
// infinite amax gives code 0xFF.
__device__ __forceinline__ uint32_t mx_scale(float amax, float& inv) {
  uint32_t ef = __float_as_uint(amax) >> 23;  // sign is 0
  int e = (ef == 0) ? -127 : max((int)ef - 129, -127);
  inv = __uint_as_float((uint32_t)(127 - e) << 23);
  return ef == 0xFF ? 0xFFu : (uint32_t)(e + 127);
}

}  // namespace fn
