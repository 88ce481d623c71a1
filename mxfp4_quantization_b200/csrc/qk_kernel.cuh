// QK Gemma-RMSNorm + gate extraction, sm_100a (sglang PR #27656, "Motivation":
// one kernel in place of the q copy, the gate copy and the q/k norm).
//
// One warp per (token, head).  A q head and its gate are adjacent in the
// interleaved row ([q_h, gate_h] = 2D contiguous elements), so the warp that
// normalizes q_h also copies gate_h; k heads get their own warps.  Rows are
// addressed through row_stride, so no contiguous copy of the projection output
// is ever made.  With head_dim 256 each lane holds one 16-byte vector.
#pragma once
#include "fn_device.cuh"
#include "quant.cuh"

namespace fn {

struct QKParams {
  const uint4* qkv;
  int64_t M;
  int64_t row_vec;  // row stride in 16-byte vectors
  int Hq, Hk;
  int dv;           // head_dim / 8
  const uint4* qw;
  const uint4* kw;
  float eps;
  float inv_d;      // 1 / head_dim
  uint4* out_q;     // bf16 outputs (optional when FP8 codes are written)
  uint4* out_k;
  uint4* out_g;
  uint8_t* out_q8;  // E4M3 codes [M, Hq, D] and fp32 scales [M, Hq] (FP8 kernel)
  float* out_qs;
  uint8_t* out_k8;  // E4M3 codes [M, Hk, D] and fp32 scales [M, Hk]
  float* out_ks;
  int prefetch_self;  // L2-prefetch each warp's head before the programmatic-launch wait
};

// FP8: also quantize each normed q and k head to E4M3 with one fp32 scale per
// (token, head) — the per-token rule of the row kernels (scale = amax / 448)
// applied to each head vector, for an FP8 attention consumer.
template <int VPL, bool FP8>
__global__ void __launch_bounds__(256) qk_kernel(const __grid_constant__ QKParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int heads = p.Hq + p.Hk;
  if (p.prefetch_self) {
    // Launched as a programmatic dependent, the block may start while the
    // previous kernel still runs: start this warp's head (q with its gate, or
    // k) and the norm weights towards L2 before the wait (a hint with no
    // result: data written meanwhile lands in L2 over the prefetched lines).
    if (lane == 0 && item < p.M * heads) {
      const int64_t m = item / heads;
      const int j = (int)(item - m * heads);
      const uint4* row = p.qkv + m * p.row_vec;
      if (j < p.Hq)
        bulk_prefetch_l2(row + (int64_t)(2 * j) * p.dv, (uint32_t)p.dv * 32u);
      else
        bulk_prefetch_l2(row + (int64_t)(2 * p.Hq + (j - p.Hq)) * p.dv, (uint32_t)p.dv * 16u);
    }
    if (threadIdx.x == 1 && p.qw != nullptr) bulk_prefetch_l2(p.qw, (uint32_t)p.dv * 16u);
    if (threadIdx.x == 2 && p.kw != nullptr) bulk_prefetch_l2(p.kw, (uint32_t)p.dv * 16u);
  }
  pdl_enter();
  if (item >= p.M * heads) return;  // warp-uniform
  const int64_t m = item / heads;
  const int j = (int)(item - m * heads);
  const bool isq = j < p.Hq;
  const uint4* row = p.qkv + m * p.row_vec;
  const uint4* src = isq ? row + (int64_t)(2 * j) * p.dv
                         : row + (int64_t)(2 * p.Hq + (j - p.Hq)) * p.dv;
  const uint4* w = isq ? p.qw : p.kw;
  const int64_t head = isq ? m * p.Hq + j : m * p.Hk + (j - p.Hq);  // output head index
  uint4* dst = isq ? p.out_q : p.out_k;
  if (dst != nullptr) dst += head * p.dv;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

  uint4 x[VPL], wv[VPL], g[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = lane + 32 * i;
    const bool ok = v < p.dv;
    x[i] = ok ? ld_stream_nc(src + v) : zero;
    g[i] = (ok && isq) ? ld_stream_nc(src + p.dv + v) : zero;
    wv[i] = ok ? ld_keep(w + v) : zero;
  }
  if (isq) {
    uint4* gdst = p.out_g + (m * p.Hq + j) * p.dv;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i < p.dv) st_stream(gdst + lane + 32 * i, g[i]);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float a = bf_lo(word(x[i], c)), b = bf_hi(word(x[i], c));
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  ss = warp_sum(ss);
  // 1 / sqrt(mean + eps): hardware reciprocal square root plus one
  // Newton-Raphson step, r <- r (3 - x r^2) / 2 (about one fp32 ulp)
  const float xm = fmaf(ss, p.inv_d, p.eps);
  const float r0 = rsqrtf(xm);
  const float rstd = r0 * fmaf(-0.5f * xm * r0, r0, 1.5f);
  uint4 y[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t xw = word(x[i], c), ww = word(wv[i], c);
      const float y0 = (bf_lo(xw) * rstd) * (1.f + bf_lo(ww));
      const float y1 = (bf_hi(xw) * rstd) * (1.f + bf_hi(ww));
      set_word(y[i], c, pack_bf16x2(y0, y1));
    }
    if (dst != nullptr && lane + 32 * i < p.dv) st_stream(dst + lane + 32 * i, y[i]);
  }
  if constexpr (FP8) {
    float am = 0.f;  // lanes past the head hold y = 0
#pragma unroll
    for (int i = 0; i < VPL; ++i) am = fmaxf(am, vec_absmax(y[i]));
    const Fp8Scale sc = fp8_scale_direct(warp_max(am));
    uint8_t* codes = (isq ? p.out_q8 : p.out_k8) + head * (int64_t)p.dv * 8;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const uint2 q = e4m3_codes(y[i], sc);  // every lane takes part
      if (lane + 32 * i < p.dv) st_stream(reinterpret_cast<uint2*>(codes) + lane + 32 * i, q);
    }
    if (lane == 0) (isq ? p.out_qs : p.out_ks)[head] = sc.s;
  }
}

}  // namespace fn
