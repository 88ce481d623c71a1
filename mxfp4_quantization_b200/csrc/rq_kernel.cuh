// Fused (partial sum) + residual add + RMSNorm + quantization, sm_100a.
//
// Follows the unfused AllReduce -> RMSNorm -> quantize sequence that the fused
// AITER kernel of sglang PR #29723 ("Accuracy Tests") must equal, with the
// all-reduce replaced by an in-kernel sum of up to 8 same-device partials, and
// the quantization of the bf16 normed row that sgl-amd-mono PR #26's monokernel
// notes call bit-exact against stand-alone quantization.
//
// HBM-bound, no tensor cores.  Two forms of one kernel share the per-vector
// stages below:
//  * rq_kernel, CL = false: one thread block per row.  Every load of the row
//    is issued before the first arithmetic; the row then lives in registers.
//    Large-M launches also start rows about one wave ahead towards L2 with a
//    bulk prefetch (cp.async.bulk.prefetch.L2, nothing waits on it).
//  * rq_kernel, CL = true (small M with rows too long for one wide block, or on
//    request): a cluster of 2..8 blocks per row; the blocks exchange their
//    partial sums through distributed shared memory.
// A thread owns 16-byte vectors (8 bf16) with index seg_base + threadIdx.x +
// k * blockDim.x, so a warp touches 512 contiguous bytes per tensor per k.
// MX blocks (32 elements) are 4 adjacent lanes and FP8 groups (128) 16
// adjacent lanes: their amax is a 2- or 4-step xor shuffle.
#pragma once
#include <cooperative_groups.h>

#include "fn_device.cuh"
#include "quant.cuh"
#include "rq_params.h"

namespace fn {

namespace cg = cooperative_groups;

// ---------------------------------------------------------------------------
// per-vector stages
// ---------------------------------------------------------------------------

// Every stage is written over the element format IO of the 16-bit tensors
// (Bf16 or F16, fn_device.cuh); "bf16" below reads "IO" for binary16 rows.

// h = bf16(((x_0 + x_1) + ...) + r) for one vector, every add in fp32.
template <int MAXP, class IO = Bf16>
__device__ __forceinline__ uint4 sum_vec(const uint4 (&x)[MAXP], const uint4& r, int P,
                                         bool has_res) {
  uint4 h;
  if constexpr (MAXP == 1) {
    h = has_res ? make_uint4(IO::add2(x[0].x, r.x), IO::add2(x[0].y, r.y),
                             IO::add2(x[0].z, r.z), IO::add2(x[0].w, r.w))
                : x[0];
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a0 = IO::lo(word(x[0], i)), a1 = IO::hi(word(x[0], i));
#pragma unroll
      for (int p = 1; p < MAXP; ++p) {
        if (p < P) {
          a0 = IO::template add<false>(word(x[p], i), a0);
          a1 = IO::template add<true>(word(x[p], i), a1);
        }
      }
      if (has_res) {
        a0 = IO::template add<false>(word(r, i), a0);
        a1 = IO::template add<true>(word(r, i), a1);
      }
      set_word(h, i, IO::pack(a0, a1));
    }
  }
  return h;
}

// Sum of squares of h (two fp32 accumulators), and (per-token mode) max |h * w|.
// h * w is exact in fp32 (two 8-bit, or two 11-bit, significands) and
// y = bf16(fl(h * w) * rstd) is monotone in |h * w|, so
// max |y| = bf16(fl(max |h * w| * rstd)) falls out of the same reduction as
// the sum of squares.
template <bool WANT_PMAX, class IO = Bf16>
__device__ __forceinline__ void stats_vec(const uint4& h, const uint4& w, float2& ss,
                                          float& pmax) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t hw = word(h, i);
    ss.x = IO::template fma<false>(hw, hw, ss.x);
    ss.y = IO::template fma<true>(hw, hw, ss.y);
    if (WANT_PMAX) {
      const uint32_t ww = word(w, i);
      pmax = fmaxf(pmax, fmaxf(fabsf(IO::template fma<false>(hw, ww, -0.f)),
                               fabsf(IO::template fma<true>(hw, ww, -0.f))));
    }
  }
}

// y = bf16(fl(h * w) * rstd).
template <class IO = Bf16>
__device__ __forceinline__ uint4 norm_vec(const uint4& h, const uint4& w, float rstd) {
  uint4 y;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t hw = word(h, i), ww = word(w, i);
    const float2 p = make_float2(IO::template fma<false>(hw, ww, -0.f),
                                 IO::template fma<true>(hw, ww, -0.f));
    const float2 q = mul_f32x2(p, make_float2(rstd, rstd));
    set_word(y, i, IO::pack(q.x, q.y));
  }
  return y;
}

// E2M1 codes of y * 2^-e for the 8 values of a vector (inv = 2^-e); each
// product is exact and keeps the sign of zeros.  For bf16 rows 2^-e is itself
// a bf16 (e <= 125), and the mixed bf16 FMA with a -0 addend forms the
// product in one instruction; a binary16 row's 2^-e can lie outside binary16
// (up to 2^26), so those products are fp32 multiplies.
template <class IO = Bf16>
__device__ __forceinline__ uint32_t e2m1_codes(const uint4& y, float inv) {
  float f[8];
  if constexpr (!IO::kF16) {
    const uint32_t ib = __float_as_uint(inv) >> 16;
    const uint32_t inv2 = ib | (ib << 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = fma_bf16<false>(word(y, i), inv2, -0.f);
      f[2 * i + 1] = fma_bf16<true>(word(y, i), inv2, -0.f);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = mul_f32x2(make_float2(IO::lo(word(y, i)), IO::hi(word(y, i))),
                                 make_float2(inv, inv));
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
  return cvt_e2m1x8(f);
}

// Byte offset (MX) or element index (FP8 groups) of the scale of group `g`
// of row `row` in the requested layout (row-major unless a flag asks
// otherwise).  The 32x4x4 swizzle is the tiling of block-scaled matrix
// multiplies on this architecture: 128 rows x 4 groups per 512-byte tile,
// tiles in row-tile-major order, and inside a tile row r, group c at
// (r % 32) * 16 + (r / 32) * 4 + c.
__device__ __forceinline__ int64_t scale_index(int layout, int64_t ld, int64_t row, int64_t g,
                                               int64_t groups_per_row) {
  if (layout == SCALE_SWIZZLE_32_4_4)
    return ((row >> 7) * ld + (g >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (g & 3);
  if (layout == SCALE_MN_MAJOR) return g * ld + row;
  return row * groups_per_row + g;
}

// Codes of one vector (y: 8 values) and, for the group modes, its group's
// scale.  All 32 lanes must call (shuffles).  `tok` is the row's scale
// (per-token mode).
struct QuantVec {
  uint2 q8;     // FP8: eight E4M3 codes
  uint32_t q4;  // MXFP4: eight E2M1 codes
  float s;      // group-128: the group's fp32 scale
  uint32_t e8;  // MXFP4: the block's E8M0 code
};

template <int MODE, class IO = Bf16>
__device__ __forceinline__ QuantVec quant_vec(const uint4& y, const Fp8Scale& tok) {
  QuantVec r;
  if constexpr (MODE == MODE_TOKEN || MODE == MODE_G128) {
    Fp8Scale c = tok;
    if constexpr (MODE == MODE_G128) c = fp8_scale_direct(half_warp_max(vec_absmax<IO>(y)));
    r.s = c.s;
    r.q8 = e4m3_codes<IO>(y, c);
  } else {
    float inv;
    r.e8 = mx_scale(group_max<4>(vec_absmax<IO>(y)), inv);
    r.q4 = e2m1_codes<IO>(y, inv);
  }
  return r;
}

// Store the codes of vector v of a row and, from the group's first lane, its
// scale; `ok` masks lanes past the row end (whole groups, by alignment).
template <int MODE>
__device__ __forceinline__ void store_quant(const QuantVec& r, bool ok, int lane, int64_t row,
                                            int v, int H, uint8_t* out_q, void* out_scale,
                                            int layout, int64_t ld) {
  if (!ok) return;
  if constexpr (MODE == MODE_TOKEN || MODE == MODE_G128) {
    if (MODE == MODE_G128 && (lane & 15) == 0)
      static_cast<float*>(out_scale)[scale_index(layout, ld, row, v / 16, H / 128)] = r.s;
    st_stream(reinterpret_cast<uint2*>(out_q + row * (int64_t)H) + v, r.q8);
  } else {
    st_stream(reinterpret_cast<uint32_t*>(out_q + row * (int64_t)(H / 2)) + v, r.q4);
    if ((lane & 3) == 0)
      static_cast<uint8_t*>(out_scale)[scale_index(layout, ld, row, v / 4, H / 32)] =
          (uint8_t)r.e8;
  }
}

// Quantize vector v of a row and store it (quant_vec, then store_quant).
template <int MODE, class IO = Bf16>
__device__ __forceinline__ void quant_store(const uint4& y, bool ok, int lane, int64_t row, int v,
                                            int H, const Fp8Scale& tok, uint8_t* out_q,
                                            void* out_scale, int layout, int64_t ld) {
  store_quant<MODE>(quant_vec<MODE, IO>(y, tok), ok, lane, row, v, H, out_q, out_scale, layout,
                    ld);
}

// Per-group-128 codes and scales of the V vectors yv[k] = vector vbase + k*T
// of a row that one thread holds (V a power of two, 2..16; T a multiple of 16,
// so each 16-lane half-warp shares one group per k), with one scale
// computation per lane instead of one per vector: the V group maxima travel
// together as bf16 pairs through four xor-shuffle steps (the amax of bf16 or
// binary16 values is one of them, so the packing is exact), lane l computes
// the scale and reciprocal pair of group k = l % V, every lane fetches the
// pairs of its V groups with two shuffles each, and lane k of each half-warp
// (which computed group k) stores that group's scale.  Same bits as V calls
// of quant_store<MODE_G128>.  All 32 lanes must call; `ok` is false in whole
// half-warps past the row end.
template <int V, class IO = Bf16>
__device__ __forceinline__ void quant_store_g128_rows(const uint4 (&yv)[V], const bool (&ok)[V],
                                                      int lane, int64_t row, int vbase, int T,
                                                      int H, uint8_t* out_q, float* out_scale,
                                                      int layout, int64_t ld) {
  static_assert(V >= 2 && V <= 16 && (V & (V - 1)) == 0, "V: a power of two in 2..16");
  // group maxima, two groups per 32-bit word
  uint32_t pm[V / 2];
#pragma unroll
  for (int i = 0; i < V / 2; ++i) {
    uint32_t m[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4& y = yv[2 * i + h];
      const uint32_t a = IO::absmax2(IO::absmax2(y.x, y.y), IO::absmax2(y.z, y.w));
      m[h] = IO::absmax2(a, __byte_perm(a, 0u, 0x1032));  // both halves: the vector's |max|
    }
    pm[i] = __byte_perm(m[0], m[1], 0x5410) & 0x7FFF7FFFu;  // (group 2i, group 2i+1)
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
#pragma unroll
    for (int i = 0; i < V / 2; ++i) pm[i] = IO::absmax2(pm[i], __shfl_xor_sync(0xffffffffu, pm[i], o));
  }
  // this lane's group: k = lane % V
  const int ks = lane & (V - 1);
  uint32_t sel = pm[0];
#pragma unroll
  for (int i = 1; i < V / 2; ++i)
    if ((ks >> 1) == i) sel = pm[i];
  const Fp8Scale own = fp8_scale_direct((ks & 1) ? IO::hi(sel) : IO::lo(sel));
  const bool exact = __any_sync(0xffffffffu, own.exact_div);
  const int src = lane & ~(V - 1);
#pragma unroll
  for (int k = 0; k < V; ++k) {
    Fp8Scale c;
    c.r = __shfl_sync(0xffffffffu, own.r, src + k);
    c.r_lo = __shfl_sync(0xffffffffu, own.r_lo, src + k);
    c.s = exact ? __shfl_sync(0xffffffffu, own.s, src + k) : 1.f;
    c.exact_div = exact;
    if (ok[k])
      st_stream(reinterpret_cast<uint2*>(out_q + row * (int64_t)H) + vbase + k * T,
                e4m3_codes_uniform<IO>(yv[k], c, exact));
  }
  if ((lane & 15) < V) {
    const int vk = vbase + ks * T;  // this lane's vector in group ks of its half-warp
    bool ok_sel = ok[0];
#pragma unroll
    for (int k = 1; k < V; ++k)
      if (ks == k) ok_sel = ok[k];
    if (ok_sel) out_scale[scale_index(layout, ld, row, vk / 16, H / 128)] = own.s;
  }
}

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------

// Cluster barrier halves (all threads of every block of the cluster take part).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Sum of `s` and max of `m` over the block and, with CL, over the cluster.
// The warps' results are combined in a fixed order, so every thread and every
// block of a cluster (ranks in rank order) gets the same bits: in index order
// by every thread (the shortest chain: decode-sized launches), or, with
// `butterfly` (uniform over the launch), lane i of every warp takes warp i's
// result and an xor butterfly combines them — both operands of every step are
// the same in all lanes and addition commutes, so all lanes agree — which
// takes fewer instructions for wide blocks (large-M launches).  With CL the
// caller must call cluster_wait() once before exiting: the last arrive here
// tells the peers this block is done reading their shared memory, and the
// wait keeps this block's own slot alive until every peer has read it.
template <bool CL, bool WANT_MAX>
__device__ __forceinline__ float2 row_reduce(float s, float m, float2* red, float2* cl_slot,
                                             bool butterfly = false) {
  s = warp_sum(s);
  if (WANT_MAX) m = warp_max(m);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) red[warp] = make_float2(s, m);
  __syncthreads();
  float2 t;
  if (butterfly) {
    t = lane < nw ? red[lane] : make_float2(0.f, 0.f);
    t.x = warp_sum(t.x);
    if (WANT_MAX) t.y = warp_max(t.y);
  } else {
    t = red[0];
    for (int i = 1; i < nw; ++i) {
      const float2 o = red[i];
      t.x += o.x;
      if (WANT_MAX) t.y = fmaxf(t.y, o.y);
    }
  }
  if constexpr (CL) {
    cg::cluster_group cl = cg::this_cluster();
    if (threadIdx.x == 0) *cl_slot = t;
    cluster_arrive();
    cluster_wait();
    const unsigned nb = cl.num_blocks();
    float2 u = *cl.map_shared_rank(cl_slot, 0);
    for (unsigned c = 1; c < nb; ++c) {
      const float2 o = *cl.map_shared_rank(cl_slot, c);
      u.x += o.x;
      if (WANT_MAX) u.y = fmaxf(u.y, o.y);
    }
    cluster_arrive();
    t = u;
  }
  return t;
}

// 1 / sqrt(mean(h^2) + eps) in fp32: the hardware reciprocal square root
// refined by one Newton-Raphson step, r <- r (3 - x r^2) / 2, which brings it
// to about one fp32 ulp (the normed row is specified to 1 bf16 ulp).
__device__ __forceinline__ float row_rstd(float ss, float inv_h, float eps) {
  const float x = fmaf(ss, inv_h, eps);
  const float r = rsqrtf(x);
  return r * fmaf(-0.5f * x * r, r, 1.5f);
}

// bf16(fl(pmax * rstd)): the row's max |y| (see stats_vec).
template <class IO = Bf16>
__device__ __forceinline__ float row_amax_from_pmax(float pmax, float rstd) {
  return IO::lo(IO::pack(pmax * rstd, 0.f));
}

// ---------------------------------------------------------------------------
// register-resident kernel: one row per block (CL = false) or per cluster
// ---------------------------------------------------------------------------

// TB > 0 marks an exact-cover instance: the block has TB threads and the row
// is exactly TB * V vectors (H = 8 * TB * V), so every offset is a
// compile-time constant and no access needs a bounds test.  TB = 0 reads the
// block size and the row length at run time.  Blocks of up to 256 threads
// keep the whole register file per thread (255); the wide exact-cover
// instances (TB = 448, 512) and the cluster kernel allow 512 threads.
template <int MODE, int MAXP, int V, bool NORM, bool CL, int TB = 0, class IO = Bf16>
__global__ void __launch_bounds__((CL || TB > 256) ? 512 : 256)
    rq_kernel(const __grid_constant__ RQParams prm) {
  static_assert(TB == 0 || !CL, "exact-cover instances are one block per row");
  __shared__ float2 red[32];
  __shared__ float2 cl_slot;
  if (!CL && prm.prefetch_self) {
    // Launched as a programmatic dependent, the block may start while the
    // previous kernel still runs: start this row's inputs towards L2 before
    // the wait (a hint with no result: data that the previous kernel writes
    // meanwhile, an in-place residual included, lands in L2 over the
    // prefetched lines, so the loads after the wait see it).
    const int nv = TB ? TB * V : prm.nvec;
    const int64_t rv = (int64_t)blockIdx.x * nv;
    const uint32_t bytes = (uint32_t)nv * 16u;
    const int i = threadIdx.x;
    if (i < prm.P)
      bulk_prefetch_l2(prm.parts[i] + rv, bytes);
    else if (i == prm.P && NORM && prm.residual != nullptr)
      bulk_prefetch_l2(prm.residual + rv, bytes);
    else if (i == prm.P + 1 && NORM)
      bulk_prefetch_l2(prm.weight, bytes);
  }
  pdl_enter();

  const int T = TB ? TB : (int)blockDim.x, t = threadIdx.x, lane = t & 31;
  const int nvec = TB ? TB * V : prm.nvec;
  int64_t row;
  int rank = 0;
  if constexpr (CL) {
    cg::cluster_group cl = cg::this_cluster();
    rank = (int)cl.block_rank();
    row = blockIdx.x / cl.num_blocks();
  } else {
    row = blockIdx.x;
  }
  const int seg_base = TB ? 0 : rank * prm.seg, seg_end = TB ? nvec : seg_base + prm.seg;
  const int64_t rowv = row * (int64_t)nvec;
  const int H = nvec * 8;
  const bool has_res = NORM && prm.residual != nullptr;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

  // The block `prefetch_rows` rows later in launch order will most likely run
  // next on this SM's slot: start its row towards L2 now.
  if (!CL && prm.prefetch_rows > 0 && t == 0 && row + prm.prefetch_rows < prm.M) {
    const int64_t prow = (row + prm.prefetch_rows) * (int64_t)nvec;
    const uint32_t bytes = (uint32_t)nvec * 16u;
    for (int p = 0; p < prm.P; ++p) bulk_prefetch_l2(prm.parts[p] + prow, bytes);
    if (prm.residual != nullptr) bulk_prefetch_l2(prm.residual + prow, bytes);
  }

  // ---- 1. issue every load of this block's part of the row -------------------
  uint4 xin[V][MAXP];
  uint4 rin[V];
  uint4 win[V];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const int v = seg_base + t + k * T;
    const bool ok = TB || v < seg_end;
#pragma unroll
    for (int p = 0; p < MAXP; ++p)
      xin[k][p] = (ok && p < prm.P) ? ld_stream_nc(prm.parts[p] + rowv + v) : zero;
    if constexpr (NORM) {
      rin[k] = (ok && has_res) ? ld_stream(prm.residual + rowv + v) : zero;
      win[k] = ok ? ld_keep(prm.weight + v) : zero;
    }
  }

  uint4 yv[V];
  Fp8Scale scale_tok = {1.f, 1.f, 0.f, false};
  if constexpr (NORM) {
    // ---- 2. h, residual_out, statistics --------------------------------------------
    uint4 hv[V];
    float2 ss = make_float2(0.f, 0.f);
    float pmax = 0.f;
#pragma unroll
    for (int k = 0; k < V; ++k) {
      hv[k] = sum_vec<MAXP, IO>(xin[k], rin[k], prm.P, has_res);
      stats_vec<MODE == MODE_TOKEN, IO>(hv[k], win[k], ss, pmax);
      const int v = seg_base + t + k * T;
      if ((TB || v < seg_end) && prm.out_residual != nullptr)
        st_stream(prm.out_residual + rowv + v, hv[k]);
    }
    // ---- 3. rstd (and the per-token amax) ---------------------------------------------
    // exact-cover instances in large-M launches take the butterfly (measured
    // on B200 at sustained clocks: MXFP4 H=7168 P=4 115.6 -> 114.0 us,
    // group-128 H=8192 294.0 -> 292.0 us; decode calls keep the in-order sum,
    // 0.3 us faster there)
    const float2 tot = row_reduce<CL, MODE == MODE_TOKEN>(ss.x + ss.y, pmax, red, &cl_slot,
                                                         TB > 0 && prm.prefetch_rows > 0);
    const float rstd = row_rstd(tot.x, prm.inv_h, prm.eps);
    if (MODE == MODE_TOKEN) scale_tok = fp8_scale_direct(row_amax_from_pmax<IO>(tot.y, rstd));
    // ---- 4. y = bf16(fl(h * w) * rstd) ----------------------------------------------
#pragma unroll
    for (int k = 0; k < V; ++k) {
      yv[k] = norm_vec<IO>(hv[k], win[k], rstd);
      const int v = seg_base + t + k * T;
      if ((TB || v < seg_end) && prm.out_y != nullptr) st_stream(prm.out_y + rowv + v, yv[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < V; ++k) yv[k] = xin[k][0];
    if (MODE == MODE_TOKEN) {
      float am = 0.f;
#pragma unroll
      for (int k = 0; k < V; ++k) am = fmaxf(am, vec_absmax<IO>(yv[k]));
      scale_tok = fp8_scale_direct(row_reduce<CL, true>(0.f, am, red, &cl_slot).y);
    }
  }
  if (MODE == MODE_TOKEN && rank == 0 && t == 0)
    static_cast<float*>(prm.out_scale)[row] = scale_tok.s;

  // ---- 5. quantize y ----------------------------------------------------------------
  if constexpr (MODE == MODE_G128 && V >= 2) {
    bool ok[V];
#pragma unroll
    for (int k = 0; k < V; ++k) ok[k] = TB || seg_base + t + k * T < seg_end;
    quant_store_g128_rows<V, IO>(yv, ok, lane, row, seg_base + t, T, H, prm.out_q,
                                 static_cast<float*>(prm.out_scale), prm.scale_layout,
                                 prm.scale_ld);
  } else {
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const int v = seg_base + t + k * T;
      quant_store<MODE, IO>(yv[k], TB || v < seg_end, lane, row, v, H, scale_tok, prm.out_q,
                            prm.out_scale, prm.scale_layout, prm.scale_ld);
    }
  }

  if constexpr (CL) {
    // No block may leave while a peer can still read its shared-memory slot.
    cluster_wait();
  }
}

}  // namespace fn
