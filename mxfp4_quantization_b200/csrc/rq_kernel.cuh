// Fused (partial sum) + residual add + RMSNorm + quantization, sm_100a.
//
// Follows the unfused AllReduce -> RMSNorm -> quantize sequence that the fused
// AITER kernel of sglang PR #29723 ("Accuracy Tests") must equal, with the
// all-reduce replaced by an in-kernel sum of up to 8 same-device partials, and
// the quantization of the bf16 normed row that sgl-amd-mono PR #26's monokernel
// notes call bit-exact against stand-alone quantization.
//
// HBM-bound, no tensor cores.  One row is owned by one thread block (large M)
// or by a cluster of 2..8 blocks that exchange their partial sums through
// distributed shared memory (small M).  Each thread owns V 16-byte vectors of
// the row (8 bf16 each), vector index seg_base + threadIdx.x + k * blockDim.x,
// so a warp touches 512 contiguous bytes per tensor per k.  Every load of the
// row is issued before the first arithmetic; the row then lives in registers
// (as packed bf16) until its codes are stored, so each byte of HBM is read
// once and written once.
//
// MX blocks (32 elements) are 4 adjacent lanes, FP8 groups (128) are 16
// adjacent lanes: their amax is a 2- or 4-step xor shuffle.
#pragma once
#include <cooperative_groups.h>

#include "fn_device.cuh"
#include "rq_params.h"

namespace fn {

namespace cg = cooperative_groups;

// Cluster barrier halves (all threads of every block of the cluster take part).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Sum of `s` and max of `m` over the block and, with CL, over the cluster.
// The combination order is fixed (warps in index order, cluster ranks in rank
// order), so every block of a cluster gets the same bits.  With CL the caller
// must call cluster_wait() once before exiting: the last arrive here tells the
// peers this block is done reading their shared memory, and the wait keeps
// this block's own slot alive until every peer has read it.
template <bool CL, bool WANT_MAX>
__device__ __forceinline__ float2 row_reduce(float s, float m, float2* red, float2* cl_slot) {
  s = warp_sum(s);
  if (WANT_MAX) m = warp_max(m);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (lane == 0) red[warp] = make_float2(s, m);
  __syncthreads();
  float2 t = red[0];
  for (int i = 1; i < nw; ++i) {
    const float2 o = red[i];
    t.x += o.x;
    if (WANT_MAX) t.y = fmaxf(t.y, o.y);
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

template <int MODE, int MAXP, int V, bool NORM, bool CL>
__global__ void __launch_bounds__(CL ? 512 : 256)
    rq_kernel(const __grid_constant__ RQParams prm) {
  __shared__ float2 red[32];
  __shared__ float2 cl_slot;

  const int T = blockDim.x, t = threadIdx.x, lane = t & 31;
  int64_t row;
  int rank = 0;
  if constexpr (CL) {
    cg::cluster_group cl = cg::this_cluster();
    rank = (int)cl.block_rank();
    row = blockIdx.x / cl.num_blocks();
  } else {
    row = blockIdx.x;
  }
  const int seg_base = rank * prm.seg, seg_end = seg_base + prm.seg;
  const int64_t rowv = row * (int64_t)prm.nvec;
  const bool has_res = NORM && prm.residual != nullptr;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

  // ---- 1. issue every load of this block's part of the row -------------------
  uint4 xin[MAXP][V];
  uint4 rin[V];
  uint4 win[V];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const int v = seg_base + t + k * T;
    const bool ok = v < seg_end;
#pragma unroll
    for (int p = 0; p < MAXP; ++p)
      xin[p][k] = (ok && p < prm.P) ? ld_stream_nc(prm.parts[p] + rowv + v) : zero;
    if constexpr (NORM) {
      rin[k] = (ok && has_res) ? ld_stream(prm.residual + rowv + v) : zero;
      win[k] = ok ? ld_keep(prm.weight + v) : zero;
    }
  }

  // ---- 2. h = bf16(((x0 + x1) + ...) + r), residual_out, sum of squares ----------
  // Also max |h * w| for the per-token scale: h * w is exact in fp32 (two
  // 8-bit significands), y = bf16(fl(h * w) * rstd) is monotone in |h * w|, so
  // max |y| = bf16(fl(max |h * w| * rstd)) comes out of the same reduction.
  uint4 yv[V];
  float row_amax = 0.f;
  if constexpr (NORM) {
    uint4 hv[V];
    float ss = 0.f, pmax = 0.f;
#pragma unroll
    for (int k = 0; k < V; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a0 = bf_lo(word(xin[0][k], i)), a1 = bf_hi(word(xin[0][k], i));
#pragma unroll
        for (int p = 1; p < MAXP; ++p) {
          if (p < prm.P) {
            a0 += bf_lo(word(xin[p][k], i));
            a1 += bf_hi(word(xin[p][k], i));
          }
        }
        if (has_res) {
          a0 += bf_lo(word(rin[k], i));
          a1 += bf_hi(word(rin[k], i));
        }
        const uint32_t hw = pack_bf16x2(a0, a1);
        set_word(hv[k], i, hw);
        const float h0 = bf_lo(hw), h1 = bf_hi(hw);
        ss = fmaf(h0, h0, ss);
        ss = fmaf(h1, h1, ss);
        if (MODE == MODE_TOKEN) {
          const uint32_t ww = word(win[k], i);
          pmax = fmaxf(pmax, fmaxf(fabsf(h0 * bf_lo(ww)), fabsf(h1 * bf_hi(ww))));
        }
      }
      const int v = seg_base + t + k * T;
      if (v < seg_end && prm.out_residual != nullptr) st_stream(prm.out_residual + rowv + v, hv[k]);
    }

    // ---- 3. rstd = 1 / sqrt(mean(h^2) + eps) --------------------------------------
    const float2 tot = row_reduce<CL, MODE == MODE_TOKEN>(ss, pmax, red, &cl_slot);
    const float rstd =
        (float)(1.0 / sqrt((double)tot.x / (double)(prm.nvec * 8) + (double)prm.eps));
    if (MODE == MODE_TOKEN) row_amax = __uint_as_float(pack_bf16x2(tot.y * rstd, 0.f) << 16);

    // ---- 4. y = bf16(fl(h * w) * rstd) --------------------------------------------
#pragma unroll
    for (int k = 0; k < V; ++k) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t hw = word(hv[k], i), ww = word(win[k], i);
        const float y0 = (bf_lo(hw) * bf_lo(ww)) * rstd;
        const float y1 = (bf_hi(hw) * bf_hi(ww)) * rstd;
        set_word(yv[k], i, pack_bf16x2(y0, y1));
      }
      const int v = seg_base + t + k * T;
      if (v < seg_end && prm.out_y != nullptr) st_stream(prm.out_y + rowv + v, yv[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < V; ++k) yv[k] = xin[0][k];
    if (MODE == MODE_TOKEN) {
      float am = 0.f;
#pragma unroll
      for (int k = 0; k < V; ++k)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          am = fmaxf(am, fmaxf(fabsf(bf_lo(word(yv[k], i))), fabsf(bf_hi(word(yv[k], i)))));
      row_amax = row_reduce<CL, true>(0.f, am, red, &cl_slot).y;
    }
  }

  // ---- 5. quantize y ----------------------------------------------------------------
  const int H = prm.nvec * 8;
  if constexpr (MODE == MODE_TOKEN || MODE == MODE_G128) {
    float scale_tok = 1.f;
    if constexpr (MODE == MODE_TOKEN) {
      scale_tok = row_amax == 0.f ? 1.f : __fdiv_rn(row_amax, 448.f);
      if (rank == 0 && t == 0) static_cast<float*>(prm.out_scale)[row] = scale_tok;
    }
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const int v = seg_base + t + k * T;
      float scale = scale_tok;
      if constexpr (MODE == MODE_G128) {
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          am = fmaxf(am, fmaxf(fabsf(bf_lo(word(yv[k], i))), fabsf(bf_hi(word(yv[k], i)))));
        const float amax = group_max<16>(am);
        scale = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
        if (v < seg_end && (lane & 15) == 0)
          static_cast<float*>(prm.out_scale)[row * (H / 128) + v / 16] = scale;
      }
      uint32_t c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        c[i] = cvt_e4m3x2(__fdiv_rn(bf_lo(word(yv[k], i)), scale),
                          __fdiv_rn(bf_hi(word(yv[k], i)), scale));
      if (v < seg_end)
        st_stream(reinterpret_cast<uint2*>(prm.out_q + row * (int64_t)H) + v,
                  make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16)));
    }
  } else {  // MODE_MX
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const int v = seg_base + t + k * T;
      float f[8];
      float am = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf_lo(word(yv[k], i));
        f[2 * i + 1] = bf_hi(word(yv[k], i));
        am = fmaxf(am, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
      }
      const float amax = group_max<4>(am);
      float inv;
      const uint32_t code = mx_scale(amax, inv);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] *= inv;  // exact: a power of two
      const uint32_t q = cvt_e2m1x8(f);
      if (v < seg_end) {
        st_stream(reinterpret_cast<uint32_t*>(prm.out_q + row * (int64_t)(H / 2)) + v, q);
        if ((lane & 3) == 0)
          static_cast<uint8_t*>(prm.out_scale)[row * (H / 32) + v / 4] = (uint8_t)code;
      }
    }
  }

  if constexpr (CL) {
    // No block may leave while a peer can still read its shared-memory slot.
    cluster_wait();
  }
}

}  // namespace fn
