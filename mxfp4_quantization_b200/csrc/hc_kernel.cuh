// hc_mix: the low-rank gate over the hyper-state, sm_100a.
//
// sglang PR #41880 ("Motivation"): the input mix of GatedResidual is a
// low-rank gate over the [M, 4*2560] hyper-state, run at decode-sized M <= 16
// and bound by reading the weights.  The page prints no formula; the reading
// computed here, per row x of hc = 4 streams of C values (stream s at
// [s*C, (s+1)*C)):
//     t = W_down x                  W_down bf16 [r, hc*C]   (rank r)
//     z = W_up t                    W_up   bf16 [hc*C, r]
//     u[c] = sum_s sigmoid(z[s*C + c]) * x[s*C + c]          -> bf16 [M, C]
//
// Two kernels, the second a programmatic dependent of the first, so that both
// weight factors stream from HBM at the same time:
//  * hc_down_kernel: t = W_down x.  Clusters of 8 blocks; cluster g owns CW
//    rows of W_down and its 8 blocks split the hc*C columns, so every block
//    reads one contiguous piece of each of its CW weight rows (the weight is
//    read exactly once from HBM over the grid) and the matching columns of
//    every x row.  A thread owns one 16-byte vector of the piece for up to 4
//    rows (more rows: more row groups of threads); the block reduces its
//    threads' partial sums with a warp reduce-scatter and shared memory,
//    every block stores its partials into rank 0's shared memory
//    (distributed shared memory), and after one cluster barrier rank 0 sums
//    them in rank order.  t (fp32 [M, r]) goes to the caller's workspace.
//  * hc_gate_mix_kernel: one block per cpb channels (no more blocks than
//    SMs).  Before it waits for the first kernel every thread loads its row
//    of W_up into registers and its x values; once t is visible it forms the
//    gate logits, the sigmoids and the mix.
// Every sum has a fixed order, so a launch shape always gives the same bits.
#pragma once
#include <cooperative_groups.h>

#include "fn_device.cuh"
#include "hc_params.h"

namespace fn {

// Sums of V values over the 32 lanes of a warp by recursive halving: at each
// step a lane keeps half of its values and adds the partner's copy of that
// half.  Afterwards, for V >= 32, a[i] (i < V/32) of lane l holds the warp sum
// of value l*V/32 + i; for V < 32, a[0] holds the sum of value l / (32/V).
// Every lane takes part.
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&a)[V]) {
  const int lane = threadIdx.x & 31;
  int n = V;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n >= 2) {
      const int h = n / 2;
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < h) {
          const float send = up ? a[i] : a[i + h];
          const float keep = up ? a[i + h] : a[i];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n = h;
    } else {
      a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
    }
  }
}

// t[m, g*CW + j] = sum_k x[m, k] * w_down[g*CW + j, k] for m < M, j < CW.
// Grid: (r / CW) clusters of kHcCluster blocks.  The rows are split over NG
// row groups of threads, MR rows each (MM = NG * MR rows at most): thread
// (rg, o) owns vector o of the block's piece for rows rg*MR .. rg*MR+MR-1, so
// each thread holds MR * CW partial sums (16 at most) whatever M is, and a
// block has NG times as many warps to cover its loads' latency.
// blockDim.x = NG * nv, nv = round32(K / 64) threads per row group.
template <int MR, int NG, int CW>
__global__ void __launch_bounds__(kHcDownThreads) hc_down_kernel(const __grid_constant__ HCParams p) {
  namespace cg = cooperative_groups;
  constexpr int V = MR * CW;         // partial sums per thread
  constexpr int VB = NG * V;         // per block: every row times CW
  __shared__ float red[kHcDownThreads / 32][V];
  __shared__ float slots[kHcCluster][VB];  // rank 0's: every block's partials
  pdl_enter();

  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int g = blockIdx.x / kHcCluster;
  const int kvec = p.K / 8, cvec = kvec / kHcCluster;
  const int nv = blockDim.x / NG;    // threads per row group (whole warps)
  const int tid = threadIdx.x, rg = tid / nv, o = tid % nv;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t v = (int64_t)rank * cvec + o;

  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (o < cvec) {
    uint4 w[CW], xv[MR];
#pragma unroll
    for (int j = 0; j < CW; ++j) w[j] = ld_keep(p.w_down + (int64_t)(g * CW + j) * kvec + v);
#pragma unroll
    for (int i = 0; i < MR; ++i) {
      const int m = rg * MR + i;
      xv[i] = m < p.M ? ld_stream_nc(p.x + (int64_t)m * kvec + v) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < MR; ++i) {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s = fma_bf16<false>(word(xv[i], e), word(w[j], e), s);
          s = fma_bf16<true>(word(xv[i], e), word(w[j], e), s);
        }
        acc[i * CW + j] = s;
      }
    }
  }

  // the block's sums: warps first, then each row group's warps in warp order
  warp_reduce_scatter<V>(acc);
  if constexpr (V >= 32) {
#pragma unroll
    for (int i = 0; i < V / 32; ++i) red[warp][lane * (V / 32) + i] = acc[i];
  } else {
    if (lane % (32 / V) == 0) red[warp][lane / (32 / V)] = acc[0];
  }
  __syncthreads();
  const int nwg = nv >> 5;  // warps per row group
  if (tid < VB) {
    const int grp = tid / V, idx = tid % V;
    float s = red[grp * nwg][idx];
    for (int w = 1; w < nwg; ++w) s += red[grp * nwg + w][idx];
    *cl.map_shared_rank(&slots[rank][tid], 0) = s;
  }
  // the stores into rank 0's shared memory are complete and visible to it
  // after the barrier; only rank 0 reads them, so the others may leave
  cl.sync();
  if (rank == 0 && tid < VB) {
    float s = slots[0][tid];
#pragma unroll
    for (int c = 1; c < kHcCluster; ++c) s += slots[c][tid];
    const int grp = tid / V, idx = tid % V;
    const int m = grp * MR + idx / CW, j = idx % CW;
    if (m < p.M) p.t[(int64_t)m * p.r + g * CW + j] = s;
  }
}

// u[m, c] for the channels [c0, c0 + cpb) of this block: gate logits of the
// 4 streams from t and W_up, logistic sigmoid, gated sum of the streams.
// Thread (mg, s, c) keeps W_up row s*C + c0 + c (r values, RV 16-byte vectors
// at most) in registers and forms the logits of rows 4mg .. 4mg+3 from t,
// read from shared memory transposed ([j][m], so one 16-byte read gives four
// rows, the same address for a whole m-group: a broadcast); the gates meet
// in shared memory, and thread (m, c) forms the gated sum of the streams in
// stream order.  Launched as a programmatic dependent of hc_down_kernel:
// every load that does not depend on t is issued before the wait.
// blockDim.x = 4 * cpb * ceil(M / 4).
template <int RV>
__global__ void __launch_bounds__(kHcMixThreads) hc_gate_mix_kernel(
    const __grid_constant__ HCParams p) {
  __shared__ __align__(16) float tt[RV * 8][kHcMaxRows];                    // [j][m]
  __shared__ float gs[kHcMaxRows][kHcStreams][kHcMaxMixChannels];         // gates
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int cpb = p.cpb, c0 = blockIdx.x * cpb, tid = threadIdx.x;
  const int rv = p.r / 8;
  const int mg = tid / (kHcStreams * cpb), rem = tid % (kHcStreams * cpb);
  const int s = rem / cpb, c = rem % cpb;
  // every global load first: this thread's W_up row ...
  uint4 w[RV];
  const uint4* wrow = p.w_up + ((int64_t)s * p.C + c0 + c) * rv;
#pragma unroll
  for (int q = 0; q < RV; ++q) w[q] = q < rv ? ld_keep(wrow + q) : make_uint4(0u, 0u, 0u, 0u);
  // ... and, as thread (xm, xc) of the mix, the four streams of x[xm, c0 + xc]
  const int xm = tid / cpb, xc = tid % cpb;
  const bool mixer = xm < p.M;
  float xv[kHcStreams];
  const uint16_t* xr = reinterpret_cast<const uint16_t*>(p.x) + (int64_t)xm * p.K + c0 + xc;
#pragma unroll
  for (int k = 0; k < kHcStreams; ++k)
    xv[k] = mixer ? __uint_as_float((uint32_t)__ldg(xr + (int64_t)k * p.C) << 16) : 0.f;

  // entries of t beyond M rows or r columns read as zero (they add nothing)
  for (int i = tid; i < RV * 8 * kHcMaxRows; i += blockDim.x) (&tt[0][0])[i] = 0.f;
  __syncthreads();

  // t is written by the kernel this one depends on: 16-byte loads, two per
  // thread in flight (M * r / 4 vectors: one pass for every C >= 1024), stored
  // transposed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int nt = p.M * p.r / 4;
  for (int i0 = 0; i0 < nt; i0 += 2 * blockDim.x) {
    float4 tq[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = i0 + tid + k * blockDim.x;
      tq[k] = i < nt ? __ldcg(reinterpret_cast<const float4*>(p.t) + i)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = i0 + tid + k * blockDim.x;
      if (i < nt) {
        const int m = (4 * i) / p.r, j = (4 * i) % p.r;
        tt[j][m] = tq[k].x;
        tt[j + 1][m] = tq[k].y;
        tt[j + 2][m] = tq[k].z;
        tt[j + 3][m] = tq[k].w;
      }
    }
  }
  __syncthreads();

  // logits of rows 4mg .. 4mg+3; two accumulator pairs per row pair (even
  // and odd j) halve the dependent chains
  float2 za[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 zb[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int q = 0; q < RV; ++q) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 8 * q + 2 * e;
      const float wl = bf_lo(word(w[q], e)), wh = bf_hi(word(w[q], e));
      const float4 t0 = *reinterpret_cast<const float4*>(&tt[j][4 * mg]);
      const float4 t1 = *reinterpret_cast<const float4*>(&tt[j + 1][4 * mg]);
      za[0] = fma_f32x2(make_float2(t0.x, t0.y), make_float2(wl, wl), za[0]);
      za[1] = fma_f32x2(make_float2(t0.z, t0.w), make_float2(wl, wl), za[1]);
      zb[0] = fma_f32x2(make_float2(t1.x, t1.y), make_float2(wh, wh), zb[0]);
      zb[1] = fma_f32x2(make_float2(t1.z, t1.w), make_float2(wh, wh), zb[1]);
    }
  }
  const float z[4] = {za[0].x + zb[0].x, za[0].y + zb[0].y, za[1].x + zb[1].x,
                      za[1].y + zb[1].y};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = 4 * mg + i;
    if (m < p.M) gs[m][s][c] = 1.f / (1.f + __expf(-z[i]));
  }
  __syncthreads();
  if (!mixer) return;
  float u = 0.f;
#pragma unroll
  for (int k = 0; k < kHcStreams; ++k) u = fmaf(gs[xm][k][xc], xv[k], u);
  p.out[(int64_t)xm * p.C + c0 + xc] = (uint16_t)(pack_bf16x2(u, 0.f) & 0xFFFFu);
}

}  // namespace fn
