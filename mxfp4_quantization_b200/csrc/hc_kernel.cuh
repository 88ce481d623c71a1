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
//    read exactly once over the grid) and the matching columns of every x row.
//    A thread owns one 16-byte vector of the piece; the block reduces its
//    threads' M * CW partial sums with a warp reduce-scatter and shared
//    memory, and the cluster's 8 partials meet in distributed shared memory,
//    summed by rank 0 in rank order.  t (fp32 [M, r]) goes to the caller's
//    workspace.
//  * hc_gate_mix_kernel: one block per 16 channels.  Before it waits for the
//    first kernel it stages its 4 * 16 rows of W_up (converted to fp32,
//    laid out [j][c][s]) and its slice of every x row in shared memory; once
//    t is visible it forms the 64 gate logits of each row, the sigmoids and
//    the mix.
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
// Grid: (r / CW) clusters of kHcCluster blocks; blockDim.x = the larger of
// round32(K / 64) and M * CW, at most kHcDownThreads.
template <int MM, int CW>
__global__ void __launch_bounds__(kHcDownThreads) hc_down_kernel(const __grid_constant__ HCParams p) {
  namespace cg = cooperative_groups;
  constexpr int V = MM * CW;
  __shared__ float red[kHcDownThreads / 32][V];
  __shared__ float part[V];
  pdl_enter();

  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int g = blockIdx.x / kHcCluster;
  const int kvec = p.K / 8, cvec = kvec / kHcCluster;
  const int o = threadIdx.x, lane = o & 31, warp = o >> 5;
  const int64_t v = (int64_t)rank * cvec + o;

  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (o < cvec) {
    uint4 w[CW], xv[MM];
#pragma unroll
    for (int j = 0; j < CW; ++j) w[j] = ld_stream_nc(p.w_down + (int64_t)(g * CW + j) * kvec + v);
#pragma unroll
    for (int m = 0; m < MM; ++m)
      xv[m] = m < p.M ? ld_stream_nc(p.x + (int64_t)m * kvec + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int m = 0; m < MM; ++m) {
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s = fma_bf16<false>(word(xv[m], i), word(w[j], i), s);
          s = fma_bf16<true>(word(xv[m], i), word(w[j], i), s);
        }
        acc[m * CW + j] = s;
      }
    }
  }

  // the block's sums: warps first, then the warps' results in warp order
  warp_reduce_scatter<V>(acc);
  if constexpr (V >= 32) {
#pragma unroll
    for (int i = 0; i < V / 32; ++i) red[warp][lane * (V / 32) + i] = acc[i];
  } else {
    if (lane % (32 / V) == 0) red[warp][lane / (32 / V)] = acc[0];
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  if (o < V) {
    float s = red[0][o];
    for (int w = 1; w < nw; ++w) s += red[w][o];
    part[o] = s;
  }
  // the cluster's sums, read by rank 0 from every block's shared memory
  cl.sync();
  if (rank == 0 && o < V) {
    float s = *cl.map_shared_rank(&part[o], 0);
#pragma unroll
    for (int c = 1; c < kHcCluster; ++c) s += *cl.map_shared_rank(&part[o], c);
    const int m = o / CW, j = o % CW;
    if (m < p.M) p.t[(int64_t)m * p.r + g * CW + j] = s;
  }
  // no block leaves while rank 0 may still read its shared memory
  cl.sync();
}

// u[m, c] for the kHcChannels channels of this block: gate logits of the 4
// streams from t and W_up, logistic sigmoid, gated sum of the streams.
// Launched as a programmatic dependent of hc_down_kernel: everything that
// does not depend on t is staged before the wait.  blockDim.x = 256.
__global__ void __launch_bounds__(kHcMixThreads) hc_gate_mix_kernel(
    const __grid_constant__ HCParams p) {
  __shared__ __align__(16) float wu[kHcMaxRank * kHcChannels * kHcStreams];  // [j][c][s]
  __shared__ __align__(16) float tt[kHcMaxRows * kHcMaxRank];                // [m][j]
  __shared__ __align__(16) uint16_t xs[kHcMaxRows][kHcStreams][kHcChannels];
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int c0 = blockIdx.x * kHcChannels;
  const int rv = p.r / 8;  // 16-byte vectors per W_up row
  // W_up rows s*C + c0 + c, in fp32 at [j][c][s]; consecutive threads take
  // consecutive channels (c fastest) so the shared stores spread over banks
  for (int i = threadIdx.x; i < kHcStreams * rv * kHcChannels; i += blockDim.x) {
    const int c = i % kHcChannels, q = (i / kHcChannels) % rv, s = i / (kHcChannels * rv);
    const uint4 wv = ld_stream_nc(p.w_up + ((int64_t)s * p.C + c0 + c) * rv + q);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 8 * q + 2 * k;
      wu[(j * kHcChannels + c) * kHcStreams + s] = bf_lo(word(wv, k));
      wu[((j + 1) * kHcChannels + c) * kHcStreams + s] = bf_hi(word(wv, k));
    }
  }
  // this block's 16 channels of every stream of every row (two vectors each)
  for (int i = threadIdx.x; i < p.M * kHcStreams * 2; i += blockDim.x) {
    const int h = i & 1, s = (i >> 1) % kHcStreams, m = i / (2 * kHcStreams);
    const uint4 xv = ld_stream_nc(p.x + ((int64_t)m * p.K + (int64_t)s * p.C + c0) / 8 + h);
    *reinterpret_cast<uint4*>(&xs[m][s][8 * h]) = xv;
  }

  // t is written by the kernel this one depends on
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i < p.M * p.r / 4; i += blockDim.x)
    reinterpret_cast<float4*>(tt)[i] = __ldcg(reinterpret_cast<const float4*>(p.t) + i);
  __syncthreads();

  const int m = threadIdx.x / kHcChannels, c = threadIdx.x % kHcChannels;
  if (m >= p.M) return;
  float2 z01 = make_float2(0.f, 0.f), z23 = make_float2(0.f, 0.f);
  const float* tm = tt + m * p.r;
  for (int j = 0; j < p.r; j += 4) {
    const float4 t4 = *reinterpret_cast<const float4*>(tm + j);
    const float tj[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 w = *reinterpret_cast<const float4*>(&wu[((j + k) * kHcChannels + c) * kHcStreams]);
      const float2 tk = make_float2(tj[k], tj[k]);
      z01 = fma_f32x2(tk, make_float2(w.x, w.y), z01);
      z23 = fma_f32x2(tk, make_float2(w.z, w.w), z23);
    }
  }
  const float z[kHcStreams] = {z01.x, z01.y, z23.x, z23.y};
  float u = 0.f;
#pragma unroll
  for (int s = 0; s < kHcStreams; ++s) {
    const float gate = 1.f / (1.f + __expf(-z[s]));
    u = fmaf(gate, __uint_as_float((uint32_t)xs[m][s][c] << 16), u);
  }
  p.out[(int64_t)m * p.C + c0 + c] = (uint16_t)(pack_bf16x2(u, 0.f) & 0xFFFFu);
}

}  // namespace fn
