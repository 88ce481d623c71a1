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
//    the other blocks store their partials into rank 0's shared memory
//    (distributed shared memory, st.async counted on rank 0's mbarrier) and
//    exit, and rank 0, once they have landed, sums them in rank order.  t
//    (fp32 [M, r]) goes to the caller's workspace.  Launched as a
//    programmatic dependent of the previous call, each block first starts
//    its pieces of W_down and x towards L2, then waits.
//  * hc_gate_mix_kernel: one block per cpb channels (no more blocks than
//    SMs).  Before it waits for the first kernel every warp loads its W_up
//    rows into tensor-core fragments and every thread its x values; once t
//    is visible the warps form the gate logits (mma tiles), the sigmoids and
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

// ---- the partial-sum handoff of hc_down_kernel ----------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// The shared::cluster address of the same variable in block `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// One 4-byte store into another block's shared memory that counts its bytes
// on that block's mbarrier (the transaction count) when it lands.
__device__ __forceinline__ void st_async_b32(uint32_t raddr, float v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               :: "r"(raddr), "r"(__float_as_uint(v)), "r"(rbar) : "memory");
}
// Whether the mbarrier's phase 0 has completed (waits a hardware-chosen
// while before answering no); acquire at cluster scope, so the stores that
// completed the phase are visible after a yes.
__device__ __forceinline__ bool mbar_phase0_done(uint32_t bar) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done) : "r"(bar) : "memory");
  return done != 0;
}
// Attempts of mbar_phase0_done before rank 0 of hc_down_kernel gives up (far
// beyond any wait that can end: the other ranks' stores land within
// microseconds of its own).
constexpr int kHcHandoffTries = 1 << 20;

// t[m, g*CW + j] = sum_k x[m, k] * w_down[g*CW + j, k] for m < M, j < CW.
// Grid: (r / CW) clusters of kHcCluster blocks.  The rows are split over NG
// row groups of threads, MR rows each (MM = NG * MR rows at most): thread
// (rg, o) owns vector o of the block's piece for rows rg*MR .. rg*MR+MR-1, so
// each thread holds MR * CW partial sums (16 at most) whatever M is, and a
// block has NG times as many warps to cover its loads' latency.
// blockDim.x = NG * nv, nv = round32(K / 64) threads per row group.
// The handoff to rank 0 is one-way: the other ranks store their partials
// into rank 0's shared memory with st.async, each store counting its bytes on
// rank 0's mbarrier, and exit; only rank 0 waits, for the byte count of all
// seven.  Rank 0 initialises the mbarrier and announces its byte count before
// an early cluster arrive, which the others wait on (long since complete by
// then) before their first store.  If the count never completes (a wait of
// kHcHandoffTries attempts) rank 0 writes NaN into its columns of t, so the
// call's outputs show the failure.
template <int MR, int NG, int CW>
__global__ void __launch_bounds__(kHcDownThreads) hc_down_kernel(const __grid_constant__ HCParams p) {
  namespace cg = cooperative_groups;
  constexpr int V = MR * CW;         // partial sums per thread
  constexpr int VB = NG * V;         // per block: every row times CW
  __shared__ float red[kHcDownThreads / 32][V];
  __shared__ float slots[kHcCluster][VB];  // rank 0's: the other blocks' partials (row 0 unused)
  __shared__ __align__(8) uint64_t handoff;  // rank 0's: the others' partials landed
  if (p.prefetch) {
    // Launched as a programmatic dependent, the block may start while the
    // previous kernel still runs: start its pieces of W_down and x towards
    // L2 before the wait (a hint with no result: data that the previous
    // kernel writes meanwhile lands in L2 over the prefetched lines, so the
    // loads after the wait see it).
    const int gq = blockIdx.x / kHcCluster, rq = blockIdx.x % kHcCluster;
    const int kv = p.K / 8, cv = kv / kHcCluster, i = threadIdx.x;
    if (i < CW)
      bulk_prefetch_l2(p.w_down + (int64_t)(gq * CW + i) * kv + rq * cv, (uint32_t)cv * 16u);
    else if (i < CW + p.M)
      bulk_prefetch_l2(p.x + (int64_t)(i - CW) * kv + rq * cv, (uint32_t)cv * 16u);
  }
  pdl_enter();

  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const uint32_t bar = smem_addr(&handoff);
  if (rank == 0 && threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(bar), "r"((kHcCluster - 1) * VB * 4) : "memory");
  }
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
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
  // rank 0's mbarrier is initialised (its early arrive is long past)
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
  if (tid >= VB) return;
  const int grp = tid / V, idx = tid % V;
  float s = red[grp * nwg][idx];
  for (int w = 1; w < nwg; ++w) s += red[grp * nwg + w][idx];
  if (rank != 0) {
    st_async_b32(cluster_map(smem_addr(&slots[rank][tid]), 0), s, cluster_map(bar, 0));
    return;
  }
  bool landed = false;
  for (int i = 0; i < kHcHandoffTries && !landed; ++i) landed = mbar_phase0_done(bar);
  if (landed) {
#pragma unroll
    for (int c = 1; c < kHcCluster; ++c) s += slots[c][tid];
  } else {
    s = __int_as_float(0x7fc00000);
  }
  const int m = grp * MR + idx / CW, j = idx % CW;
  if (m < p.M) p.t[(int64_t)m * p.r + g * CW + j] = s;
}

// D += A B for one m16n8k16 tile: A bf16 16 x 16 (row-major fragment a0..a3),
// B bf16 16 x 8 (column fragment b0, b1), D fp32 16 x 8 (d0..d3).  Lane (g,
// q) = (lane / 4, lane % 4) holds A rows g and g+8 at k = 2q, 2q+1 (a0, a1)
// and k = 2q+8, 2q+9 (a2, a3), B column g at those k (b0, b1), and D rows g
// and g+8 at columns 2q, 2q+1.
__device__ __forceinline__ void mma_bf16_16x8x16(float (&d)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two fp32 values as three bf16 pairs whose sum is the pair to within 2^-24
// relative: hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid).  Each
// difference is exact in fp32 (v and its bf16 rounding share their leading
// bits), so only the last rounding is lost.
struct Bf16Split3 {
  uint32_t hi, mid, lo;
};
__device__ __forceinline__ Bf16Split3 split3_bf16x2(float v0, float v1) {
  Bf16Split3 r;
  r.hi = pack_bf16x2(v0, v1);
  const float e0 = v0 - bf_lo(r.hi), e1 = v1 - bf_hi(r.hi);
  r.mid = pack_bf16x2(e0, e1);
  r.lo = pack_bf16x2(e0 - bf_lo(r.mid), e1 - bf_hi(r.mid));
  return r;
}

// u[m, c] for the channels [c0, c0 + cpb) of this block: gate logits of the
// 4 streams from t and W_up, logistic sigmoid, gated sum of the streams.
// The logits of the block are one small product z = t W_up^T of 16 rows
// (M <= 16; rows beyond M are zero) by 4 * cpb W_up rows (n = s * cpb + c
// is W_up row s*C + c0 + c) over the rank, on the tensor cores: warp w owns
// the 8 W_up rows 8w .. 8w+7 (one n-tile) and runs m16n8k16 tiles over the
// rank padded to 16 * KS.  t (fp32) enters as three bf16 parts (hi + mid +
// lo, exact to 2^-24 relative): every product of a part with a bf16 weight
// is exact in fp32, so the logits carry fp32 accuracy.  The thread that
// reads a vector of t splits it and stores the parts in shared memory, once
// per block; the warps read their A fragments from there and accumulate
// each part's products separately, adding them from the smallest.  The
// W_up fragments come straight from global memory.  The gates meet in
// shared memory, and thread (m, c) forms the gated sum of the streams in
// stream order.  Launched as a programmatic dependent of hc_down_kernel: the
// W_up fragments and the x values, which do not depend on t, are loaded
// before the wait.  blockDim.x = 32 * (4 * cpb / 8); the padded rank 16 * KS
// covers r (RV = r / 8 rounded up to a power of two).
template <int RV>
__global__ void __launch_bounds__(kHcMixThreads) hc_gate_mix_kernel(
    const __grid_constant__ HCParams p) {
  constexpr int KS = RV >= 2 ? RV / 2 : 1;  // k-steps of 16
  // the parts of t in shared memory: per row, per 4 columns, 8 words {hi01,
  // hi23, mid01, mid23, lo01, lo23, -, -} (bf16 pairs of columns 0-1 and
  // 2-3); row stride 32 KS + 4 words, so the two rows a quarter-warp reads
  // fall in disjoint banks
  constexpr int RS = 32 * KS + 4;
  __shared__ __align__(16) uint32_t tp[kHcMaxRows][RS];
  __shared__ float gs[kHcMaxRows][kHcStreams][kHcMaxMixChannels];  // gates
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int cpb = p.cpb, c0 = blockIdx.x * cpb, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, q = lane & 3;
  // Lane quarter q takes columns 16k + 4q .. 16k + 4q + 3 of k-step k (the
  // order of the rank inside a tile is free: the tile sums over it).  B
  // fragments: W_up row of n = 8 * warp + g at those columns; columns at or
  // beyond r (whole 4-column chunks, since r % 8 == 0) are zero.
  uint32_t b[KS][2];
  {
    const int n = 8 * warp + g;
    const uint16_t* wrow =
        reinterpret_cast<const uint16_t*>(p.w_up) + ((int64_t)(n / cpb) * p.C + c0 + n % cpb) * p.r;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const int col = 16 * k + 4 * q;
      const uint2 w = col < p.r ? __ldg(reinterpret_cast<const uint2*>(wrow + col)) : make_uint2(0u, 0u);
      b[k][0] = w.x;
      b[k][1] = w.y;
    }
  }
  // ... and, as thread (xm, xc) of the mix, the four streams of x[xm, c0 + xc]
  const int xm = tid / cpb, xc = tid % cpb;
  const bool mixer = xm < p.M;
  float xv[kHcStreams];
  const uint16_t* xr = reinterpret_cast<const uint16_t*>(p.x) + (int64_t)xm * p.K + c0 + xc;
#pragma unroll
  for (int k = 0; k < kHcStreams; ++k)
    xv[k] = mixer ? __uint_as_float((uint32_t)__ldg(xr + (int64_t)k * p.C) << 16) : 0.f;

  // entries of t beyond M rows or r columns read as zero (they add nothing);
  // cleared before the wait, where the barrier costs nothing
  for (int i = tid; i < kHcMaxRows * RS / 4; i += blockDim.x)
    reinterpret_cast<uint4*>(&tp[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();

  // t is written by the kernel this one depends on: 16-byte loads, two per
  // thread in flight (M * r / 4 vectors: one pass for every C >= 256), each
  // split into its parts
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
      if (i >= nt) continue;
      const Bf16Split3 v01 = split3_bf16x2(tq[k].x, tq[k].y), v23 = split3_bf16x2(tq[k].z, tq[k].w);
      uint32_t* dst = &tp[(4 * i) / p.r][2 * ((4 * i) % p.r)];
      *reinterpret_cast<uint4*>(dst) = make_uint4(v01.hi, v23.hi, v01.mid, v23.mid);
      *reinterpret_cast<uint2*>(dst + 4) = make_uint2(v01.lo, v23.lo);
    }
  }
  __syncthreads();

  // one chain of tiles per part; rows g+8 only where M has them (warp-uniform)
  float dh[4] = {0.f, 0.f, 0.f, 0.f}, dm[4] = {0.f, 0.f, 0.f, 0.f}, dl[4] = {0.f, 0.f, 0.f, 0.f};
  const bool upper = p.M > 8;
#pragma unroll
  for (int k = 0; k < KS; ++k) {
    const uint32_t* ra = &tp[g][8 * (4 * k + q)];
    const uint32_t* rb = &tp[g + 8][8 * (4 * k + q)];
    const uint4 a4 = *reinterpret_cast<const uint4*>(ra);
    const uint2 a2 = *reinterpret_cast<const uint2*>(ra + 4);
    const uint4 b4 = upper ? *reinterpret_cast<const uint4*>(rb) : make_uint4(0u, 0u, 0u, 0u);
    const uint2 b2 = upper ? *reinterpret_cast<const uint2*>(rb + 4) : make_uint2(0u, 0u);
    const uint32_t hi[4] = {a4.x, b4.x, a4.y, b4.y};
    const uint32_t mid[4] = {a4.z, b4.z, a4.w, b4.w};
    const uint32_t lo[4] = {a2.x, b2.x, a2.y, b2.y};
    mma_bf16_16x8x16(dl, lo, b[k][0], b[k][1]);
    mma_bf16_16x8x16(dm, mid, b[k][0], b[k][1]);
    mma_bf16_16x8x16(dh, hi, b[k][0], b[k][1]);
  }
  // z at rows g, g+8 and W_up rows n = 8 * warp + 2q, 2q+1: the same stream
  // (n is even and cpb a multiple of 4), channels cc and cc + 1
  const int n0 = 8 * warp + 2 * q, sn = n0 / cpb, cc = n0 % cpb;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = g + 8 * (i >> 1);
    if (m < p.M) gs[m][sn][cc + (i & 1)] = 1.f / (1.f + __expf(-((dl[i] + dm[i]) + dh[i])));
  }
  __syncthreads();
  if (!mixer) return;
  float u = 0.f;
#pragma unroll
  for (int k = 0; k < kHcStreams; ++k) u = fmaf(gs[xm][k][xc], xv[k], u);
  p.out[(int64_t)xm * p.C + c0 + xc] = (uint16_t)(pack_bf16x2(u, 0.f) & 0xFFFFu);
}

}  // namespace fn
