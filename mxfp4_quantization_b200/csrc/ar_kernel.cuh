// Fused all-reduce + residual add + RMSNorm + quantization across the ranks of
// a tensor-parallel group, over peer memory (the cross-GPU step that sglang
// PR #29723 fuses in front of the norm, "Motivation" and "Modifications":
// AllReduce -> RMSNorm -> quantize in one kernel).
//
// Two-stage form in one kernel: rank r owns the rows [row0, row0 + gridDim.x)
// of the batch.  Each block reads its row from every rank's partial buffer
// (peer loads), sums them in rank order with the residual (the reduce-scatter
// step, in the order of the one-GPU kernel's partial sum), normalises and
// quantizes it, and writes residual_out, y and the quantized tuple into every
// rank's output buffers (peer stores: the all-gather step).  Every row is
// computed once, on one rank, so all ranks end with the same bits.
//
// The one-stage form (every rank computes every row from all partials, and
// writes only its own outputs) is the one-GPU kernel itself, given the peer
// partial pointers.  Ordering between ranks (partials complete before the
// loads; pushes complete before the outputs are consumed) is the caller's
// barrier around the launch.  Loads of peer data use the coherent path.
#pragma once
#include "rq_kernel.cuh"

namespace fn {

constexpr int kMaxRanks = 8;

struct ARParams {
  RQParams rq;                     // parts: every rank's partial; residual, weight: local
  int64_t row0;                    // first row of this rank's shard
  int ndst;                        // ranks whose outputs are written (all of them)
  uint4* out_residual[kMaxRanks];  // per rank, or all nullptr
  uint4* out_y[kMaxRanks];         // per rank, or all nullptr
  uint8_t* out_q[kMaxRanks];
  void* out_scale[kMaxRanks];
};

using RQArKernel = void (*)(const ARParams);

template <int MODE, int MAXP, int V>
__global__ void __launch_bounds__(256) rq_ar_kernel(const __grid_constant__ ARParams ap) {
  __shared__ float2 red[32];
  pdl_enter();
  const RQParams& prm = ap.rq;
  const int T = blockDim.x, t = threadIdx.x, lane = t & 31;
  const int nvec = prm.nvec, H = nvec * 8;
  const int64_t row = ap.row0 + blockIdx.x;
  const int64_t rowv = row * (int64_t)nvec;
  const bool has_res = prm.residual != nullptr;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);

  uint4 xin[V][MAXP];
  uint4 rin[V];
  uint4 win[V];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const int v = t + k * T;
    const bool ok = v < nvec;
#pragma unroll
    for (int p = 0; p < MAXP; ++p)
      xin[k][p] = (ok && p < prm.P) ? ld_stream(prm.parts[p] + rowv + v) : zero;
    rin[k] = (ok && has_res) ? ld_stream(prm.residual + rowv + v) : zero;
    win[k] = ok ? ld_keep(prm.weight + v) : zero;
  }

  uint4 hv[V];
  float2 ss = make_float2(0.f, 0.f);
  float pmax = 0.f;
#pragma unroll
  for (int k = 0; k < V; ++k) {
    hv[k] = sum_vec<MAXP>(xin[k], rin[k], prm.P, has_res);
    stats_vec<MODE == MODE_TOKEN>(hv[k], win[k], ss, pmax);
    const int v = t + k * T;
    if (v < nvec && ap.out_residual[0] != nullptr)
      for (int d = 0; d < ap.ndst; ++d) st_stream(ap.out_residual[d] + rowv + v, hv[k]);
  }
  const float2 tot = row_reduce<false, MODE == MODE_TOKEN>(ss.x + ss.y, pmax, red, nullptr);
  const float rstd = row_rstd(tot.x, prm.inv_h, prm.eps);
  Fp8Scale scale_tok = {1.f, 1.f, 0.f, false};
  if (MODE == MODE_TOKEN) {
    scale_tok = fp8_scale_direct(row_amax_from_pmax(tot.y, rstd));
    if (t == 0)
      for (int d = 0; d < ap.ndst; ++d) static_cast<float*>(ap.out_scale[d])[row] = scale_tok.s;
  }
#pragma unroll
  for (int k = 0; k < V; ++k) {
    const int v = t + k * T;
    const bool ok = v < nvec;
    const uint4 y = norm_vec(hv[k], win[k], rstd);
    if (ok && ap.out_y[0] != nullptr)
      for (int d = 0; d < ap.ndst; ++d) st_stream(ap.out_y[d] + rowv + v, y);
    const QuantVec qv = quant_vec<MODE>(y, scale_tok);
    for (int d = 0; d < ap.ndst; ++d)
      store_quant<MODE>(qv, ok, lane, row, v, H, ap.out_q[d], ap.out_scale[d], prm.scale_layout,
                        prm.scale_ld);
  }
}

// Instances per quantization mode (ar_inst.cu): partial bound 2, 4 or 8
// ranks, V in {1, 2, 4, 8}.
#define FN_AR_DECL(MODE) RQArKernel rq_ar_pick_##MODE(int maxp, int V);
FN_AR_DECL(0)
FN_AR_DECL(1)
FN_AR_DECL(2)
#undef FN_AR_DECL

}  // namespace fn
