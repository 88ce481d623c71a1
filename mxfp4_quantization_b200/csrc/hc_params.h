// Parameter block and instance table of the hc_mix kernels (hc_kernel.cuh),
// shared by the host dispatch and the instantiation unit.
#pragma once
#include <cstdint>
#include <vector_types.h>

namespace fn {

struct HCParams {
  const uint4* x;       // bf16 [M, hc*C] (16-byte vectors)
  const uint4* w_down;  // bf16 [r, hc*C]
  const uint4* w_up;    // bf16 [hc*C, r]
  float* t;             // workspace: fp32 [M, r]
  uint16_t* out;        // bf16 [M, C]
  int M, C, K, r;       // K = hc * C
  int cpb;              // channels per block of hc_gate_mix_kernel
  int prefetch;         // hc_down_kernel: L2-prefetch its pieces before its wait
};

constexpr int kHcStreams = 4;     // hc: the streams of the hyper-state
constexpr int kHcCluster = 8;     // blocks per cluster of hc_down_kernel (column split)
constexpr int kHcMaxRows = 16;         // M <= 16 (decode-sized)
constexpr int kHcMaxRank = 128;        // r <= 128
constexpr int kHcMaxMixChannels = 32;  // channels per block of hc_gate_mix_kernel, at most
constexpr int kHcMixThreads = 512;     // a warp per 8 of the 4 x channels W_up rows, at most
constexpr int kHcDownThreads = 1024;   // row groups x (one 16-byte vector per thread)
constexpr int kHcMaxK = 16384;         // hc*C: K / 64 <= 256 vectors per block and row group

// Instances (hc_inst.cu): hc_down_kernel for rows bound MM in {1, 2, 4, 8, 16}
// (rows per thread MR = min(MM, 4), row groups MM / MR) and weight rows per
// cluster CW in {1, 2, 4}; hc_gate_mix_kernel for W_up
// row vectors RV in {1, 2, 4, 8, 16} (rows of r <= 8 * RV values).
using HCKernel = void (*)(const HCParams);
HCKernel hc_down_pick(int mm, int cw);
HCKernel hc_gate_mix_pick(int rv);

}  // namespace fn
