// Instances of the hc_mix kernels: the column-split kernel per rows bound and
// weight rows per block, the gate-and-mix kernel per W_up row length.
#include "hc_kernel.cuh"

namespace fn {

HCKernel hc_down_pick(int mm, int cw) {
#define FN_HC(MM, MR, NG)                             \
  if (mm == MM) {                                     \
    if (cw == 1) return hc_down_kernel<MR, NG, 1>;    \
    if (cw == 2) return hc_down_kernel<MR, NG, 2>;    \
    if (cw == 4) return hc_down_kernel<MR, NG, 4>;    \
    return nullptr;                                   \
  }
  FN_HC(1, 1, 1) FN_HC(2, 2, 1) FN_HC(4, 4, 1) FN_HC(8, 4, 2) FN_HC(16, 4, 4)
#undef FN_HC
  return nullptr;
}

HCKernel hc_gate_mix_pick(int rv) {
  if (rv <= 1) return hc_gate_mix_kernel<1>;
  if (rv <= 2) return hc_gate_mix_kernel<2>;
  if (rv <= 4) return hc_gate_mix_kernel<4>;
  if (rv <= 8) return hc_gate_mix_kernel<8>;
  if (rv <= 16) return hc_gate_mix_kernel<16>;
  return nullptr;
}

}  // namespace fn
