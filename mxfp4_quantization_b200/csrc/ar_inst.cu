// One instantiation unit of the fused all-reduce kernels: the quantization
// mode comes from -DFN_INST_MODE.
#include "ar_kernel.cuh"

#ifndef FN_INST_MODE
#error "FN_INST_MODE is required"
#endif

#define FN_AR_NAME_(m) rq_ar_pick_##m
#define FN_AR_NAME(m) FN_AR_NAME_(m)

namespace fn {

RQArKernel FN_AR_NAME(FN_INST_MODE)(int maxp, int V) {
  constexpr int MODE = FN_INST_MODE;
#define FN_AR(MP, VV) \
  if (maxp == MP && V == VV) return rq_ar_kernel<MODE, MP, VV>;
  FN_AR(2, 1) FN_AR(2, 2) FN_AR(2, 4) FN_AR(2, 8)
  FN_AR(4, 1) FN_AR(4, 2) FN_AR(4, 4) FN_AR(4, 8)
  FN_AR(8, 1) FN_AR(8, 2) FN_AR(8, 4) FN_AR(8, 8)
#undef FN_AR
  return nullptr;
}

}  // namespace fn
