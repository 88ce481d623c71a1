// One instantiation unit of the rmsnorm_quant kernels: the mode, the
// partial-count bound and the row format (0 bf16, 1 binary16) come from
// -DFN_INST_MODE / -DFN_INST_MAXP / -DFN_INST_IO.
#include <type_traits>

#include "rq_kernel.cuh"

#ifndef FN_INST_MODE
#error "FN_INST_MODE is required"
#endif
#ifndef FN_INST_MAXP
#error "FN_INST_MAXP is required"
#endif
#ifndef FN_INST_IO
#error "FN_INST_IO is required"
#endif

#define FN_CAT_(a, b, c, d) a##_##b##_##c##_##d
#define FN_CAT4(a, b, c, d) FN_CAT_(a, b, c, d)
#define FN_CAT(a, b, c) FN_CAT4(a, b, c, FN_INST_IO)

namespace fn {

RQKernel FN_CAT(rq_pick, FN_INST_MODE, FN_INST_MAXP)(int V, bool cluster, bool norm) {
  constexpr int MODE = FN_INST_MODE, MAXP = FN_INST_MAXP;
  using IO = std::conditional_t<FN_INST_IO == 1, F16, Bf16>;
  if (cluster) {
    if (!norm) return nullptr;
    return rq_kernel<MODE, MAXP, 1, true, true, 0, IO>;
  }
  if (!norm) {
    if constexpr (MAXP != 1) {
      return nullptr;
    } else {
      switch (V) {
        case 1: return rq_kernel<MODE, 1, 1, false, false, 0, IO>;
        case 2: return rq_kernel<MODE, 1, 2, false, false, 0, IO>;
        case 4: return rq_kernel<MODE, 1, 4, false, false, 0, IO>;
        case 8: return rq_kernel<MODE, 1, 8, false, false, 0, IO>;
        default: return rq_kernel<MODE, 1, 16, false, false, 0, IO>;
      }
    }
  }
  switch (V) {
    case 1: return rq_kernel<MODE, MAXP, 1, true, false, 0, IO>;
    case 2: return rq_kernel<MODE, MAXP, 2, true, false, 0, IO>;
    case 4: return rq_kernel<MODE, MAXP, 4, true, false, 0, IO>;
    case 8: return rq_kernel<MODE, MAXP, 8, true, false, 0, IO>;
    default: return rq_kernel<MODE, MAXP, 16, true, false, 0, IO>;
  }
}

// Exact-cover instances (one block of T threads per row of T * V vectors):
// T = 224 serves H = 3584, 7168, 14336; T = 256 serves H = 4096, 8192, 16384;
// T = 448 and 512 are the same rows split more finely (more warps per SM when
// the partials leave room for few blocks; the widest block for decode-sized M).
RQKernel FN_CAT(rq_exact_pick, FN_INST_MODE, FN_INST_MAXP)(int T, int V, bool norm) {
  constexpr int MODE = FN_INST_MODE, MAXP = FN_INST_MAXP;
  using IO = std::conditional_t<FN_INST_IO == 1, F16, Bf16>;
  if (!norm) {  // the quantization step alone (fn_quant): one input, MAXP = 1
    if constexpr (MAXP != 1) {
      return nullptr;
    } else {
      if (T == 224 && V == 4) return rq_kernel<MODE, 1, 4, false, false, 224, IO>;
      if (T == 256 && V == 4) return rq_kernel<MODE, 1, 4, false, false, 256, IO>;
      if (T == 256 && V == 2) return rq_kernel<MODE, 1, 2, false, false, 256, IO>;
      if (T == 224 && V == 8) return rq_kernel<MODE, 1, 8, false, false, 224, IO>;
      if (T == 256 && V == 8) return rq_kernel<MODE, 1, 8, false, false, 256, IO>;
      return nullptr;
    }
  }
#define FN_EXACT(TT, VV) \
  if (T == TT && V == VV) return rq_kernel<MODE, MAXP, VV, true, false, TT, IO>;
  FN_EXACT(224, 2) FN_EXACT(224, 4) FN_EXACT(224, 8)
  FN_EXACT(256, 2) FN_EXACT(256, 4) FN_EXACT(256, 8)
  FN_EXACT(448, 1) FN_EXACT(448, 2) FN_EXACT(448, 4)
  FN_EXACT(512, 1) FN_EXACT(512, 2) FN_EXACT(512, 4)
#undef FN_EXACT
  return nullptr;
}

}  // namespace fn
