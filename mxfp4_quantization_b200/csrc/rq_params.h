// Parameter block shared by the host dispatch and the rmsnorm_quant kernels.
#pragma once
#include <cstdint>
#include <vector_types.h>

namespace fn {

enum : int { MODE_TOKEN = 0, MODE_G128 = 1, MODE_MX = 2 };

// Scale layouts (include/fusednorm.h, FN_SCALE_*).
enum : int { SCALE_ROW_MAJOR = 0, SCALE_SWIZZLE_32_4_4 = 1, SCALE_MN_MAJOR = 2 };

struct RQParams {
  const uint4* parts[8];   // P bf16 [M, H] inputs (as 16-byte vectors)
  const uint4* residual;   // bf16 [M, H] or nullptr
  const uint4* weight;     // bf16 [H]
  uint4* out_residual;     // bf16 [M, H] or nullptr (may equal residual)
  uint4* out_y;            // bf16 [M, H] or nullptr
  uint8_t* out_q;          // codes
  void* out_scale;         // fp32 or E8M0 bytes
  int64_t M;
  int nvec;                // H / 8
  int seg;                 // vectors of a row handled by one block
  int P;                   // partial count, <= MAXP
  float eps;
  float inv_h;             // 1 / H (fp32), for the mean of squares
  int prefetch_rows;       // L2 prefetch distance in rows of this block (0: none); a
                           // positive distance also marks a large-M launch (row_reduce)
  int prefetch_self;       // one block per row: L2-prefetch the block's own row inputs
                           // before the programmatic-launch wait
  int scale_layout;        // SCALE_*
  int64_t scale_ld;        // swizzled: column tiles per row tile; MN-major: row stride
};

// A kernel instance: every (mode, partial bound, vectors per thread, norm,
// cluster) combination has the same signature.
using RQKernel = void (*)(const RQParams);

// Per-(mode, partial bound) instantiation units, each compiled separately
// (rq_inst.cu) so the library builds in parallel.  `V` is ignored for
// cluster launches (always one vector per thread there).

// IO: 0 = bf16 rows, 1 = binary16 rows.
#define FN_RQ_DECL(MODE, MAXP, IO)                                          \
  RQKernel rq_pick_##MODE##_##MAXP##_##IO(int V, bool cluster, bool norm); \
  RQKernel rq_exact_pick_##MODE##_##MAXP##_##IO(int T, int V, bool norm);
#define FN_RQ_DECL_IO(MODE, MAXP) FN_RQ_DECL(MODE, MAXP, 0) FN_RQ_DECL(MODE, MAXP, 1)
FN_RQ_DECL_IO(0, 1)
FN_RQ_DECL_IO(0, 2)
FN_RQ_DECL_IO(0, 4)
FN_RQ_DECL_IO(0, 8)
FN_RQ_DECL_IO(1, 1)
FN_RQ_DECL_IO(1, 2)
FN_RQ_DECL_IO(1, 4)
FN_RQ_DECL_IO(1, 8)
FN_RQ_DECL_IO(2, 1)
FN_RQ_DECL_IO(2, 2)
FN_RQ_DECL_IO(2, 4)
FN_RQ_DECL_IO(2, 8)
#undef FN_RQ_DECL_IO
#undef FN_RQ_DECL

}  // namespace fn
