// Host side of libfusednorm.so: argument checks, dispatch, launches.
// The C ABI and its contract are declared in include/fusednorm.h.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "fusednorm.h"
#include "ar_kernel.cuh"
#include "hc_params.h"
#include "qk_kernel.cuh"
#include "rq_params.h"

namespace {

thread_local int tl_variant = FN_VARIANT_NONE;
thread_local int32_t tl_launch[4] = {0, 0, 0, 0};
thread_local int tl_prefer = FN_VARIANT_NONE;
thread_local int tl_pdl = 0;  // launch as a programmatic dependent (fn_programmatic_launch)

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

Range range_of(const void* p, int64_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Range{lo, lo + static_cast<uintptr_t>(bytes)};
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

int round32(int x) { return (x + 31) / 32 * 32; }

// ---- rmsnorm_quant / quant dispatch -----------------------------------------

using fn::RQKernel;

// Kernel instance for (mode, P, V, cluster, norm).
// `f16`: binary16 rows (FN_IO_FP16), else bf16.
RQKernel pick_kernel(int mode, int P, int V, bool cluster, bool norm, bool f16) {
  const int maxp = (!norm || P == 1) ? 1 : P == 2 ? 2 : P <= 4 ? 4 : 8;
#define FN_CASE(MODE, MAXP)                                                       \
  if (mode == MODE && maxp == MAXP)                                               \
    return f16 ? fn::rq_pick_##MODE##_##MAXP##_1(V, cluster, norm)                \
               : fn::rq_pick_##MODE##_##MAXP##_0(V, cluster, norm);
  FN_CASE(0, 1) FN_CASE(0, 2) FN_CASE(0, 4) FN_CASE(0, 8)
  FN_CASE(1, 1) FN_CASE(1, 2) FN_CASE(1, 4) FN_CASE(1, 8)
  FN_CASE(2, 1) FN_CASE(2, 2) FN_CASE(2, 4) FN_CASE(2, 8)
#undef FN_CASE
  return nullptr;
}

// The exact-cover instance for a row of T * V vectors, or nullptr.
RQKernel pick_exact_kernel(int mode, int P, int T, int V, bool f16, bool norm = true) {
  const int maxp = P == 1 ? 1 : P == 2 ? 2 : P <= 4 ? 4 : 8;
#define FN_CASE(MODE, MAXP)                                                              \
  if (mode == MODE && maxp == MAXP)                                                      \
    return f16 ? fn::rq_exact_pick_##MODE##_##MAXP##_1(T, V, norm)                       \
               : fn::rq_exact_pick_##MODE##_##MAXP##_0(T, V, norm);
  FN_CASE(0, 1) FN_CASE(0, 2) FN_CASE(0, 4) FN_CASE(0, 8)
  FN_CASE(1, 1) FN_CASE(1, 2) FN_CASE(1, 4) FN_CASE(1, 8)
  FN_CASE(2, 1) FN_CASE(2, 2) FN_CASE(2, 4) FN_CASE(2, 8)
#undef FN_CASE
  return nullptr;
}

// Smallest power-of-two V in {1..vmax} with ceil(nvec / V) <= max_threads.
int vectors_per_thread(int nvec, int max_threads, int vmax) {
  int V = 1;
  while (V < vmax && (nvec + V - 1) / V > max_threads) V *= 2;
  return V;
}

int row_vectors_per_thread(int nvec) { return vectors_per_thread(nvec, 256, 16); }

// L2 prefetch distance, in rows, of the one-block-per-row kernel, in units of
// SMs: a block starts the row 2 * #SMs blocks later towards L2, about one
// wave ahead.  Measured on B200 (prefill MXFP4 H=7168 P=4 / group-128
// H=8192 P=1): 0 -> 121.8 / 315 us, 2 SMs' worth -> 114.6 / 281-305 us;
// 4 SMs' worth and more is slower again.
constexpr int kRowPrefetchSms = 2;

// True when `p` is device memory of device `dev`.  The L2 bulk prefetch is
// issued only on such memory: a partial that lives on a peer GPU (the
// one-stage form of the fused all-reduce passes the peers' partials here) or
// in host memory is read with plain loads alone, so no bulk operation ever
// takes another device's memory as its source.
bool on_device(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// Every row input of a call (the partials and the residual) is on `dev`.
bool rows_on_device(const fn::RQParams& p, int dev) {
  for (int i = 0; i < p.P; ++i)
    if (!on_device(p.parts[i], dev)) return false;
  return p.residual == nullptr || on_device(p.residual, dev);
}

// Launch `k(args...)` on `st`: with a cluster dimension when `cluster` > 1,
// and, when the calling thread asked for it (fn_programmatic_launch), as a
// programmatic dependent of the work before it on the stream.  Every kernel
// starts by waiting for the grids it depends on (griddepcontrol.wait), so the
// dependent launch only lets its blocks be scheduled early.
template <typename... KArgs, typename... Args>
int launch_kernel_pdl(void (*k)(KArgs...), unsigned grid, unsigned threads, size_t smem,
                      cudaStream_t st, int cluster, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = (unsigned)n;
  if (cudaLaunchKernelEx(&cfg, k, args...) != cudaSuccess) {
    (void)cudaGetLastError();
    return FN_ERR_CUDA;
  }
  return FN_OK;
}

template <typename... KArgs, typename... Args>
int launch_kernel(void (*k)(KArgs...), unsigned grid, unsigned threads, size_t smem,
                  cudaStream_t st, int cluster, Args... args) {
  return launch_kernel_pdl(k, grid, threads, smem, st, cluster, tl_pdl != 0, args...);
}

// Fewest resident warps per SM the one-block-per-row kernel should run with
// before its row is split more finely.  Measured on B200 (sustained, power
// capped): MXFP4 H=7168 P=4 at 224 threads x 4 vectors (114 registers, 2
// blocks = 14 warps per SM) 118.4 us; at 448 x 2 (28 warps) 115.5 us even at a
// 70 MHz lower SM clock.  Group-128 H=8192 P=1 already runs 32 warps at 256 x 4
// (297.2 us) and loses at 512 x 2 (310.6 us): more warps only pay below ~16.
constexpr int kMinRowWarps = 16;

// Resident warps per SM of `k` at `threads` per block (-1 if the runtime
// cannot tell), cached per (kernel, block size).
int resident_warps(RQKernel k, int threads) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  const auto key = std::make_pair(reinterpret_cast<const void*>(k), threads);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int blocks = 0;
  int w = -1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, k, threads, 0) == cudaSuccess)
    w = blocks * (threads / 32);
  else
    (void)cudaGetLastError();
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = w;
  return w;
}

// The block for a decode-sized launch (M at most one row per SM): the fewest
// vectors per thread V <= 4 with at most 512 threads per row, taken from an
// exact-cover instance or, up to 256 threads, the generic one.  Each thread's
// chain of dependent steps is then shortest, with no cluster barrier.
// Measured on B200 (CUDA graph, cold inputs, programmatic launch), H=7168:
// MXFP4 M=1/16 2.33/2.51 us at 448 x 2 against 2.94/3.31 us for an 8-block
// cluster and 2.60/2.80 us at 224 x 4; group-128 2.77/2.94 against
// 3.16/3.54 and 3.31/3.52; per-token 2.32/2.50 against 2.95/3.34 and
// 2.30/2.51; H=2048 M=16 per-token 2.01 us at 256 x 1 against 3.06 us.
// nullptr when no such block exists (the cluster kernel is used).
RQKernel wide_row_block(int mode, int P, int nvec, bool f16, int* T, int* V) {
  for (int v = 1; v <= 4; v *= 2) {
    const int t = round32((nvec + v - 1) / v);
    if (t > 512) continue;
    RQKernel k = t * v == nvec ? pick_exact_kernel(mode, P, t, v, f16) : nullptr;
    if (!k && t <= 256) k = pick_kernel(mode, P, v, false, true, f16);
    if (k) {
      *T = t;
      *V = v;
      return k;
    }
  }
  return nullptr;
}

// Cluster size for a small-M launch: the largest C in 2..8 that splits the
// row into equal segments aligned to the quantization group, each at most 512
// vectors, with M * C blocks fitting on the GPU at once.  0 when none fits.
int pick_cluster(int64_t M, int nvec, int mode, int sms) {
  const int align = mode == FN_FP8_PER_GROUP128 ? 16 : mode == FN_MXFP4 ? 4 : 1;
  for (int C = 8; C >= 2; --C) {
    if (nvec % C) continue;
    const int seg = nvec / C;
    if (seg % align || seg > 512 || seg < 32) continue;
    if (M * C > sms) continue;
    return C;
  }
  return 0;
}

// `mode` carries the quantization (low byte), scale-layout and row-format flags.
struct ModeInfo {
  int q = -1;       // FN_FP8_PER_TOKEN / FN_FP8_PER_GROUP128 / FN_MXFP4
  int layout = 0;   // fn::SCALE_ROW_MAJOR / SCALE_SWIZZLE_32_4_4 / SCALE_MN_MAJOR
  bool f16 = false; // FN_IO_FP16: the 16-bit tensors are IEEE binary16
};

int parse_mode(int mode, ModeInfo* mi) {
  const int q = mode & FN_MODE_MASK, flags = mode & ~(FN_MODE_MASK | FN_IO_FP16);
  if (q < FN_FP8_PER_TOKEN || q > FN_MXFP4) return FN_ERR_INVALID;
  mi->q = q;
  mi->f16 = (mode & FN_IO_FP16) != 0;
  mi->layout = fn::SCALE_ROW_MAJOR;
  if (flags == FN_SCALE_SWIZZLE_32_4_4) {
    if (q != FN_MXFP4) return FN_ERR_INVALID;
    mi->layout = fn::SCALE_SWIZZLE_32_4_4;
  } else if (flags == FN_SCALE_MN_MAJOR) {
    if (q != FN_FP8_PER_GROUP128) return FN_ERR_INVALID;
    mi->layout = fn::SCALE_MN_MAJOR;
  } else if (flags != 0) {
    return FN_ERR_INVALID;
  }
  return FN_OK;
}

int check_mode_shape(const ModeInfo& mi, int64_t M, int64_t H) {
  if (M < 0 || H <= 0 || H % 8) return FN_ERR_INVALID;
  if (mi.q == FN_FP8_PER_GROUP128 && H % 128) return FN_ERR_INVALID;
  if (mi.q == FN_MXFP4 && H % 32) return FN_ERR_INVALID;
  if (H > FN_MAX_H) return FN_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX / 8) return FN_ERR_UNSUPPORTED;  // grid size
  return FN_OK;
}

int64_t code_bytes(const ModeInfo& mi, int64_t M, int64_t H) {
  return mi.q == FN_MXFP4 ? M * H / 2 : M * H;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Bytes of the scale buffer, including a layout's padding.
int64_t scale_bytes(const ModeInfo& mi, int64_t M, int64_t H) {
  if (mi.q == FN_FP8_PER_TOKEN) return M * 4;
  if (mi.q == FN_FP8_PER_GROUP128)
    return (mi.layout == fn::SCALE_MN_MAJOR ? round_up(M, 4) : M) * (H / 128) * 4;
  if (mi.layout == fn::SCALE_SWIZZLE_32_4_4) return round_up(M, 128) * round_up(H / 32, 4);
  return M * (H / 32);
}

// The kernel's scale-index parameter for a layout.
int64_t scale_ld(const ModeInfo& mi, int64_t M, int64_t H) {
  if (mi.layout == fn::SCALE_SWIZZLE_32_4_4) return round_up(H / 32, 4) / 4;  // column tiles
  if (mi.layout == fn::SCALE_MN_MAJOR) return round_up(M, 4);
  return 0;
}

int check_outputs_align(const ModeInfo& mi, const void* out_q, const void* out_scale) {
  if (!aligned(out_q, mi.q == FN_MXFP4 ? 4 : 8)) return FN_ERR_ALIGN;
  if (mi.q != FN_MXFP4 && !aligned(out_scale, 4)) return FN_ERR_ALIGN;
  return FN_OK;
}

int launch_rq(const fn::RQParams& prm, int mode, int P, int64_t M, bool norm, bool f16,
              void* stream, int variant_if_norm) {
  // `mode` is the quantization alone here (the layout travels in prm)
  const int nvec = prm.nvec;
  const int sms = sm_count();
  if (sms <= 0) return FN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fn::RQParams p = prm;

  const int pref = tl_prefer;
  // Decode-sized M: one wide block per row when one fits (see wide_row_block).
  int wide_T = 0, wide_V = 0;
  RQKernel wide_k = nullptr;
  if (norm && M <= sms && pref != FN_VARIANT_ROW_CLUSTER)
    wide_k = wide_row_block(mode, P, nvec, f16, &wide_T, &wide_V);
  int C = norm && !wide_k ? pick_cluster(M, nvec, mode, sms) : 0;
  if (pref == FN_VARIANT_ROW_CTA) C = 0;

  if (C >= 2) {
    p.seg = nvec / C;
    const int threads = round32(p.seg);
    RQKernel k = pick_kernel(mode, P, 1, true, true, f16);
    if (!k) return FN_ERR_UNSUPPORTED;
    if (launch_kernel(k, (unsigned)(M * C), (unsigned)threads, 0, st, C, p) != FN_OK)
      return FN_ERR_CUDA;
    tl_variant = FN_VARIANT_ROW_CLUSTER;
    tl_launch[0] = (int32_t)(M * C);
    tl_launch[1] = threads;
    tl_launch[2] = C;
    tl_launch[3] = 1;
  } else {
    int V = wide_k ? wide_V : row_vectors_per_thread(nvec);
    p.seg = nvec;
    p.prefetch_rows = M > (int64_t)kRowPrefetchSms * sms ? kRowPrefetchSms * sms : 0;
    if (p.prefetch_rows > 0) {
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess) return FN_ERR_CUDA;
      if (!rows_on_device(p, dev)) p.prefetch_rows = 0;
    }
    // as a programmatic dependent, each block prefetches its own row before
    // its wait (never from another device's memory)
    p.prefetch_self = 0;
    if (tl_pdl && p.prefetch_rows == 0) {
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess) return FN_ERR_CUDA;
      p.prefetch_self =
          rows_on_device(p, dev) && (!norm || on_device(p.weight, dev)) ? 1 : 0;
    }
    int threads = wide_k ? wide_T : round32((nvec + V - 1) / V);
    RQKernel k = wide_k;
    if (!k && threads * V == nvec) k = pick_exact_kernel(mode, P, threads, V, f16, norm);
    if (k && !wide_k && V >= 4) {
      // Many partials held in registers leave room for few blocks per SM:
      // below kMinRowWarps resident warps, split the row twice as finely.
      const int w = resident_warps(k, threads);
      RQKernel k2 = w >= 0 && w < kMinRowWarps
                        ? pick_exact_kernel(mode, P, 2 * threads, V / 2, f16)
                        : nullptr;
      if (k2 && resident_warps(k2, 2 * threads) > w) {
        k = k2;
        threads *= 2;
        V /= 2;
      }
    }
    if (!k) k = pick_kernel(mode, P, V, false, norm, f16);
    if (!k) return FN_ERR_UNSUPPORTED;
    if (launch_kernel(k, (unsigned)M, (unsigned)threads, 0, st, 1, p) != FN_OK)
      return FN_ERR_CUDA;
    tl_variant = norm ? variant_if_norm : FN_VARIANT_QUANT_ONLY;
    tl_launch[0] = (int32_t)M;
    tl_launch[1] = threads;
    tl_launch[2] = p.prefetch_self ? -1 : p.prefetch_rows;
    tl_launch[3] = V;
  }
  return FN_OK;
}

template <int VPL, bool FP8>
int launch_qk_v(const fn::QKParams& p, int64_t items, int sms, cudaStream_t st) {
  const int wpb = items <= (int64_t)8 * sms ? 1 : 8;
  const int64_t blocks = (items + wpb - 1) / wpb;
  if (launch_kernel(fn::qk_kernel<VPL, FP8>, (unsigned)blocks, (unsigned)(wpb * 32), 0, st, 1,
                    p) != FN_OK)
    return FN_ERR_CUDA;
  tl_launch[0] = (int32_t)blocks;
  tl_launch[1] = wpb * 32;
  tl_launch[2] = 1;
  tl_launch[3] = VPL;
  return FN_OK;
}


// Shared body of fn_qk_norm_gate and fn_qk_norm_gate_fp8 (fp8 when out_q8 or
// out_k8 is given; the bf16 q / k outputs are then optional).
int qk_impl(const void* qkv, int64_t M, int64_t row_stride, int Hq, int Hk, int D,
            const void* q_weight, const void* k_weight, float eps, void* out_q, void* out_k,
            void* out_gate, void* out_q8, void* out_qs, void* out_k8, void* out_ks,
            void* stream) {
  tl_variant = FN_VARIANT_NONE;
  const bool fp8 = out_q8 != nullptr || out_k8 != nullptr;
  if (M < 0 || Hq < 0 || Hk < 0 || Hq + Hk < 1 || D <= 0 || D % 8) return FN_ERR_INVALID;
  if (D > FN_MAX_HEAD_DIM) return FN_ERR_UNSUPPORTED;
  if (row_stride % 8 || row_stride < (int64_t)(2 * Hq + Hk) * D) return FN_ERR_INVALID;
  if (!std::isfinite(eps) || eps < 0.f) return FN_ERR_INVALID;
  if (M == 0) return FN_OK;
  if (!qkv || (Hq > 0 && (!q_weight || !out_gate || (!out_q && !fp8))) ||
      (Hk > 0 && (!k_weight || (!out_k && !fp8))))
    return FN_ERR_INVALID;
  if (!aligned(qkv, 16) || (q_weight && !aligned(q_weight, 16)) ||
      (k_weight && !aligned(k_weight, 16)) || (out_q && !aligned(out_q, 16)) ||
      (out_k && !aligned(out_k, 16)) || (out_gate && !aligned(out_gate, 16)) ||
      (out_q8 && !aligned(out_q8, 8)) || (out_k8 && !aligned(out_k8, 8)) ||
      (out_qs && !aligned(out_qs, 4)) || (out_ks && !aligned(out_ks, 4)))
    return FN_ERR_ALIGN;
  if (M > (int64_t)INT32_MAX / 8 || (int64_t)M * (Hq + Hk) > (int64_t)INT32_MAX)
    return FN_ERR_UNSUPPORTED;
  {
    const Range in = range_of(qkv, ((M - 1) * row_stride + (int64_t)(2 * Hq + Hk) * D) * 2);
    Range outs[7];
    int no = 0;
    if (Hq > 0) {
      if (out_q) outs[no++] = range_of(out_q, M * Hq * D * 2);
      outs[no++] = range_of(out_gate, M * Hq * D * 2);
      if (out_q8) outs[no++] = range_of(out_q8, M * Hq * D);
      if (out_qs) outs[no++] = range_of(out_qs, M * Hq * 4);
    }
    if (Hk > 0) {
      if (out_k) outs[no++] = range_of(out_k, M * Hk * D * 2);
      if (out_k8) outs[no++] = range_of(out_k8, M * Hk * D);
      if (out_ks) outs[no++] = range_of(out_ks, M * Hk * 4);
    }
    for (int i = 0; i < no; ++i) {
      if (overlap(outs[i], in)) return FN_ERR_INVALID;
      if (q_weight && overlap(outs[i], range_of(q_weight, D * 2))) return FN_ERR_INVALID;
      if (k_weight && overlap(outs[i], range_of(k_weight, D * 2))) return FN_ERR_INVALID;
      for (int j = i + 1; j < no; ++j)
        if (overlap(outs[i], outs[j])) return FN_ERR_INVALID;
    }
  }
  const int sms = sm_count();
  if (sms <= 0) return FN_ERR_CUDA;
  fn::QKParams p;
  std::memset(&p, 0, sizeof p);
  p.qkv = static_cast<const uint4*>(qkv);
  p.M = M;
  p.row_vec = row_stride / 8;
  p.Hq = Hq;
  p.Hk = Hk;
  p.dv = D / 8;
  p.qw = static_cast<const uint4*>(q_weight);
  p.kw = static_cast<const uint4*>(k_weight);
  p.eps = eps;
  p.inv_d = 1.0f / (float)D;
  p.out_q = static_cast<uint4*>(out_q);
  p.out_k = static_cast<uint4*>(out_k);
  p.out_g = static_cast<uint4*>(out_gate);
  p.out_q8 = static_cast<uint8_t*>(out_q8);
  p.out_qs = static_cast<float*>(out_qs);
  p.out_k8 = static_cast<uint8_t*>(out_k8);
  p.out_ks = static_cast<float*>(out_ks);
  // as a programmatic dependent, each warp prefetches its head before its
  // wait (never from another device's memory)
  if (tl_pdl) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FN_ERR_CUDA;
    p.prefetch_self = on_device(qkv, dev) && (!q_weight || on_device(q_weight, dev)) &&
                              (!k_weight || on_device(k_weight, dev))
                          ? 1
                          : 0;
  }
  const int64_t items = M * (Hq + Hk);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  const int nv = D / 8;
  if (fp8) {
    if (nv <= 32) rc = launch_qk_v<1, true>(p, items, sms, st);
    else if (nv <= 64) rc = launch_qk_v<2, true>(p, items, sms, st);
    else rc = launch_qk_v<4, true>(p, items, sms, st);
  } else {
    if (nv <= 32) rc = launch_qk_v<1, false>(p, items, sms, st);
    else if (nv <= 64) rc = launch_qk_v<2, false>(p, items, sms, st);
    else rc = launch_qk_v<4, false>(p, items, sms, st);
  }
  if (rc == FN_OK) tl_variant = fp8 ? FN_VARIANT_QK_WARP_FP8 : FN_VARIANT_QK_WARP;
  return rc;
}

// ---- hc_mix -------------------------------------------------------------------

// Weight rows of W_down per cluster: 4, or fewer for small ranks, so that the
// (r / CW) clusters of 8 blocks still spread the weight over about 128 SMs.
int hc_rows_per_cluster(int r) { return r >= 64 ? 4 : r >= 32 ? 2 : 1; }

int hc_rows_bound(int64_t M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

int hc_check(const void* x, const void* w_down, const void* w_up, int64_t M, int hc, int64_t C,
             int r, const void* out) {
  if (M < 0 || hc < 1 || C <= 0 || r <= 0) return FN_ERR_INVALID;
  if (hc != fn::kHcStreams || M > fn::kHcMaxRows || C % 16 ||
      (int64_t)hc * C > fn::kHcMaxK || r % 8 || r > fn::kHcMaxRank)
    return FN_ERR_UNSUPPORTED;
  if (M == 0) return FN_OK;
  if (!x || !w_down || !w_up || !out) return FN_ERR_INVALID;
  if (!aligned(x, 16) || !aligned(w_down, 16) || !aligned(w_up, 16) || !aligned(out, 16))
    return FN_ERR_ALIGN;
  return FN_OK;
}

// Channels per block of the gate-and-mix kernel: the fewest, in steps of 4,
// that divide C and need no more blocks than SMs (C = 2560 on 148 SMs: 20,
// 128 blocks), else 16 (C % 16 == 0), with more blocks than SMs.
int hc_mix_channels(int64_t C, int sms) {
  for (int64_t cpb = std::max<int64_t>(4, (C + sms - 1) / sms + 3) / 4 * 4;
       cpb <= fn::kHcMaxMixChannels; cpb += 4)
    if (C % cpb == 0) return (int)cpb;
  return 16;
}

// Shared memory a launch of the gate-and-mix kernel `k` asks for so that no SM
// holds two of its blocks (more than half of an SM's shared memory, with the
// kernel's shared-memory carveout at its maximum); the attributes are set
// once per kernel and device (function attributes belong to a device's
// context) and cached, -1 if the runtime refuses.  Launched early as a programmatic dependent, the small
// gate blocks were otherwise packed up to five to an SM onto the SMs the first
// kernel left free (measured on B200 with per-block SM ids: 128 blocks on 28
// SMs at M = 4 and 8), multiplying their logit time.  The first kernel keeps
// the default carveout: setting it to the maximum there too was measured
// slightly slower at M >= 4 (5.07 -> 5.15 us at M = 4, 6.09 -> 6.16 at 16).
int hc_spread_blocks(fn::HCKernel k) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  const auto key = std::make_pair(reinterpret_cast<const void*>(k), dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int per_sm = 0, bytes = -1;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
          cudaSuccess &&
      cudaFuncGetAttributes(&fa, k) == cudaSuccess) {
    const int want = per_sm / 2 + 1 - (int)fa.sharedSizeBytes;
    if (cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100) ==
            cudaSuccess &&
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, want) == cudaSuccess)
      bytes = want;
  }
  if (bytes < 0) (void)cudaGetLastError();
  cache[key] = bytes;
  return bytes;
}

// Launches the two hc_mix kernels with t in `ws` (fp32 [M, r], checked by the
// caller): the column-split product t = W_down x, then the gate and mix as its
// programmatic dependent.
int hc_launch(const void* x, const void* w_down, const void* w_up, int64_t M, int64_t C, int r,
              void* out, float* ws, void* stream) {
  fn::HCParams p;
  std::memset(&p, 0, sizeof p);
  p.x = static_cast<const uint4*>(x);
  p.w_down = static_cast<const uint4*>(w_down);
  p.w_up = static_cast<const uint4*>(w_up);
  p.t = ws;
  p.out = static_cast<uint16_t*>(out);
  p.M = (int)M;
  p.C = (int)C;
  p.K = (int)(fn::kHcStreams * C);
  p.r = r;
  // the first kernel's prologue prefetch (only as a programmatic dependent,
  // and never from another device's memory)
  if (tl_pdl) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FN_ERR_CUDA;
    p.prefetch = on_device(x, dev) && on_device(w_down, dev) ? 1 : 0;
  }
  const int cw = hc_rows_per_cluster(r);
  fn::HCKernel k1 = fn::hc_down_pick(hc_rows_bound(M), cw);
  if (!k1) return FN_ERR_UNSUPPORTED;
  const int cvec = p.K / 8 / fn::kHcCluster;
  // row groups of 4 rows: one warp-aligned set of threads per row group
  const int t1 = round32(cvec) * std::max(1, hc_rows_bound(M) / 4);
  const unsigned g1 = (unsigned)(r / cw * fn::kHcCluster);
  const int sms = sm_count();
  if (sms <= 0) return FN_ERR_CUDA;
  p.cpb = hc_mix_channels(C, sms);
  if (p.cpb == 0) return FN_ERR_UNSUPPORTED;
  const unsigned g2 = (unsigned)(C / p.cpb);
  // one warp per 8 of the block's 4 * cpb W_up rows
  const int t2 = 32 * (fn::kHcStreams * p.cpb / 8);
  fn::HCKernel k2 = fn::hc_gate_mix_pick(r / 8);
  if (!k2) return FN_ERR_UNSUPPORTED;
  // one gate block per SM while the blocks fit the GPU at once
  const int smem2 = (int)g2 <= sms ? hc_spread_blocks(k2) : 0;
  if (smem2 < 0) return FN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_kernel(k1, g1, (unsigned)t1, 0, st, fn::kHcCluster, p) != FN_OK) return FN_ERR_CUDA;
  if (launch_kernel_pdl(k2, g2, (unsigned)t2, (size_t)smem2, st, 1, true, p) != FN_OK)
    return FN_ERR_CUDA;
  tl_variant = FN_VARIANT_HC_MIX;
  tl_launch[0] = (int32_t)g1;
  tl_launch[1] = t1;
  tl_launch[2] = (int32_t)g2;
  tl_launch[3] = t2;
  return FN_OK;
}

}  // namespace

extern "C" {

int fn_version(void) { return 100; }

int fn_last_variant(void) { return tl_variant; }

int fn_prefer_variant(int variant) {
  const int old = tl_prefer;
  tl_prefer = variant;
  return old;
}

int fn_programmatic_launch(int on) {
  const int old = tl_pdl;
  tl_pdl = on ? 1 : 0;
  return old;
}

void fn_last_launch(int32_t out[4]) {
  if (out) std::memcpy(out, tl_launch, sizeof tl_launch);
}

const char* fn_status_string(int status) {
  switch (status) {
    case FN_OK: return "ok";
    case FN_ERR_INVALID: return "invalid argument (null pointer, size, mode or overlap)";
    case FN_ERR_ALIGN: return "misaligned pointer or stride";
    case FN_ERR_UNSUPPORTED: return "shape outside the built kernels";
    case FN_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
  }
}

int fn_rmsnorm_quant(const void* const* x_parts, int num_parts, const void* residual,
                     const void* weight, float eps, int mode, int64_t M, int64_t H,
                     void* out_q, void* out_scale, void* out_residual, void* out_y,
                     void* stream) {
  tl_variant = FN_VARIANT_NONE;
  if (!x_parts || num_parts < 1 || num_parts > FN_MAX_PARTS) return FN_ERR_INVALID;
  ModeInfo mi;
  int rc = parse_mode(mode, &mi);
  if (rc != FN_OK) return rc;
  if ((rc = check_mode_shape(mi, M, H)) != FN_OK) return rc;
  if (!std::isfinite(eps) || eps < 0.f) return FN_ERR_INVALID;
  if (M == 0) return FN_OK;  // nothing to read or write: data pointers may be NULL
  if (!weight || !out_q || !out_scale) return FN_ERR_INVALID;
  if (residual && !out_residual) return FN_ERR_INVALID;
  for (int p = 0; p < num_parts; ++p) {
    if (!x_parts[p]) return FN_ERR_INVALID;  // (M > 0 here)
    if (!aligned(x_parts[p], 16)) return FN_ERR_ALIGN;
  }
  if (!aligned(weight, 16) || (residual && !aligned(residual, 16)) ||
      (out_residual && !aligned(out_residual, 16)) || (out_y && !aligned(out_y, 16)))
    return FN_ERR_ALIGN;
  if ((rc = check_outputs_align(mi, out_q, out_scale)) != FN_OK) return rc;

  const int64_t row_bytes = M * H * 2;
  Range outs[4];
  int no = 0;
  outs[no++] = range_of(out_q, code_bytes(mi, M, H));
  outs[no++] = range_of(out_scale, scale_bytes(mi, M, H));
  if (out_residual) outs[no++] = range_of(out_residual, row_bytes);
  if (out_y) outs[no++] = range_of(out_y, row_bytes);
  if (M > 0) {
    for (int i = 0; i < no; ++i)
      for (int j = i + 1; j < no; ++j)
        if (overlap(outs[i], outs[j])) return FN_ERR_INVALID;
    Range ins[FN_MAX_PARTS + 2];
    int ni = 0;
    for (int p = 0; p < num_parts; ++p) ins[ni++] = range_of(x_parts[p], row_bytes);
    ins[ni++] = range_of(weight, H * 2);
    const Range res_in = residual ? range_of(residual, row_bytes) : Range{0, 0};
    for (int i = 0; i < no; ++i) {
      for (int j = 0; j < ni; ++j)
        if (overlap(outs[i], ins[j])) return FN_ERR_INVALID;
      if (residual && overlap(outs[i], res_in) &&
          !(out_residual == residual && i == 2))
        return FN_ERR_INVALID;
    }
  }
  if (M == 0) return FN_OK;

  fn::RQParams prm;
  std::memset(&prm, 0, sizeof prm);
  for (int p = 0; p < num_parts; ++p) prm.parts[p] = static_cast<const uint4*>(x_parts[p]);
  prm.residual = static_cast<const uint4*>(residual);
  prm.weight = static_cast<const uint4*>(weight);
  prm.out_residual = static_cast<uint4*>(out_residual);
  prm.out_y = static_cast<uint4*>(out_y);
  prm.out_q = static_cast<uint8_t*>(out_q);
  prm.out_scale = out_scale;
  prm.M = M;
  prm.nvec = (int)(H / 8);
  prm.P = num_parts;
  prm.eps = eps;
  prm.inv_h = 1.0f / (float)H;
  prm.scale_layout = mi.layout;
  prm.scale_ld = scale_ld(mi, M, H);
  return launch_rq(prm, mi.q, num_parts, M, true, mi.f16, stream, FN_VARIANT_ROW_CTA);
}

int fn_ar_rmsnorm_quant(const void* const* x_parts, int num_ranks, int rank, const void* residual,
                        const void* weight, float eps, int mode, int64_t M, int64_t H,
                        void* const* out_q, void* const* out_scale, void* const* out_residual,
                        void* const* out_y, void* stream) {
  tl_variant = FN_VARIANT_NONE;
  if (!x_parts || num_ranks < 2 || num_ranks > fn::kMaxRanks || rank < 0 || rank >= num_ranks)
    return FN_ERR_INVALID;
  ModeInfo mi;
  int rc = parse_mode(mode, &mi);
  if (rc != FN_OK) return rc;
  if (mi.f16) return FN_ERR_UNSUPPORTED;  // bf16 rows only
  if ((rc = check_mode_shape(mi, M, H)) != FN_OK) return rc;
  if (!std::isfinite(eps) || eps < 0.f) return FN_ERR_INVALID;
  const int64_t row0 = M * rank / num_ranks, row1 = M * (rank + 1) / num_ranks;
  if (row1 == row0) return FN_OK;  // an empty shard: nothing to read or write
  if (!weight || !out_q || !out_scale || (residual && !out_residual)) return FN_ERR_INVALID;
  const int n = num_ranks;
  for (int d = 0; d < n; ++d) {
    if (!x_parts[d] || !out_q[d] || !out_scale[d]) return FN_ERR_INVALID;
    if ((out_residual && !out_residual[d]) || (out_y && !out_y[d])) return FN_ERR_INVALID;
    if (!aligned(x_parts[d], 16) || (out_residual && !aligned(out_residual[d], 16)) ||
        (out_y && !aligned(out_y[d], 16)))
      return FN_ERR_ALIGN;
    if ((rc = check_outputs_align(mi, out_q[d], out_scale[d])) != FN_OK) return rc;
  }
  if (!aligned(weight, 16) || (residual && !aligned(residual, 16))) return FN_ERR_ALIGN;

  // Outputs (every rank's) must not overlap one another or any input; the one
  // exception is this rank's residual_out on its own residual (in place).
  const int64_t row_bytes = M * H * 2;
  Range outs[4 * fn::kMaxRanks];
  int own_res = -1, no = 0;
  for (int d = 0; d < n; ++d) {
    outs[no++] = range_of(out_q[d], code_bytes(mi, M, H));
    outs[no++] = range_of(out_scale[d], scale_bytes(mi, M, H));
    if (out_residual) {
      if (d == rank) own_res = no;
      outs[no++] = range_of(out_residual[d], row_bytes);
    }
    if (out_y) outs[no++] = range_of(out_y[d], row_bytes);
  }
  Range ins[fn::kMaxRanks + 1];
  int ni = 0;
  for (int d = 0; d < n; ++d) ins[ni++] = range_of(x_parts[d], row_bytes);
  ins[ni++] = range_of(weight, H * 2);
  const Range res_in = residual ? range_of(residual, row_bytes) : Range{0, 0};
  for (int i = 0; i < no; ++i) {
    for (int j = i + 1; j < no; ++j)
      if (overlap(outs[i], outs[j])) return FN_ERR_INVALID;
    for (int j = 0; j < ni; ++j)
      if (overlap(outs[i], ins[j])) return FN_ERR_INVALID;
    if (residual && overlap(outs[i], res_in) && !(i == own_res && out_residual[rank] == residual))
      return FN_ERR_INVALID;
  }

  const int sms = sm_count();
  if (sms <= 0) return FN_ERR_CUDA;
  fn::ARParams ap;
  std::memset(&ap, 0, sizeof ap);
  fn::RQParams& prm = ap.rq;
  for (int d = 0; d < n; ++d) prm.parts[d] = static_cast<const uint4*>(x_parts[d]);
  prm.residual = static_cast<const uint4*>(residual);
  prm.weight = static_cast<const uint4*>(weight);
  prm.M = M;
  prm.nvec = (int)(H / 8);
  prm.seg = prm.nvec;
  prm.P = n;
  prm.eps = eps;
  prm.inv_h = 1.0f / (float)H;
  prm.scale_layout = mi.layout;
  prm.scale_ld = scale_ld(mi, M, H);
  ap.row0 = row0;
  ap.ndst = n;
  for (int d = 0; d < n; ++d) {
    ap.out_q[d] = static_cast<uint8_t*>(out_q[d]);
    ap.out_scale[d] = out_scale[d];
    ap.out_residual[d] = out_residual ? static_cast<uint4*>(out_residual[d]) : nullptr;
    ap.out_y[d] = out_y ? static_cast<uint4*>(out_y[d]) : nullptr;
  }
  const int V = vectors_per_thread(prm.nvec, 256, 8);
  const int threads = round32((prm.nvec + V - 1) / V);
  if (threads > 256) return FN_ERR_UNSUPPORTED;
  const int maxp = n == 2 ? 2 : n <= 4 ? 4 : 8;
  fn::RQArKernel k = mi.q == FN_FP8_PER_TOKEN      ? fn::rq_ar_pick_0(maxp, V)
                     : mi.q == FN_FP8_PER_GROUP128 ? fn::rq_ar_pick_1(maxp, V)
                                                   : fn::rq_ar_pick_2(maxp, V);
  if (!k) return FN_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_kernel(k, (unsigned)(row1 - row0), (unsigned)threads, 0, st, 1, ap) != FN_OK)
    return FN_ERR_CUDA;
  tl_variant = FN_VARIANT_ROW_ALLREDUCE;
  tl_launch[0] = (int32_t)(row1 - row0);
  tl_launch[1] = threads;
  tl_launch[2] = 1;
  tl_launch[3] = V;
  return FN_OK;
}

int64_t fn_hc_mix_workspace_bytes(int64_t M, int r) {
  if (M < 0 || r <= 0) return -1;
  return M * r * (int64_t)sizeof(float);
}

int fn_hc_mix(const void* x, const void* w_down, const void* w_up, int64_t M, int hc, int64_t C,
              int r, void* out, void* workspace, void* stream) {
  tl_variant = FN_VARIANT_NONE;
  int rc = hc_check(x, w_down, w_up, M, hc, C, r, out);
  if (rc != FN_OK || M == 0) return rc;
  if (!workspace) return FN_ERR_INVALID;
  if (!aligned(workspace, 16)) return FN_ERR_ALIGN;
  const int64_t K = (int64_t)hc * C;
  const Range ins[3] = {range_of(x, M * K * 2), range_of(w_down, (int64_t)r * K * 2),
                        range_of(w_up, K * r * 2)};
  const Range o = range_of(out, M * C * 2), ws = range_of(workspace, M * r * 4);
  if (overlap(o, ws)) return FN_ERR_INVALID;
  for (const Range& in : ins)
    if (overlap(o, in) || overlap(ws, in)) return FN_ERR_INVALID;
  return hc_launch(x, w_down, w_up, M, C, r, out, static_cast<float*>(workspace), stream);
}

}  // extern "C"

// ---- hc_mix without a caller-provided workspace ------------------------------------

// The intermediate t of fn_hc_mix_noalloc: fp32 [M, r] for at most 16 rows at
// rank 128, 8 KB.  A file-scope device array, so it exists on every device
// that loads the library, from load until exit, and no call allocates it.  In
// host code this name is only a stand-in for the array: its device address
// comes from cudaGetSymbolAddress, once per device (hc_noalloc_scratch).
static __device__ __align__(256) float g_hc_noalloc_t[fn::kHcMaxRows * fn::kHcMaxRank];

namespace {

constexpr int64_t kHcNoallocFloats = (int64_t)fn::kHcMaxRows * fn::kHcMaxRank;

std::mutex g_hc_noalloc_mu;
float* g_hc_noalloc_ptr[64];  // device address of g_hc_noalloc_t, per device ordinal

// The device address of the scratch array on the current device, looked up on
// the first call with that device current and cached; nullptr if the runtime
// cannot tell (the call then returns FN_ERR_CUDA).
float* hc_noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_hc_noalloc_mu);
  if (!g_hc_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_hc_noalloc_t) != cudaSuccess || ptr == nullptr) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_hc_noalloc_ptr[dev] = static_cast<float*>(ptr);
  }
  return g_hc_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

int fn_hc_mix_noalloc(const void* x, const void* w_down, const void* w_up, int64_t M, int hc,
                      int64_t C, int r, void* out, void* stream) {
  tl_variant = FN_VARIANT_NONE;
  int rc = hc_check(x, w_down, w_up, M, hc, C, r, out);
  if (rc != FN_OK || M == 0) return rc;
  if (M * (int64_t)r > kHcNoallocFloats) return FN_ERR_UNSUPPORTED;  // beyond the static scratch
  const int64_t K = (int64_t)hc * C;
  const Range ins[3] = {range_of(x, M * K * 2), range_of(w_down, (int64_t)r * K * 2),
                        range_of(w_up, K * r * 2)};
  const Range o = range_of(out, M * C * 2);
  for (const Range& in : ins)
    if (overlap(o, in)) return FN_ERR_INVALID;
  float* scratch = hc_noalloc_scratch();
  if (!scratch) return FN_ERR_CUDA;
  return hc_launch(x, w_down, w_up, M, C, r, out, scratch, stream);
}

int fn_quant(const void* y, int mode, int64_t M, int64_t H, void* out_q, void* out_scale,
             void* stream) {
  tl_variant = FN_VARIANT_NONE;
  ModeInfo mi;
  int rc = parse_mode(mode, &mi);
  if (rc != FN_OK) return rc;
  if ((rc = check_mode_shape(mi, M, H)) != FN_OK) return rc;
  if (M == 0) return FN_OK;
  if (!y || !out_q || !out_scale) return FN_ERR_INVALID;
  if (!aligned(y, 16)) return FN_ERR_ALIGN;
  if ((rc = check_outputs_align(mi, out_q, out_scale)) != FN_OK) return rc;
  if (M > 0) {
    const Range in = range_of(y, M * H * 2);
    const Range q = range_of(out_q, code_bytes(mi, M, H));
    const Range s = range_of(out_scale, scale_bytes(mi, M, H));
    if (overlap(in, q) || overlap(in, s) || overlap(q, s)) return FN_ERR_INVALID;
  }
  if (M == 0) return FN_OK;
  fn::RQParams prm;
  std::memset(&prm, 0, sizeof prm);
  prm.parts[0] = static_cast<const uint4*>(y);
  prm.out_q = static_cast<uint8_t*>(out_q);
  prm.out_scale = out_scale;
  prm.M = M;
  prm.nvec = (int)(H / 8);
  prm.P = 1;
  prm.scale_layout = mi.layout;
  prm.scale_ld = scale_ld(mi, M, H);
  return launch_rq(prm, mi.q, 1, M, false, mi.f16, stream, FN_VARIANT_QUANT_ONLY);
}

int fn_qk_norm_gate(const void* qkv, int64_t M, int64_t row_stride, int Hq, int Hk, int D,
                    const void* q_weight, const void* k_weight, float eps, void* out_q,
                    void* out_k, void* out_gate, void* stream) {
  return qk_impl(qkv, M, row_stride, Hq, Hk, D, q_weight, k_weight, eps, out_q, out_k, out_gate,
                 nullptr, nullptr, nullptr, nullptr, stream);
}

int fn_qk_norm_gate_fp8(const void* qkv, int64_t M, int64_t row_stride, int Hq, int Hk, int D,
                        const void* q_weight, const void* k_weight, float eps, void* out_q8,
                        void* out_q_scale, void* out_k8, void* out_k_scale, void* out_gate,
                        void* out_q, void* out_k, void* stream) {
  tl_variant = FN_VARIANT_NONE;
  if (M > 0 && ((Hq > 0 && (!out_q8 || !out_q_scale)) || (Hk > 0 && (!out_k8 || !out_k_scale))))
    return FN_ERR_INVALID;
  return qk_impl(qkv, M, row_stride, Hq, Hk, D, q_weight, k_weight, eps, out_q, out_k, out_gate,
                 out_q8, out_q_scale, out_k8, out_k_scale, stream);
}

}  // extern "C"
