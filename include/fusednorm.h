/*
 * fusednorm.h — C ABI of the B200 (sm_100a) fused residual-add + RMSNorm +
 * activation-quantization library, libfusednorm.so.
 *
 * Sources (page title, then section):
 *  - sglang PR #29723, "Fused AllReduce + RMSNorm + per-token FP8 / MXFP4 quant
 *    on AMD (AITER)", "Modifications": the fused call returns the tuple
 *    (fp8_output, residual_out, per_token_scale) with the scale shaped (M, 1),
 *    or signals "cannot fuse" before any work; "Accuracy Tests": the fused
 *    kernel equals the unfused AllReduce -> RMSNorm -> quantize sequence.
 *    Review comments: a failure after collective entry must not turn into a
 *    silent per-rank fallback; the carried output dtype must not be lost.
 *  - sgl-amd-mono PR #26, "Whole-layer monokernels for Muse Spark", commit
 *    notes: online MXFP4 quantization of the bf16 normed row, bit-exact
 *    against the stand-alone quantization of that row.
 *  - sglang PR #27656, "Fuse QK RMSNorm + gate extraction Triton kernel for
 *    Qwen3.5 on HIP", "Motivation"/"Modifications": one kernel reads q and gate
 *    from the interleaved [q_h0, gate_h0, q_h1, gate_h1, ...] projection output
 *    with strides, applies GemmaRMSNorm to q and k, and writes contiguous q, k
 *    and gate.
 *  - OCP Microscaling (MX) v1.0: MXFP4 = E2M1 elements, one E8M0 scale per
 *    32-element block, X = 2^(floor(log2 amax) - 2).
 *
 * The cross-GPU all-reduce in front of the norm is replaced by an in-kernel
 * sum of up to 8 partial buffers that live on the same device
 * (fn_rmsnorm_quant), or done by the kernel itself over peer memory across
 * the ranks of a tensor-parallel group (fn_ar_rmsnorm_quant).
 *
 * Conventions for every entry point:
 *  - bf16 tensors are IEEE bfloat16 bit patterns, row-major, contiguous rows
 *    (row stride H elements unless a stride argument says otherwise).
 *  - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *    allocates nothing and never synchronizes: work is queued on `stream` (a
 *    cudaStream_t passed as void*; NULL means the legacy default stream).
 *    Its only state: thread-local settings, a record of the last dispatch,
 *    and a cache of occupancy queries.
 *  - All argument checks run on the host before anything is launched; on any
 *    error nothing is launched and no output is touched.  M == 0 returns
 *    FN_OK and launches nothing once the sizes and the mode are valid; the
 *    data pointers are not examined then and may be NULL (an empty torch
 *    tensor has a NULL data pointer).
 *  - A launch that the CUDA runtime rejects returns FN_ERR_CUDA.
 *  - Calls are thread-safe.  No kernel waits on another thread block or on
 *    another kernel (beyond the launch ordering of the stream), so no kernel
 *    of the library has a device-side wait that could fail to end.
 */
#ifndef FUSEDNORM_H
#define FUSEDNORM_H

#include <stdint.h>

#if defined(__GNUC__)
#define FN_API __attribute__((visibility("default")))
#else
#define FN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Quantization of the normed row y (sglang PR #29723, "Modifications"). */
typedef enum {
    FN_FP8_PER_TOKEN = 0,    /* E4M3, one fp32 scale per row: scale [M]          */
    FN_FP8_PER_GROUP128 = 1, /* E4M3, one fp32 scale per 128 elements [M, H/128] */
    FN_MXFP4 = 2             /* E2M1 codes, one E8M0 byte per 32 elements [M, H/32] */
} fn_mode;

typedef enum {
    FN_OK = 0,
    FN_ERR_INVALID = -1,     /* null pointer, bad size, bad mode, forbidden overlap */
    FN_ERR_ALIGN = -2,       /* a pointer or stride breaks the alignment rule      */
    FN_ERR_UNSUPPORTED = -3, /* valid request outside the built shapes (e.g. H)    */
    FN_ERR_CUDA = -4         /* the CUDA runtime rejected the launch               */
} fn_status;

/* Which kernel the calling thread's last successful call launched. */
typedef enum {
    FN_VARIANT_NONE = 0,        /* nothing launched (M == 0 or an error)          */
    FN_VARIANT_ROW_CTA = 1,     /* one thread block per row                        */
    FN_VARIANT_ROW_CLUSTER = 2, /* a cluster of 2..8 blocks per row (small M, long rows) */
    FN_VARIANT_QUANT_ONLY = 3,  /* fn_quant                                        */
    FN_VARIANT_QK_WARP = 4,     /* fn_qk_norm_gate: one warp per (token, head)     */
    /* 5 is not used */
    FN_VARIANT_QK_WARP_FP8 = 6, /* fn_qk_norm_gate_fp8                             */
    FN_VARIANT_ROW_ALLREDUCE = 7, /* fn_ar_rmsnorm_quant: one block per row of the shard */
    FN_VARIANT_HC_MIX = 8        /* fn_hc_mix: column-split product, then gate and mix */
} fn_variant;

/* Scale-layout flags, OR-ed into `mode` (fn_rmsnorm_quant, fn_quant).  No
 * flag: scales row-major as listed below.  These lay the scales out for the
 * GEMM that consumes the quantized tuple (the pages' "pre-shuffled" scales for
 * the consumer, sglang PR #29723, "Modifications"; the layouts themselves are
 * this architecture's, not the pages'):
 *  FN_SCALE_SWIZZLE_32_4_4  (FN_MXFP4 only) E8M0 scales in the tiling that
 *      block-scaled matrix multiplies read on B200: the [M, H/32] scale
 *      matrix padded to [roundup(M,128), roundup(H/32,4)] and cut into
 *      128 x 4 tiles of 512 bytes, tiles in row-tile-major order; inside a
 *      tile, row r and group c sit at byte (r % 32) * 16 + (r / 32) * 4 + c.
 *      out_scale must hold roundup(M,128) * roundup(H/32,4) bytes; padding
 *      entries are not written.
 *  FN_SCALE_MN_MAJOR  (FN_FP8_PER_GROUP128 only) fp32 scales group-major:
 *      scale of row m, group g at out_scale[g * roundup(M,4) + m];
 *      out_scale must hold (H/128) * roundup(M,4) floats; padding not written. */
#define FN_MODE_MASK 0xFF
#define FN_SCALE_SWIZZLE_32_4_4 0x100
#define FN_SCALE_MN_MAJOR 0x200

/* Row-format flag, OR-ed into `mode` (fn_rmsnorm_quant, fn_quant): every
 * 16-bit tensor of the call (x_parts, residual, weight, out_residual, out_y;
 * y of fn_quant) is IEEE binary16 instead of bf16, and every "bf16_rn" in the
 * formulas below is the binary16 rounding (nearest even, subnormals kept,
 * overflow to infinity).  Codes and scales are unchanged.  This carries an
 * FP16 producer's dtype through the quantized tuple instead of promoting it to
 * BF16 (sglang PR #29723, review of the tuple path's output dtype). */
#define FN_IO_FP16 0x1000

#define FN_MAX_PARTS 8
#define FN_MAX_H 32768
#define FN_MAX_HEAD_DIM 1024

/*
 * Fused (partial sum) + residual add + RMSNorm + quantization over M rows of
 * H elements.  Per row, with every add in fp32:
 *     h  = bf16_rn( ((x_0 + x_1) + ... + x_{P-1}) + residual )
 *     residual_out = h
 *     y  = bf16_rn( h * rsqrt(mean(h^2) + eps) * weight )
 *     (out_q, out_scale) = quantize(y, mode)
 *   FP8 modes:  scale = amax / 448 (fp32 division; 1.0 when amax == 0),
 *               code  = E4M3 round-to-nearest-even, saturating, of y / scale.
 *   MXFP4:      per 32-element block e = floor(log2 amax) - 2 clamped to
 *               [-127, 127], scale byte = e + 127 (0 for an all-zero block),
 *               code = E2M1 round-to-nearest-even, saturating to 6, of
 *               y * 2^-e; element 2i in the low nibble of byte i.
 *
 * x_parts      HOST array of num_parts DEVICE pointers, each bf16 [M, H].
 * num_parts    P, 1..FN_MAX_PARTS.
 * residual     bf16 [M, H], or NULL (no residual add).
 * weight       bf16 [H].
 * eps          finite, >= 0.
 * mode         fn_mode, optionally OR-ed with one FN_SCALE_* layout flag and
 *              with FN_IO_FP16 (every "bf16" tensor here is then binary16).
 * M, H         M >= 0; H % 8 == 0, 8 <= H <= FN_MAX_H; H % 128 == 0 for
 *              FN_FP8_PER_GROUP128, H % 32 == 0 for FN_MXFP4.
 * out_q        FP8: u8 [M, H]; MXFP4: u8 [M, H/2].
 * out_scale    FN_FP8_PER_TOKEN: fp32 [M]; FN_FP8_PER_GROUP128: fp32 [M, H/128];
 *              FN_MXFP4: u8 E8M0 [M, H/32].  All row-major.
 * out_residual bf16 [M, H].  Required when residual != NULL and may then be
 *              the residual pointer itself (in-place update).  With residual
 *              == NULL it is optional and receives the partial sum h.
 * out_y        bf16 [M, H] normed row (the "emit bf16" side output), or NULL.
 * Alignment    every bf16 pointer 16 bytes; out_q 8 bytes; out_scale 4 bytes
 *              for fp32 scales.  Otherwise FN_ERR_ALIGN.
 * Overlap      outputs must not overlap each other or any input, except
 *              out_residual == residual exactly.  Otherwise FN_ERR_INVALID.
 */
FN_API int fn_rmsnorm_quant(const void* const* x_parts, int num_parts, const void* residual,
                     const void* weight, float eps, int mode, int64_t M, int64_t H,
                     void* out_q, void* out_scale, void* out_residual, void* out_y,
                     void* stream);

/*
 * Fused all-reduce + residual add + RMSNorm + quantization across the
 * num_ranks ranks of a tensor-parallel group (sglang PR #29723, "Motivation"
 * and "Modifications": the AllReduce -> RMSNorm -> quantize sequence in one
 * kernel), two-stage form, one call per rank.  Rank `rank` computes the rows
 * [M*rank/num_ranks, M*(rank+1)/num_ranks) exactly as fn_rmsnorm_quant with
 * P = num_ranks partials would (partials summed in rank order, then the
 * residual), reading each row from every rank's partial buffer, and writes the
 * results into every rank's output buffers: the reduce-scatter and the
 * all-gather of the tuple are the kernel's own peer loads and stores.  After
 * all ranks' calls every rank holds the same outputs for all M rows.
 * (The one-stage form — each rank computes all rows from all partials and
 * writes only its own outputs — is fn_rmsnorm_quant given the peer partials.)
 *
 * x_parts      HOST array of num_ranks pointers: rank p's partial bf16 [M, H]
 *              (this rank's own, and peer-mapped memory of the others).
 * num_ranks    2..8.  rank: 0..num_ranks-1.
 * residual     this rank's residual replica bf16 [M, H], or NULL.
 * weight, eps, mode, M, H   as fn_rmsnorm_quant (FN_IO_FP16 is not
 *              supported here: FN_ERR_UNSUPPORTED).
 * out_q, out_scale   HOST arrays of num_ranks pointers: rank d's code and
 *              scale buffers for all M rows (layouts as fn_rmsnorm_quant).
 * out_residual HOST array of num_ranks pointers to every rank's residual_out
 *              [M, H] (required when residual != NULL; entry `rank` may be
 *              `residual` itself, in place), or NULL.
 * out_y        HOST array of num_ranks bf16 [M, H] pointers, or NULL.
 * Ordering     the caller orders the call between two group barriers: every
 *              rank's partial (and residual) complete before any rank's call
 *              starts, and every rank's call complete before any output is
 *              read.  The kernel itself never waits on another rank.
 * Errors       argument checks as fn_rmsnorm_quant, applied to every rank's
 *              pointers, all before launch; an empty shard returns FN_OK with
 *              nothing launched.  H above 16384 is FN_ERR_UNSUPPORTED here.
 */
FN_API int fn_ar_rmsnorm_quant(const void* const* x_parts, int num_ranks, int rank,
                               const void* residual, const void* weight, float eps, int mode,
                               int64_t M, int64_t H, void* const* out_q, void* const* out_scale,
                               void* const* out_residual, void* const* out_y, void* stream);

/*
 * The quantization step alone on existing bf16 (or, with FN_IO_FP16,
 * binary16) rows y [M, H] (the third
 * launch of the unfused AllReduce -> RMSNorm -> quantize sequence in sglang
 * PR #29723; the stand-alone row quantization the monokernel notes compare
 * against).  Same modes, layouts, alignment and overlap rules as
 * fn_rmsnorm_quant; runs the same device code as its quantization stage.
 */
FN_API int fn_quant(const void* y, int mode, int64_t M, int64_t H, void* out_q, void* out_scale,
             void* stream);

/*
 * QK Gemma-RMSNorm + gate extraction (sglang PR #27656, "Motivation").
 * Token m's row starts at qkv + m * row_stride (elements).  Within it, q head
 * h (h < Hq) is at [2hD, 2hD + D), its gate at [(2h+1)D, (2h+2)D), and k head
 * h (h < Hk) at [2 Hq D + hD, 2 Hq D + (h+1)D); what follows (v) is not read.
 *     out_q[m,h,:]    = bf16_rn( q * rsqrt(mean(q^2) + eps) * (1 + q_weight) )
 *     out_k[m,h,:]    = bf16_rn( k * rsqrt(mean(k^2) + eps) * (1 + k_weight) )
 *     out_gate[m,h,:] = gate (bit copy)
 * qkv          bf16, M rows of row_stride elements; 16-byte aligned.
 * row_stride   elements, multiple of 8, >= (2 Hq + Hk) D.
 * Hq, Hk       >= 0 (Hq + Hk >= 1).   D: multiple of 8, 8..FN_MAX_HEAD_DIM.
 * q_weight, k_weight   bf16 [D] (k_weight may be NULL when Hk == 0).
 * out_q [M,Hq,D], out_k [M,Hk,D], out_gate [M,Hq,D]: bf16, contiguous,
 *              16-byte aligned, no overlap with each other or with qkv.
 */
FN_API int fn_qk_norm_gate(const void* qkv, int64_t M, int64_t row_stride, int Hq, int Hk, int D,
                    const void* q_weight, const void* k_weight, float eps, void* out_q,
                    void* out_k, void* out_gate, void* stream);

/*
 * fn_qk_norm_gate with an FP8 epilogue for an FP8 attention consumer (the
 * pages' MXFP4-AttnFP8 serving runs attention in FP8; sglang PR #29723,
 * "Speed Tests").  Each normed q and k head (D values) is quantized with the
 * per-token rule of fn_rmsnorm_quant applied to the head vector: scale =
 * amax / 448 (fp32 division, 1.0 for an all-zero head), code = E4M3 of
 * y / scale, nearest even, saturating.
 * out_q8     u8 E4M3 [M, Hq, D], 8-byte aligned;  out_q_scale fp32 [M, Hq].
 * out_k8     u8 E4M3 [M, Hk, D], 8-byte aligned;  out_k_scale fp32 [M, Hk].
 * out_gate   bf16 [M, Hq, D] as in fn_qk_norm_gate.
 * out_q, out_k  the bf16 normed heads as in fn_qk_norm_gate, or NULL.
 * Other arguments, checks and errors as fn_qk_norm_gate.
 */
FN_API int fn_qk_norm_gate_fp8(const void* qkv, int64_t M, int64_t row_stride, int Hq, int Hk,
                               int D, const void* q_weight, const void* k_weight, float eps,
                               void* out_q8, void* out_q_scale, void* out_k8, void* out_k_scale,
                               void* out_gate, void* out_q, void* out_k, void* stream);

/*
 * hc_mix: the low-rank gate over the hyper-state (sglang PR #41880,
 * "Motivation": the input mix of GatedResidual, a low-rank gate over the
 * [M, 4*2560] hyper-state, decode-sized M <= 16, bound by reading the
 * weights; "Modifications": BF16, contiguous, 1 <= M <= 16, hc = 4).  The
 * page prints no formula; per row x of hc streams of C values (stream s at
 * columns [s*C, (s+1)*C)) this computes
 *     t    = W_down x                     (fp32, rank r)
 *     z    = W_up t
 *     u[c] = sum_s sigmoid(z[s*C + c]) * x[s*C + c],   sigmoid(z) = 1/(1+e^-z)
 *     out  = bf16_rn(u)                   [M, C]
 * in fp32 with one rounding to bf16; accuracy against the float64 definition:
 * |out - u| <= 4e-3 + 1e-2 |u| (the page's "Accuracy Tests").  Two kernels
 * run, the second launched as a programmatic dependent of the first.
 *
 * x          bf16 [M, hc*C], row-major, 16-byte aligned.
 * w_down     bf16 [r, hc*C] (a linear layer's weight layout: row j is the
 *            j-th down vector), 16-byte aligned.
 * w_up       bf16 [hc*C, r], 16-byte aligned.
 * M          0..16 (above: FN_ERR_UNSUPPORTED); M == 0 launches nothing.
 * hc         4 (other values: FN_ERR_UNSUPPORTED).
 * C          multiple of 16, hc*C <= 16384 (else FN_ERR_UNSUPPORTED).
 * r          multiple of 8, 8..128 (else FN_ERR_UNSUPPORTED).
 * out        bf16 [M, C], 16-byte aligned.
 * workspace  device memory of at least fn_hc_mix_workspace_bytes(M, r) bytes,
 *            16-byte aligned, owned by the caller; it receives t (fp32 [M, r])
 *            and may be reused as soon as the call's work on `stream` is done.
 * Overlap    out and workspace must not overlap each other or any input
 *            (FN_ERR_INVALID).
 * Device     the first kernel's blocks hand their partial sums to one block
 *            of their cluster, which waits for them with a bounded wait; if
 *            that wait ever ran out (not seen on working hardware) the
 *            affected entries of t, and so the outputs, are NaN.
 * fn_last_launch: out[0] blocks (clusters of 8) and out[1] threads of the
 * first kernel, out[2] blocks and out[3] threads of the second.
 */
FN_API int fn_hc_mix(const void* x, const void* w_down, const void* w_up, int64_t M, int hc,
                     int64_t C, int r, void* out, void* workspace, void* stream);

/* Bytes of workspace fn_hc_mix needs for M rows at rank r (M * r * 4), or -1
 * for a negative M or a non-positive r. */
FN_API int64_t fn_hc_mix_workspace_bytes(int64_t M, int r);

/*
 * fn_hc_mix for callers that cannot allocate device memory: the same
 * computation, kernels and results as fn_hc_mix, with the intermediate t kept
 * in a fixed scratch array inside the library instead of a caller-provided
 * workspace.  Some callers cannot call cudaMalloc or any allocator at the
 * point where they run this step: code inside a section that must not
 * allocate (a real-time or inference loop that has reserved all its memory up
 * front, a host callback, a plugin whose framework owns every allocation).
 * The pages have no counterpart; they describe no memory management.
 *
 * Arguments, checks and errors as fn_hc_mix, without `workspace`.
 * Scratch    a file-scope device array of the library holding t for at most
 *            16 rows at rank 128 (fp32 [M, r], M * r <= 2048: 8 KB); a larger
 *            M * r returns FN_ERR_UNSUPPORTED.  Every device that loads the
 *            library holds the array from load until the process exits; no
 *            call allocates or frees anything.
 * First call the first call on a device, with that device current, looks up
 *            the array's device address (cudaGetSymbolAddress) and caches it;
 *            make that first call before any stream capture.
 * Sharing    every call on a device uses the same array and finds there what
 *            the previous call left; each call writes all of t before reading
 *            it, so nothing needs clearing, but calls that overlap on the GPU
 *            (different streams, concurrent graphs) race on the array: order
 *            them on one stream.
 */
FN_API int fn_hc_mix_noalloc(const void* x, const void* w_down, const void* w_up, int64_t M,
                             int hc, int64_t C, int r, void* out, void* stream);

/* Static, NUL-terminated description of a status code. */
FN_API const char* fn_status_string(int status);

/* Thread-local launch mode for the calling thread's later calls (every entry
 * point): on != 0 launches each kernel as a programmatic dependent of the
 * work before it on its stream (CUDA programmatic dependent launch, sm_90
 * and later), so its blocks may be scheduled while the previous kernel
 * drains; every kernel of this library first waits, on the device, until the
 * grids it depends on have completed and their writes are visible, so results
 * are those of ordinary stream order.  Before that wait, decode-sized row
 * calls, the QK prologue and hc_mix's first kernel start their inputs
 * towards L2 (cp.async.bulk.prefetch.L2: a hint with no result, and only
 * for the current device's memory), so their loads after the wait find L2.
 * Works inside CUDA graph capture.  Default 0.  Returns the previous
 * setting.  (A launch-latency measure for decode-sized calls; the pages
 * describe no counterpart.) */
FN_API int fn_programmatic_launch(int on);

/* fn_variant of the calling thread's last call (FN_VARIANT_NONE after an error). */
FN_API int fn_last_variant(void);

/* Launch shape of the calling thread's last launch: out[0] grid blocks,
 * out[1] threads per block, out[2] blocks per cluster for
 * FN_VARIANT_ROW_CLUSTER, or, for one block per row (FN_VARIANT_ROW_CTA,
 * FN_VARIANT_QUANT_ONLY), the L2 prefetch: the distance in rows (large-M
 * launches start the rows about one wave ahead towards L2), -1 (launched as
 * programmatic dependents, every block starts its own row towards L2 before
 * it waits for the previous kernel) or 0 (none); either prefetch is taken
 * only when every row input (and, for -1, the weight) is device memory of
 * the current device: memory of another GPU or of the host is read with
 * plain loads alone.  out[3] 16-byte vectors per thread per tensor. */
FN_API void fn_last_launch(int32_t out[4]);

/* Thread-local kernel preference for fn_rmsnorm_quant: FN_VARIANT_NONE (the
 * default) lets the library choose by M, H and P; FN_VARIANT_ROW_CTA or
 * FN_VARIANT_ROW_CLUSTER asks for that kernel where the shape allows it (the
 * cluster kernel needs a row that splits into 2..8 group-aligned segments
 * with M * blocks <= SMs).  Every kernel meets the same accuracy contract;
 * kernels that reduce a row in another order (block size, cluster split) may
 * differ from one another by the one-ulp rounding of y it allows, while any
 * one kernel and launch shape always gives the same bits.  Returns the
 * previous preference. */
FN_API int fn_prefer_variant(int variant);

/* Library ABI version (major * 100 + minor). */
FN_API int fn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FUSEDNORM_H */
