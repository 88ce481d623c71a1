/*
 * Plain CPU oracle for the fused residual-add + RMSNorm + activation
 * quantization path and for the QK Gemma-RMSNorm + gate prologue.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU baseline of the
 * benchmark do.  It shares no code, header, table or constant generator with
 * the CUDA library: every format rule below is written out here from its
 * definition, single-threaded, in fp64 wherever the definition does not fix
 * the precision.
 *
 * Sources (page title, then section):
 *  [AR]   sglang PR #29723, "Fused AllReduce + RMSNorm + per-token FP8 /
 *         MXFP4 quant on AMD (AITER)": "Modifications" (the tuple
 *         (fp8_output, residual_out, per_token_scale), scale shaped (M,1)) and
 *         "Accuracy Tests" (the fused kernel equals the unfused
 *         AllReduce -> RMSNorm -> quantize sequence).
 *  [MONO] sgl-amd-mono PR #26, "Whole-layer monokernels for Muse Spark",
 *         commit notes: online MXFP4 quantization of activations; the xn task
 *         quantizes the bf16 normed row and is bit-exact against the
 *         stand-alone quantization of that row.
 *  [QK]   sglang PR #27656, "Fuse QK RMSNorm + gate extraction Triton kernel
 *         for Qwen3.5 on HIP": "Motivation" (interleaved
 *         [q_h0, gate_h0, q_h1, gate_h1, ...] layout, GemmaRMSNorm on q and k,
 *         contiguous q, k, gate outputs).
 *  [OCP]  OCP Microscaling (MX) v1.0: shared scale X = 2^(floor(log2 amax) -
 *         emax_elem), emax_elem = 2 for E2M1; E8M0 scale; E4M3 "fn" element
 *         format (max 448, no infinities).
 *  [HC]   sglang PR #41880, "AITER FlyDSL hc_mix for Qwen3.8 hyper-connections
 *         on gfx950": "Motivation" (the input mix of GatedResidual is a
 *         low-rank gate over the [M, 4*2560] hyper-state; decode-sized M <= 16,
 *         bound by reading the weights), "Modifications" (BF16, contiguous,
 *         1 <= M <= 16, hc = 4), "Accuracy Tests" (float64 reference,
 *         atol 4e-3, rtol 1e-2).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes under the same tag):
 *  A1  RMSNorm is h * 1/sqrt(mean(h^2) + eps) * w, mean over the row.
 *  A2  Gemma weight is (1 + w) formed in fp64, not rounded to bf16.
 *  A3  partials are summed in fp32 in order p = 0..P-1, then the residual is
 *      added in fp32, then ONE rounding to bf16 gives h (= residual_out);
 *      the norm reads the bf16 h.
 *  A4  y = bf16_rn(h * rstd * w): one rounding of the fp64 product.
 *  A5  FP8 is OCP E4M3 "fn" (max 448), round-to-nearest-even, saturating.
 *  A6  FP8 scale = fl32(amax / 448); code = e4m3(fl32(y / scale)) with a true
 *      fp32 division.
 *  A7  all-zero FP8 row/group: scale 1.0, codes 0.
 *  A8  all-zero MX block: scale code 0 (2^-127), codes 0.
 *  A9  element 2i in the low nibble of byte i; scales row-major.
 *  A11 a NaN or infinite MX block amax gives scale code 0xFF.
 *  A17 fp16 input/output ([AR] review: the producer's activation dtype is
 *      carried through the quantized tuple, FP16 beside BF16): with
 *      io = ORC_IO_FP16 every 16-bit tensor (partials, residual, weight,
 *      residual_out, y, the rows given to orc_quant_rows) is IEEE binary16
 *      instead of bf16, and every "bf16(...)" rounding above is a binary16
 *      rounding (nearest even, subnormals kept, overflow to infinity).
 *      Codes and scales are unchanged.
 *  A19 [HC] prints no formula.  Reading: the hyper-state row x holds hc
 *      streams of C values (stream s at [s*C, (s+1)*C)); the gate has the
 *      hyper-state's shape, its logits a rank-r linear map of the whole row,
 *      z = W_up (W_down x) with W_down [r, hc*C] and W_up [hc*C, r] (the two
 *      low-rank factors, each in the row layout of a linear layer's weight),
 *      g = logistic sigmoid(z) = 1 / (1 + exp(-z)), and the input mix is the
 *      gated sum of the streams, u[c] = sum_s g[s*C + c] * x[s*C + c], one
 *      value per channel: the sublayer's input [M, C].  No bias, no norm
 *      (the norm is a separate step before the mix).  Evaluated in fp64.
 *
 * Build: plain C99, -O2 -ffp-contract=off, no fast-math, x86-64 SSE float
 * arithmetic (FLT_EVAL_METHOD == 0), so `float` operations are IEEE binary32
 * with round-to-nearest-even.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs float arithmetic evaluated in binary32"
#endif

/* Mode numbers of the quantization step (the interface's values). */
#define ORC_FP8_PER_TOKEN 0
#define ORC_FP8_PER_GROUP128 1
#define ORC_MXFP4 2

#define ORC_OK 0
#define ORC_BAD -1

/* Storage format of the 16-bit tensors (A17). */
#define ORC_IO_BF16 0
#define ORC_IO_FP16 1

/* ------------------------------------------------------------------ */
/* Number formats                                                       */
/* ------------------------------------------------------------------ */

/* bf16 bit pattern -> its exact value (bf16 is the top half of binary32). */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Round a finite double to the nearest point of a binary floating-point grid
 * with `mbits` stored mantissa bits and minimum normal exponent `emin`
 * (subnormals below it, spacing 2^(emin - mbits)); ties go to the even
 * multiple of the spacing, i.e. the even mantissa.  The exponent range is
 * unbounded above: overflow is handled by the caller.
 */
static double round_to_grid(double v, int mbits, int emin)
{
    if (v == 0.0 || !isfinite(v))
        return v;
    int e2;
    (void)frexp(fabs(v), &e2);    /* |v| = m 2^e2, m in [0.5, 1) */
    int ex = e2 - 1;              /* floor(log2 |v|) */
    if (ex < emin)
        ex = emin;
    double quantum = ldexp(1.0, ex - mbits);
    double n = nearbyint(fabs(v) / quantum); /* exact quotient; ties-to-even */
    return copysign(n * quantum, v);
}

/* IEEE round-to-nearest-even of a double to bf16 (8 significant bits,
 * emin -126, overflow to infinity), returned as a bit pattern. */
uint16_t orc_bf16_from_double(double v)
{
    if (isnan(v))
        return (uint16_t)(signbit(v) ? 0xFFC0u : 0x7FC0u);
    double r = round_to_grid(v, 7, -126);
    float f;
    if (fabs(r) >= 0x1p128)
        f = signbit(r) ? -INFINITY : INFINITY;
    else
        f = (float)r; /* exact: r has <= 8 significant bits within binary32 range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits; exponent
 * field 0 holds zero and the subnormals m 2^-24; field 31 holds infinity
 * (m == 0) and NaN. */
double orc_fp16_to_double(uint16_t b)
{
    int s = b >> 15, e = (b >> 10) & 0x1F, m = b & 0x3FF;
    double mag;
    if (e == 31)
        mag = m ? NAN : INFINITY;
    else if (e == 0)
        mag = ldexp((double)m, -24);
    else
        mag = ldexp(1024.0 + m, e - 25);
    return s ? -mag : mag;
}

/* IEEE round-to-nearest-even of a double to binary16 (11 significant bits,
 * emin -14, subnormals kept); magnitudes that round beyond the largest
 * finite value 65504 become infinity. */
uint16_t orc_fp16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    if (isnan(v))
        return (uint16_t)(sign | 0x7E00u);
    double r = fabs(round_to_grid(v, 10, -14));
    if (r >= 65536.0)
        return (uint16_t)(sign | 0x7C00u);
    if (r == 0.0)
        return sign;
    int e2;
    (void)frexp(r, &e2);
    int ex = e2 - 1;
    if (ex < -14) /* subnormal: r = m 2^-24 */
        return (uint16_t)(sign | (uint16_t)(r / 0x1p-24));
    int m = (int)((r / ldexp(1.0, ex) - 1.0) * 1024.0);
    return (uint16_t)(sign | ((ex + 15) << 10) | m);
}

/* The value of a stored 16-bit element, and the rounding of a value to the
 * storage format. */
static double elem_to_double(int io, uint16_t b)
{
    return io == ORC_IO_FP16 ? orc_fp16_to_double(b) : orc_bf16_to_double(b);
}

static float elem_to_float(int io, uint16_t b)
{
    return (float)elem_to_double(io, b); /* exact: both formats fit binary32 */
}

static uint16_t elem_from_double(int io, double v)
{
    return io == ORC_IO_FP16 ? orc_fp16_from_double(v) : orc_bf16_from_double(v);
}

/* OCP E4M3 "fn": 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinity;
 * S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448; smallest subnormal 2^-9. */
double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round to E4M3 with round-to-nearest-even and saturation to +-448
 * ("satfinite"); NaN gives 0x7F. */
uint8_t orc_e4m3_encode(double v)
{
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double r = fabs(round_to_grid(v, 3, -6));
    if (r > 448.0)
        r = 448.0;
    if (r == 0.0)
        return sign;
    int e2;
    (void)frexp(r, &e2);
    int ex = e2 - 1;
    if (ex < -6) /* subnormal: r = m * 2^-9 */
        return (uint8_t)(sign | (uint8_t)(r / 0x1p-9));
    int m = (int)((r / ldexp(1.0, ex) - 1.0) * 8.0);
    return (uint8_t)(sign | ((ex + 7) << 3) | m);
}

/* OCP E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no NaN, no infinity. */
double orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Round to E2M1, nearest-even, saturating to +-6; the sign is kept, so a
 * negative value that rounds to zero gives -0 (code 0x8). */
uint8_t orc_e2m1_encode(double v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double r = fabs(round_to_grid(v, 1, 0));
    if (r > 6.0)
        r = 6.0;
    if (r == 0.0)
        return sign;
    int e2;
    (void)frexp(r, &e2);
    int ex = e2 - 1;
    if (ex < 0) /* subnormal: only 0.5 */
        return (uint8_t)(sign | 0x1);
    int m = (int)((r / ldexp(1.0, ex) - 1.0) * 2.0);
    return (uint8_t)(sign | ((ex + 1) << 1) | m);
}

/* [OCP] shared exponent of an MX block: e = floor(log2(amax)) - 2 (2 is the
 * largest exponent of E2M1), clamped to the E8M0 range [-127, 127].
 * Returns the E8M0 code e + 127; amax == 0 gives code 0 (A8); a NaN or
 * infinite amax gives 0xFF (A11). */
uint8_t orc_mx_scale_code(double amax)
{
    if (!isfinite(amax))
        return 0xFF;
    if (amax == 0.0)
        return 0x00;
    int e2;
    (void)frexp(amax, &e2);
    int e = (e2 - 1) - 2;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return (uint8_t)(e + 127);
}

/* ------------------------------------------------------------------ */
/* Quantization of bf16 rows ([AR] "Modifications", [MONO] bit-exact    */
/* quantization of the bf16 row, [OCP])                                 */
/* ------------------------------------------------------------------ */

/* FP8 E4M3 of one group of n 16-bit values with one fp32 scale (A5-A7). */
static void quant_fp8_group(const uint16_t* y, int64_t n, uint8_t* q, float* scale_out, int io)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < n; ++j) {
        float a = fabsf(elem_to_float(io, y[j]));
        if (a > amax)
            amax = a;
    }
    float scale = (amax == 0.0f) ? 1.0f : amax / 448.0f; /* one binary32 division */
    for (int64_t j = 0; j < n; ++j) {
        float t = elem_to_float(io, y[j]) / scale;        /* one binary32 division */
        q[j] = orc_e4m3_encode((double)t);
    }
    *scale_out = scale;
}

/* MXFP4 of one 32-element block: E8M0 scale code, then E2M1 codes of
 * y_j * 2^-e, packed two per byte, element 2i in the low nibble (A9). */
static void quant_mx_block(const uint16_t* y, uint8_t* packed, uint8_t* scale_code, int io)
{
    double amax = 0.0;
    int any_nan = 0;
    for (int j = 0; j < 32; ++j) {
        double a = fabs(elem_to_double(io, y[j]));
        if (isnan(a))
            any_nan = 1;
        else if (a > amax)
            amax = a;
    }
    if (any_nan)
        amax = NAN;
    uint8_t sc = orc_mx_scale_code(amax);
    int e = (int)sc - 127;
    for (int i = 0; i < 16; ++i) {
        double v0 = ldexp(elem_to_double(io, y[2 * i]), -e);     /* exact */
        double v1 = ldexp(elem_to_double(io, y[2 * i + 1]), -e); /* exact */
        uint8_t c0 = orc_e2m1_encode(v0), c1 = orc_e2m1_encode(v1);
        packed[i] = (uint8_t)(c0 | (c1 << 4));
    }
    *scale_code = sc;
}

/*
 * Quantize M rows of length H (bf16, or binary16 with io = ORC_IO_FP16).
 *   mode 0: out_q [M,H] E4M3, out_scale fp32 [M]
 *   mode 1: out_q [M,H] E4M3, out_scale fp32 [M, H/128] row-major
 *   mode 2: out_q [M,H/2] packed E2M1, out_scale u8 E8M0 [M, H/32] row-major
 */
int orc_quant_rows(const uint16_t* y, int mode, int64_t M, int64_t H,
                   uint8_t* out_q, void* out_scale, int io)
{
    if (M < 0 || H <= 0 || (io != ORC_IO_BF16 && io != ORC_IO_FP16))
        return ORC_BAD;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* yr = y + m * H;
        if (mode == ORC_FP8_PER_TOKEN) {
            quant_fp8_group(yr, H, out_q + m * H, (float*)out_scale + m, io);
        } else if (mode == ORC_FP8_PER_GROUP128) {
            if (H % 128)
                return ORC_BAD;
            for (int64_t g = 0; g < H / 128; ++g)
                quant_fp8_group(yr + g * 128, 128, out_q + m * H + g * 128,
                                (float*)out_scale + m * (H / 128) + g, io);
        } else if (mode == ORC_MXFP4) {
            if (H % 32)
                return ORC_BAD;
            for (int64_t b = 0; b < H / 32; ++b)
                quant_mx_block(yr + b * 32, out_q + m * (H / 2) + b * 16,
                               (uint8_t*)out_scale + m * (H / 32) + b, io);
        } else {
            return ORC_BAD;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* RMSNorm ([AR] "Accuracy Tests": the unfused sequence)                */
/* ------------------------------------------------------------------ */

/* rstd = 1/sqrt(mean(h^2) + eps) in fp64 over n 16-bit values (A1). */
double orc_rstd(const uint16_t* h, int64_t n, float eps, int io)
{
    double ss = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double v = elem_to_double(io, h[j]);
        ss += v * v;
    }
    return 1.0 / sqrt(ss / (double)n + (double)eps);
}

/*
 * The unfused reference sequence, row by row:
 *   h  = bf16( (((part_0 + part_1) + ...) + part_{P-1}) + residual )   fp32 adds (A3)
 *   residual_out = h
 *   y  = bf16( h * rstd * w )                                           fp64 (A1, A4)
 *   (q, scale) = quantize(y)                                            (A5-A9)
 * residual may be NULL (no residual add); out_residual and out_y may be NULL.
 * io = ORC_IO_FP16: every 16-bit tensor and rounding is binary16 (A17).
 */
int orc_rmsnorm_quant(const uint16_t* const* parts, int P, const uint16_t* residual,
                      const uint16_t* weight, float eps, int mode, int64_t M, int64_t H,
                      uint8_t* out_q, void* out_scale, uint16_t* out_residual,
                      uint16_t* out_y, int io)
{
    if (P < 1 || P > 8 || M < 0 || H <= 0 || !parts || !weight)
        return ORC_BAD;
    if (io != ORC_IO_BF16 && io != ORC_IO_FP16)
        return ORC_BAD;
    if (mode == ORC_FP8_PER_GROUP128 && H % 128)
        return ORC_BAD;
    if (mode == ORC_MXFP4 && H % 32)
        return ORC_BAD;
    if (mode < 0 || mode > 2)
        return ORC_BAD;
    uint16_t* hbuf = (uint16_t*)malloc((size_t)H * sizeof(uint16_t));
    uint16_t* ybuf = (uint16_t*)malloc((size_t)H * sizeof(uint16_t));
    if (!hbuf || !ybuf) {
        free(hbuf);
        free(ybuf);
        return ORC_BAD;
    }
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < H; ++j) {
            float s = elem_to_float(io, parts[0][m * H + j]);
            for (int p = 1; p < P; ++p)
                s = s + elem_to_float(io, parts[p][m * H + j]);
            if (residual)
                s = s + elem_to_float(io, residual[m * H + j]);
            hbuf[j] = elem_from_double(io, (double)s);
        }
        double rstd = orc_rstd(hbuf, H, eps, io);
        for (int64_t j = 0; j < H; ++j)
            ybuf[j] = elem_from_double(io, elem_to_double(io, hbuf[j]) * rstd *
                                               elem_to_double(io, weight[j]));
        if (out_residual)
            memcpy(out_residual + m * H, hbuf, (size_t)H * sizeof(uint16_t));
        if (out_y)
            memcpy(out_y + m * H, ybuf, (size_t)H * sizeof(uint16_t));
        int rc;
        if (mode == ORC_FP8_PER_TOKEN)
            rc = orc_quant_rows(ybuf, mode, 1, H, out_q + m * H, (float*)out_scale + m, io);
        else if (mode == ORC_FP8_PER_GROUP128)
            rc = orc_quant_rows(ybuf, mode, 1, H, out_q + m * H,
                                (float*)out_scale + m * (H / 128), io);
        else
            rc = orc_quant_rows(ybuf, mode, 1, H, out_q + m * (H / 2),
                                (uint8_t*)out_scale + m * (H / 32), io);
        if (rc != ORC_OK) {
            free(hbuf);
            free(ybuf);
            return rc;
        }
    }
    free(hbuf);
    free(ybuf);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* QK Gemma-RMSNorm + gate ([QK] "Motivation", "Modifications")         */
/* ------------------------------------------------------------------ */

/* One head: y = bf16(x * rstd * (1 + w)) over D values (A1, A2, A4). */
static void gemma_norm_head(const uint16_t* x, const uint16_t* w, int D, float eps,
                            uint16_t* y)
{
    double rstd = orc_rstd(x, D, eps, ORC_IO_BF16);
    for (int d = 0; d < D; ++d)
        y[d] = orc_bf16_from_double(orc_bf16_to_double(x[d]) * rstd *
                                    (1.0 + orc_bf16_to_double(w[d])));
}

/*
 * Token m's row starts at qkv + m*row_stride (elements).  Head h < Hq of q
 * sits at [2hD, 2hD + D), its gate at [(2h+1)D, (2h+2)D); head h < Hk of k
 * sits at [2 Hq D + hD, 2 Hq D + (h+1)D).  Outputs are contiguous
 * q [M,Hq,D], k [M,Hk,D], gate [M,Hq,D]; the gate is a bit copy.
 */
int orc_qk_norm_gate(const uint16_t* qkv, int64_t M, int64_t row_stride, int Hq, int Hk,
                     int D, const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                     uint16_t* out_q, uint16_t* out_k, uint16_t* out_gate)
{
    if (M < 0 || Hq < 0 || Hk < 0 || D <= 0 ||
        row_stride < (int64_t)(2 * Hq + Hk) * D)
        return ORC_BAD;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = qkv + m * row_stride;
        for (int h = 0; h < Hq; ++h) {
            gemma_norm_head(row + (int64_t)2 * h * D, q_weight, D, eps,
                            out_q + (m * Hq + h) * D);
            memcpy(out_gate + (m * Hq + h) * D, row + (int64_t)(2 * h + 1) * D,
                   (size_t)D * sizeof(uint16_t));
        }
        for (int h = 0; h < Hk; ++h)
            gemma_norm_head(row + (int64_t)2 * Hq * D + (int64_t)h * D, k_weight, D, eps,
                            out_k + (m * Hk + h) * D);
    }
    return ORC_OK;
}

/*
 * The QK prologue with E4M3 q and k for an FP8 attention consumer (reading:
 * the per-token FP8 rule of [AR] applied to each normed head vector of D
 * values — scale = fl32(amax / 448), code = e4m3(fl32(y / scale)), scale 1
 * for an all-zero head).  q8 [M,Hq,D] with scales qs [M,Hq]; k8 [M,Hk,D]
 * with ks [M,Hk]; gate as orc_qk_norm_gate.  out_q / out_k may be NULL.
 */
int orc_qk_norm_gate_fp8(const uint16_t* qkv, int64_t M, int64_t row_stride, int Hq, int Hk,
                         int D, const uint16_t* q_weight, const uint16_t* k_weight, float eps,
                         uint8_t* q8, float* qs, uint8_t* k8, float* ks, uint16_t* out_gate,
                         uint16_t* out_q, uint16_t* out_k)
{
    if (M < 0 || Hq < 0 || Hk < 0 || D <= 0 || row_stride < (int64_t)(2 * Hq + Hk) * D)
        return ORC_BAD;
    uint16_t* y = (uint16_t*)malloc((size_t)D * sizeof(uint16_t));
    if (!y)
        return ORC_BAD;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = qkv + m * row_stride;
        for (int h = 0; h < Hq; ++h) {
            const int64_t o = m * Hq + h;
            gemma_norm_head(row + (int64_t)2 * h * D, q_weight, D, eps, y);
            quant_fp8_group(y, D, q8 + o * D, qs + o, ORC_IO_BF16);
            if (out_q)
                memcpy(out_q + o * D, y, (size_t)D * sizeof(uint16_t));
            memcpy(out_gate + o * D, row + (int64_t)(2 * h + 1) * D, (size_t)D * sizeof(uint16_t));
        }
        for (int h = 0; h < Hk; ++h) {
            const int64_t o = m * Hk + h;
            gemma_norm_head(row + (int64_t)2 * Hq * D + (int64_t)h * D, k_weight, D, eps, y);
            quant_fp8_group(y, D, k8 + o * D, ks + o, ORC_IO_BF16);
            if (out_k)
                memcpy(out_k + o * D, y, (size_t)D * sizeof(uint16_t));
        }
    }
    free(y);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* hc_mix: low-rank gate over the hyper-state ([HC], reading A19)       */
/* ------------------------------------------------------------------ */

/*
 * For each row m of x [M, hc*C] (bf16):
 *     t[j]  = sum_k x[k] * w_down[j, k]            j < r, k < hc*C
 *     z[e]  = sum_j t[j] * w_up[e, j]              e < hc*C
 *     g[e]  = 1 / (1 + exp(-z[e]))
 *     u[c]  = sum_s g[s*C + c] * x[s*C + c]        c < C
 * every sum in fp64, in index order.  out_u (fp64 [M, C]) receives u and
 * out_bf16 (bf16 [M, C]), if not NULL, bf16_rn(u).  w_down is bf16 [r, hc*C]
 * and w_up bf16 [hc*C, r], both row-major.
 */
int orc_hc_mix(const uint16_t* x, const uint16_t* w_down, const uint16_t* w_up, int64_t M,
               int hc, int64_t C, int r, double* out_u, uint16_t* out_bf16)
{
    if (M < 0 || hc < 1 || C < 1 || r < 1 || !x || !w_down || !w_up || !out_u)
        return ORC_BAD;
    const int64_t K = (int64_t)hc * C;
    double* t = (double*)malloc((size_t)r * sizeof(double));
    double* g = (double*)malloc((size_t)K * sizeof(double));
    if (!t || !g) {
        free(t);
        free(g);
        return ORC_BAD;
    }
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xr = x + m * K;
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += orc_bf16_to_double(xr[k]) * orc_bf16_to_double(w_down[(int64_t)j * K + k]);
            t[j] = acc;
        }
        for (int64_t e = 0; e < K; ++e) {
            double z = 0.0;
            for (int j = 0; j < r; ++j)
                z += t[j] * orc_bf16_to_double(w_up[e * r + j]);
            g[e] = 1.0 / (1.0 + exp(-z));
        }
        for (int64_t c = 0; c < C; ++c) {
            double u = 0.0;
            for (int s = 0; s < hc; ++s)
                u += g[(int64_t)s * C + c] * orc_bf16_to_double(xr[(int64_t)s * C + c]);
            out_u[m * C + c] = u;
            if (out_bf16)
                out_bf16[m * C + c] = orc_bf16_from_double(u);
        }
    }
    free(t);
    free(g);
    return ORC_OK;
}
