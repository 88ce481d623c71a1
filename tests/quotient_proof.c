/*
 * Exhaustive check of the E4M3 quotient used by the FP8 kernels.
 *
 * The kernels need code = E4M3_rn_satfinite(RN(y / s)) for a bf16 element y of
 * a group whose bf16 amax gives the scale s = RN(amax / 448).  Instead of an
 * IEEE division per element they compute, from |y| and once per group
 *     r    = RN(1 / s)
 *     r_lo = RN(RN(1 - s r) * r)          (1 - s r by one fused multiply-add)
 *     q    = RN(|y| r + RN(|y| r_lo))      (one multiply, one fused multiply-add)
 * (a negative y gives minus the same quotient: every step rounds to nearest
 * even, which is odd-symmetric).  This program runs every positive finite
 * bf16 amax with s >= 2^-120 against every bf16 |y| <= amax (about 5.3e8
 * pairs) and counts the pairs whose E4M3 codes differ.  It exits 0 iff there
 * are none.  argv[1] (optional) strides the amax loop for a quicker run;
 * argv[2] = "fp16" runs the same check over IEEE binary16 amax and y (every
 * positive finite binary16 amax, whose scale is always above 2^-120, against
 * every binary16 |y| <= amax: about 5.0e8 pairs).
 *
 * Build: cc -O2 -ffp-contract=off -o quotient_proof quotient_proof.c -lm
 * (fmaf must be the correctly rounded fused multiply-add: glibc's is.)
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bf16(uint32_t b)
{
    uint32_t u = b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float from_fp16(uint32_t b)
{
    int e = (int)(b >> 10) & 0x1F, m = (int)(b & 0x3FF);
    return e == 0 ? (float)ldexp((double)m, -24) : (float)ldexp(1024.0 + m, e - 25);
}

/* E4M3 ("fn") code of a non-negative float: nearest even on the grid with 3
 * mantissa bits and minimum normal exponent -6, saturating at 448. */
static int e4m3_code(float v)
{
    double a = (double)v;
    if (a == 0.0)
        return 0;
    int e;
    (void)frexp(a, &e);
    int ex = e - 1 < -6 ? -6 : e - 1;
    double quantum = ldexp(1.0, ex - 3);
    double r = nearbyint(a / quantum) * quantum;
    if (r > 448.0)
        r = 448.0;
    if (r == 0.0)
        return 0;
    (void)frexp(r, &e);
    ex = e - 1;
    if (ex < -6)
        return (int)(r / ldexp(1.0, -9));
    return ((ex + 7) << 3) | (int)((r / ldexp(1.0, ex) - 1.0) * 8.0);
}

/* The kernels' scale: RN(amax / 448) without a division, by the FMA
 * correction of a product with the rounded reciprocal (Markstein's method):
 * q0 = RN(amax c) with c = RN(1/448), rem = amax - 448 q0 (exact in one FMA),
 * s = RN(q0 + rem c). */
static float scale_fma(float amax)
{
    const float c = 1.0f / 448.0f;
    const float q0 = amax * c;
    const float rem = fmaf(-448.0f, q0, amax);
    return fmaf(rem, c, q0);
}

int main(int argc, char** argv)
{
    uint32_t stride = argc > 1 ? (uint32_t)strtoul(argv[1], NULL, 10) : 1u;
    if (stride == 0)
        stride = 1;
    const int fp16 = argc > 2 && strcmp(argv[2], "fp16") == 0;
    /* "near": every r within one ulp of RN(1/s), not only RN(1/s) itself */
    const int near = argc > 3 && strcmp(argv[3], "near") == 0;
    float (*from_bits)(uint32_t) = fp16 ? from_fp16 : from_bf16;
    const uint32_t end = fp16 ? 0x7C00u : 0x7F80u; /* first non-finite pattern */
    long pairs = 0, bad = 0, scales = 0, bad_scales = 0;
    for (uint32_t ab = 1; ab < end; ++ab) { /* the scale formula, every amax */
        const float amax = from_bits(ab);
        if (scale_fma(amax) != amax / 448.0f) {
            if (bad_scales < 10)
                printf("scale mismatch: amax=%a fma=%a div=%a\n", amax, scale_fma(amax),
                       amax / 448.0f);
            ++bad_scales;
        }
        ++scales;
    }
    for (uint32_t ab = 1; ab < end; ab += stride) {
        const float amax = from_bits(ab);
        const float s = amax / 448.0f;
        if (!(s >= 0x1p-120f))
            continue;
        const float r_rn = 1.0f / s;
        const float cand[3] = {nextafterf(r_rn, 0.0f), r_rn, nextafterf(r_rn, INFINITY)};
        for (int c = near ? 0 : 1; c < (near ? 3 : 2); ++c) {
            const float r = cand[c];
            const float r_lo = fmaf(-s, r, 1.0f) * r;
            for (uint32_t yb = 0; yb <= ab; ++yb) {
                const float y = from_bits(yb);
                const float q = fmaf(y, r, y * r_lo);
                if (e4m3_code(q) != e4m3_code(y / s)) {
                    if (bad < 10)
                        printf("mismatch: amax=%a y=%a r=%a q=%a y/s=%a\n", amax, y, r, q, y / s);
                    ++bad;
                }
                ++pairs;
            }
        }
    }
    printf("scales %ld scale mismatches %ld\n", scales, bad_scales);
    printf("pairs %ld mismatches %ld\n", pairs, bad);
    return bad != 0 || bad_scales != 0;
}
