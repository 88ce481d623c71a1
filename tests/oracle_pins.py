"""Pins of the CPU oracle against things other than itself.

Each pin takes a loaded oracle library (`lib`) and raises AssertionError when
the oracle disagrees with: values printed by the format specifications
(tests/golden/), an independent brute-force or library computation (torch's
float8 conversion, exhaustive nearest-point search over a format's grid,
Python `decimal` at 60 digits), closed forms, or invariants.  The same pins
run against deliberately broken copies of the oracle in
test_oracle_mutations.py, where at least one of them must fail.
"""
import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# ----------------------------------------------------------------------------
# helpers that do not use the oracle
# ----------------------------------------------------------------------------


def all_finite_bf16():
    """All finite bf16 bit patterns and their values (float64)."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).astype(np.uint32).view(np.float32)
    keep = np.isfinite(f)
    return bits[keep].astype(np.uint16), f[keep].astype(np.float64)


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).astype(np.uint32).view(np.float32).astype(np.float64)


def f32_to_bf16_bits_torch(a):
    """binary32 -> bf16 round-to-nearest-even, by torch's own conversion."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                c, v = line.split()
                rows.append((int(c, 16), float(v)))
    return rows


def brute_encode(v, grid_vals, grid_codes, sign_bit):
    """Nearest point of a sign-magnitude grid by exhaustive search; ties go to
    the even code; beyond the largest point, the largest point (saturation)."""
    v = np.asarray(v, dtype=np.float64)
    # Any magnitude above the largest point has that point as its nearest;
    # clipping keeps the differences below exact in binary64.
    mag = np.minimum(np.abs(v), 2.0 * grid_vals.max())
    d = np.abs(mag[:, None] - grid_vals[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = (grid_codes[None, :] & 1) == 0
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    idx = np.where(has_even, pick_even.argmax(axis=1), cand.argmax(axis=1))
    codes = grid_codes[idx].astype(np.int64)
    codes = np.where(np.signbit(v), codes | sign_bit, codes)
    return codes.astype(np.uint8)


def e4m3_grid_torch():
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x00..0x7E: the positive finite points
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals, codes


def e2m1_grid_golden():
    t = read_table("ocp_e2m1.txt")
    codes = np.array([c for c, v in t if c < 8], dtype=np.uint8)
    vals = np.array([v for c, v in t if c < 8], dtype=np.float64)
    return vals, codes


def brute_mx_scale_code(amax):
    """The E8M0 code c with 4 * 2^(c-127) <= amax < 8 * 2^(c-127), found by
    comparing against exact powers of two; c = 0 when amax is below 2^-125."""
    if amax == 0:
        return 0
    for c in range(0, 255):
        lo, hi = 4.0 * 2.0 ** (c - 127), 8.0 * 2.0 ** (c - 127)
        if amax < hi and (amax >= lo or c == 0):
            return c
    raise AssertionError("no E8M0 code")


def nearest_bf16_decimal(x: Decimal) -> int:
    """bf16 bit pattern nearest to a high-precision value (ties to even)."""
    if x == 0:
        return 0x8000 if x.is_signed() else 0
    neg = x < 0
    ax = -x if neg else x
    f = np.float32(float(ax))
    base = int(np.array([f]).view(np.uint32)[0] >> 16)
    best = None
    for b in range(max(base - 2, 0), min(base + 3, 0x7F80)):
        val = Decimal(float(bf16_bits_to_f64([b])[0]))
        d = abs(val - ax)
        key = (d, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    b = best[1]
    return b | 0x8000 if neg else b


def decimal_rstd(h_vals, eps32):
    getcontext().prec = 60
    ss = sum(Decimal(float(v)) ** 2 for v in h_vals)
    ms = ss / Decimal(len(h_vals))
    return Decimal(1) / (ms + Decimal(float(eps32))).sqrt()


def ref_y_bits(h_vals, w_vals, eps, gemma=False):
    getcontext().prec = 60
    r = decimal_rstd(h_vals, np.float32(eps))
    out = []
    for h, w in zip(h_vals, w_vals):
        wd = Decimal(float(w))
        if gemma:
            wd = Decimal(1) + wd
        out.append(nearest_bf16_decimal(Decimal(float(h)) * r * wd))
    return np.array(out, dtype=np.uint16)


def ref_quant_fp8(y_bits, group, decode=None):
    """Library formulation: fp32 amax, fp32 amax/448, fp32 y/scale, torch's
    float8_e4m3fn conversion (nearest-even; never reached above 464 here).
    `decode` maps the stored bits to values (bf16 by default)."""
    y = (decode or bf16_bits_to_f64)(y_bits).astype(np.float32)
    M, H = y.shape
    codes = np.zeros((M, H), dtype=np.uint8)
    scales = np.zeros((M, H // group), dtype=np.float32)
    for m in range(M):
        for g in range(H // group):
            seg = y[m, g * group:(g + 1) * group]
            amax = np.float32(np.max(np.abs(seg)))
            scale = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(448.0))
            t = (seg / scale).astype(np.float32)
            c = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            codes[m, g * group:(g + 1) * group] = c
            scales[m, g] = scale
    return codes, scales


def ref_quant_mx(y_bits, decode=None):
    y = (decode or bf16_bits_to_f64)(y_bits)
    M, H = y.shape
    gv, gc = e2m1_grid_golden()
    packed = np.zeros((M, H // 2), dtype=np.uint8)
    sc = np.zeros((M, H // 32), dtype=np.uint8)
    for m in range(M):
        for b in range(H // 32):
            blk = y[m, b * 32:(b + 1) * 32]
            c = brute_mx_scale_code(float(np.max(np.abs(blk))))
            v = blk * 2.0 ** (-(c - 127))
            codes = brute_encode(v, gv, gc, 0x8)
            packed[m, b * 16:(b + 1) * 16] = codes[0::2] | (codes[1::2] << 4)
            sc[m, b] = c
    return packed, sc


def ref_residual_bits(parts_bits, res_bits):
    s = bf16_bits_to_f64(parts_bits[0]).astype(np.float32)
    for p in parts_bits[1:]:
        s = (s + bf16_bits_to_f64(p).astype(np.float32)).astype(np.float32)
    if res_bits is not None:
        s = (s + bf16_bits_to_f64(res_bits).astype(np.float32)).astype(np.float32)
    return f32_to_bf16_bits_torch(s)


def bf16_bits_from_torch(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------


def pin_e4m3_decode(lib):
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes, lib)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref)), "E4M3 NaN codes"
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok]), "E4M3 decode vs torch"
    assert np.array_equal(np.signbit(mine[ok]), np.signbit(ref[ok])), "E4M3 signed zero"
    for c, v in read_table("ocp_e4m3_points.txt"):
        got = lib.orc_e4m3_decode(c)
        if math.isnan(v):
            assert math.isnan(got), f"code {c:#x} must be NaN"
        else:
            assert got == v and math.copysign(1, got) == math.copysign(1, v), f"code {c:#x}"


def pin_e4m3_encode(lib):
    bits, vals = all_finite_bf16()
    mine = oracle.e4m3_encode(vals, lib)
    gv, gc = e4m3_grid_torch()
    brute = brute_encode(vals, gv, gc, 0x80)
    assert np.array_equal(mine, brute), "E4M3 encode vs exhaustive nearest-even search"
    inr = np.abs(vals) <= 464.0
    tq = torch.from_numpy(vals[inr].astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(mine[inr], tq.view(torch.uint8).numpy()), "E4M3 encode vs torch"
    assert lib.orc_e4m3_encode(1e30) == 0x7E and lib.orc_e4m3_encode(-1e30) == 0xFE
    assert lib.orc_e4m3_encode(float("nan")) == 0x7F
    # every finite code survives decode -> encode
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert lib.orc_e4m3_encode(lib.orc_e4m3_decode(c)) == c, f"round trip {c:#x}"


def pin_e2m1(lib):
    for c, v in read_table("ocp_e2m1.txt"):
        got = lib.orc_e2m1_decode(c)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), f"E2M1 decode {c:#x}"
        assert lib.orc_e2m1_encode(v) == c, f"E2M1 round trip {c:#x}"
    bits, vals = all_finite_bf16()
    gv, gc = e2m1_grid_golden()
    assert np.array_equal(oracle.e2m1_encode(vals, lib), brute_encode(vals, gv, gc, 0x8)), \
        "E2M1 encode vs exhaustive nearest-even search"
    # the tie points of the grid go to the even code
    ties = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6}
    for v, c in ties.items():
        assert lib.orc_e2m1_encode(v) == c and lib.orc_e2m1_encode(-v) == c | 0x8, f"tie {v}"


def pin_bf16_rounding(lib):
    rng = np.random.default_rng(7)
    # binary32 inputs: torch's float -> bfloat16 conversion is nearest-even
    f = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)).view(np.float32),
    ])
    f = f[np.isfinite(f)]
    mine = oracle.bf16_from_double(f.astype(np.float64), lib)
    assert np.array_equal(mine, f32_to_bf16_bits_torch(f)), "bf16 rounding of binary32"
    # binary64 inputs near bf16 midpoints: exact comparison with Fractions
    b = rng.integers(1, 0x7F7F, 400).astype(np.uint16)
    lo = bf16_bits_to_f64(b)
    hi = bf16_bits_to_f64(b + 1)
    cases = []
    for a, c in zip(lo, hi):
        mid = (a + c) / 2
        cases += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), a, c]
    for v in cases + [-x for x in cases]:
        got = int(lib.orc_bf16_from_double(float(v)))
        fv = Fraction(float(v))
        base = int(np.array([np.float32(abs(float(v)))]).view(np.uint32)[0] >> 16)
        best = None
        for cand in range(max(base - 2, 0), base + 3):
            d = abs(Fraction(float(bf16_bits_to_f64([cand])[0])) - abs(fv))
            key = (d, cand & 1)
            if best is None or key < best[0]:
                best = (key, cand)
        want = best[1] | (0x8000 if v < 0 else 0)
        assert got == want, f"bf16 rounding of {v!r}: {got:#x} vs {want:#x}"
    # ties go to even, and one bf16 step in [8, 16) is the page's 6.25e-2
    pv = json.load(open(os.path.join(GOLDEN, "page_values.json")))["cases"][0]
    step, low = pv["value"], pv["binade_low"]
    assert lib.orc_bf16_to_double(lib.orc_bf16_from_double(low + step)) == low + step
    assert lib.orc_bf16_to_double(lib.orc_bf16_from_double(low + step / 2)) == low
    assert lib.orc_bf16_to_double(lib.orc_bf16_from_double(low + 1.5 * step)) == low + 2 * step
    assert lib.orc_bf16_from_double(3.5e38) == 0x7F80


def pin_mx_scale(lib):
    bits, vals = all_finite_bf16()
    pos = vals[vals > 0]
    mine = oracle.mx_scale_code(pos, lib)
    sample = np.concatenate([pos[::7], pos[:300], pos[-300:]])
    want = np.array([brute_mx_scale_code(float(a)) for a in sample], dtype=np.uint8)
    got = oracle.mx_scale_code(sample, lib)
    assert np.array_equal(got, want), "E8M0 code vs exact power-of-two brackets"
    # power-of-two boundaries: 2^k -> k - 2; the bf16 just below 2^k -> k - 3
    for k in range(-120, 127):
        assert lib.orc_mx_scale_code(2.0 ** k) == k - 2 + 127, f"2^{k}"
        below = 2.0 ** k * (1 - 2 ** -8)
        assert lib.orc_mx_scale_code(below) == max(k - 3 + 127, 0), f"below 2^{k}"
    assert lib.orc_mx_scale_code(0.0) == 0
    assert lib.orc_mx_scale_code(2.0 ** -133) == 0  # smallest bf16 subnormal
    assert lib.orc_mx_scale_code(float("inf")) == 0xFF
    assert np.all(mine <= 252)


def pin_worked_rows(lib):
    cases = {c["id"]: c for c in json.load(open(os.path.join(GOLDEN, "worked_rows.json")))["cases"]}
    w1 = cases["W1"]
    H = w1["H"]
    x = bf16_bits_from_torch(torch.full((1, H), w1["x_value"], dtype=torch.bfloat16))
    w = bf16_bits_from_torch(torch.full((H,), w1["w_value"], dtype=torch.bfloat16))
    r = oracle.rmsnorm_quant([x], None, w, w1["eps"], oracle.FP8_PER_TOKEN, lib)
    assert np.all(bf16_bits_to_f64(r["y"]) == w1["y_value"]), "W1 y"
    assert r["scale"][0] == np.float32(w1["fp8_per_token"]["scale"]), "W1 scale"
    assert np.all(r["q"] == int(w1["fp8_per_token"]["code"], 16)), "W1 codes"
    r = oracle.rmsnorm_quant([x], None, w, w1["eps"], oracle.MXFP4, lib)
    assert np.all(r["scale"] == w1["mxfp4"]["scale_code"]), "W1 MX scale"
    assert np.all(r["q"] == int(w1["mxfp4"]["byte"], 16)), "W1 MX bytes"

    w2 = cases["W2"]
    y = np.zeros((1, w2["pad_to"]), dtype=np.float32)
    y[0, :len(w2["y"])] = w2["y"]
    q, s = oracle.quant_rows(f32_to_bf16_bits_torch(y), w2["mode"], lib)
    assert s[0, 0] == np.float32(w2["scale"]), "W2 scale"
    want = [int(c, 16) for c in w2["codes"]]
    assert list(q[0, :len(want)]) == want, f"W2 codes {q[0, :3]}"
    assert np.all(q[0, len(want):] == int(w2["pad_code"], 16))

    w3 = cases["W3"]
    y = np.zeros((1, w3["pad_to"]), dtype=np.float32)
    y[0, :len(w3["y"])] = w3["y"]
    q, s = oracle.quant_rows(f32_to_bf16_bits_torch(y), w3["mode"], lib)
    assert s[0, 0] == w3["scale_code"], "W3 scale"
    want = [int(c, 16) for c in w3["bytes"]]
    assert list(q[0, :len(want)]) == want, f"W3 bytes {[hex(v) for v in q[0, :3]]}"
    assert np.all(q[0, len(want):] == int(w3["pad_byte"], 16))

    w4 = cases["W4"]
    z = np.zeros((1, w4["H"]), dtype=np.uint16)
    q, s = oracle.quant_rows(z, oracle.MXFP4, lib)
    assert np.all(s == w4["mx_scale_code"]) and np.all(q == int(w4["mx_byte"], 16)), "W4 MX"
    for mode in (oracle.FP8_PER_TOKEN, oracle.FP8_PER_GROUP128):
        q, s = oracle.quant_rows(z, mode, lib)
        assert np.all(s == w4["fp8_scale"]) and np.all(q == int(w4["fp8_code"], 16)), "W4 FP8"


def pin_rstd_closed_form(lib):
    for c in (0.5, 2.0, 3.0, -7.25, 1e-3, 100.0):
        for H in (32, 96, 7168):
            for eps in (1e-6, 1e-5, 0.0):
                h = bf16_bits_from_torch(torch.full((H,), c, dtype=torch.bfloat16))
                cb = float(bf16_bits_to_f64(h[:1])[0])
                want = 1.0 / math.sqrt(cb * cb + float(np.float32(eps)))
                got = oracle.rstd(h, eps, lib)
                assert got == want, f"rstd c={c} H={H} eps={eps}: {got} vs {want}"
                w = bf16_bits_from_torch(torch.full((H,), 1.25, dtype=torch.bfloat16))
                r = oracle.rmsnorm_quant([h.reshape(1, H)], None, w, eps, oracle.MXFP4, lib)
                yb = ref_y_bits([cb], [1.25], eps)[0]
                assert np.all(r["y"] == yb), f"constant-row y c={c} H={H}"


def pin_quant_stage_random(lib):
    """Quantization stage on random bf16 rows vs the library/brute formulations."""
    g = torch.Generator().manual_seed(11)
    y = torch.randn((6, 512), generator=g) * torch.pow(10.0, torch.rand((6, 1), generator=g) * 4 - 2)
    y[1, 5] *= 50.0
    y[2, :128] = 0.0
    y[3, 32:64] = 0.0
    y[4, 64:96] = 2.0 ** -130  # subnormal block
    yb = bf16_bits_from_torch(y.to(torch.bfloat16))
    for mode, group in ((oracle.FP8_PER_TOKEN, 512), (oracle.FP8_PER_GROUP128, 128)):
        q, s = oracle.quant_rows(yb, mode, lib)
        rq, rs = ref_quant_fp8(yb, group)
        assert np.array_equal(q, rq), f"FP8 codes mode {mode}"
        assert np.array_equal(s.reshape(rs.shape), rs), f"FP8 scales mode {mode}"
        # invariant: the largest element of a non-zero group encodes as +-448
        for m in range(yb.shape[0]):
            for gi in range(512 // group):
                seg = bf16_bits_to_f64(yb[m, gi * group:(gi + 1) * group])
                if np.any(seg != 0):
                    j = int(np.argmax(np.abs(seg)))
                    assert q[m, gi * group + j] & 0x7F == 0x7E, "amax element is 448"
    q, s = oracle.quant_rows(yb, oracle.MXFP4, lib)
    rq, rs = ref_quant_mx(yb)
    assert np.array_equal(q, rq), "MXFP4 codes"
    assert np.array_equal(s, rs), "MXFP4 scales"


def _small_case(seed, M, H, P, residual):
    g = torch.Generator().manual_seed(seed)
    parts = []
    for _ in range(P):
        t = torch.randn((M, H), generator=g) * (torch.rand((M, 1), generator=g) * 8 + 0.1)
        parts.append(bf16_bits_from_torch(t.to(torch.bfloat16)))
    res = bf16_bits_from_torch(torch.randn((M, H), generator=g).to(torch.bfloat16)) if residual else None
    w = bf16_bits_from_torch((1 + 0.3 * torch.randn((H,), generator=g)).to(torch.bfloat16))
    return parts, res, w


def pin_full_path_bruteforce(lib):
    """Tiny rows: the whole unfused sequence recomputed independently."""
    cases = [(1, 2, 32, 1, True, oracle.FP8_PER_TOKEN), (2, 3, 32, 2, True, oracle.MXFP4),
             (3, 2, 64, 3, False, oracle.MXFP4), (4, 2, 128, 4, True, oracle.FP8_PER_GROUP128),
             (5, 2, 256, 1, True, oracle.FP8_PER_GROUP128), (6, 1, 96, 4, True, oracle.FP8_PER_TOKEN)]
    for seed, M, H, P, has_res, mode in cases:
        parts, res, w = _small_case(seed, M, H, P, has_res)
        eps = 1e-6 if seed % 2 else 1e-5
        r = oracle.rmsnorm_quant(parts, res, w, eps, mode, lib)
        h = ref_residual_bits(parts, res)
        assert np.array_equal(r["residual_out"], h), f"residual case {seed}"
        wv = bf16_bits_to_f64(w)
        y = np.stack([ref_y_bits(bf16_bits_to_f64(h[m]), wv, eps) for m in range(M)])
        assert np.array_equal(r["y"], y), f"y case {seed}"
        if mode == oracle.MXFP4:
            rq, rs = ref_quant_mx(y)
        else:
            rq, rs = ref_quant_fp8(y, H if mode == oracle.FP8_PER_TOKEN else 128)
        assert np.array_equal(r["q"], rq), f"codes case {seed}"
        assert np.array_equal(r["scale"].reshape(rs.shape), rs), f"scales case {seed}"


def pin_partial_sum_order(lib):
    """A3: fp32 sums in order p = 0..P-1, then the residual, one bf16 rounding."""
    g = torch.Generator().manual_seed(21)
    M, H, P = 16, 2048, 4
    c = torch.pow(10.0, torch.rand((H,), generator=g) * 2 - 1)
    parts = [bf16_bits_from_torch((torch.randn((M, H), generator=g) * c).to(torch.bfloat16))
             for _ in range(P)]
    res = bf16_bits_from_torch(torch.randn((M, H), generator=g).to(torch.bfloat16))
    w = bf16_bits_from_torch(torch.ones((H,), dtype=torch.bfloat16))
    # Rows where binary32 rounding of the running sum decides the bf16 result:
    # p0 = s(1 + 2^-7), p1 = s 2^-30, r = -s 2^-8.  Exactly, h is just above
    # the bf16 midpoint s(1 + 2^-8) and rounds up; in binary32, p0 + p1 drops
    # the 2^-30 term, the sum lands on the midpoint and rounds to even (down).
    k = np.arange(-20, 20)
    s = 2.0 ** k
    vals = [np.concatenate([s * (1 + 2 ** -7), -s * (1 + 2 ** -7)]),
            np.concatenate([s * 2.0 ** -30, -s * 2.0 ** -30]),
            np.concatenate([-s * 2.0 ** -8, s * 2.0 ** -8])]
    cons = [f32_to_bf16_bits_torch(v.astype(np.float32)) for v in vals]
    n = cons[0].size
    for i in range(3):
        tgt = parts[i] if i < 2 else res
        tgt[0, :n] = cons[i]
    for i in range(2, P):
        parts[i][0, :n] = 0
    r = oracle.rmsnorm_quant(parts, res, w, 1e-6, oracle.MXFP4, lib)
    want = ref_residual_bits(parts, res)
    assert np.array_equal(r["residual_out"], want), "fp32 partial sum order"
    # the construction really separates the two orders of rounding
    exact = [nearest_bf16_decimal(sum(Decimal(float(bf16_bits_to_f64([c[i]])[0])) for c in cons))
             for i in range(n)]
    assert not np.any(np.array(exact, dtype=np.uint16) == want[0, :n])


def pin_qk_layout(lib):
    """Interleaved q/gate heads, k after them, v never read; each head checked
    against the decimal Gemma norm, each gate against its own source slice."""
    M, Hq, Hk, D = 2, 3, 2, 32
    stride = (2 * Hq + 2 * Hk) * D + 16  # v heads, then padding
    g = torch.Generator().manual_seed(5)
    qkv = torch.randn((M, stride), generator=g).to(torch.bfloat16)
    # per head a distinct offset, so a misplaced slice cannot pass
    for h in range(2 * Hq + Hk):
        qkv[:, h * D:(h + 1) * D] += float(h + 1)
    x = bf16_bits_from_torch(qkv)
    x[:, (2 * Hq + Hk) * D:] = 0x7FC0  # v heads and padding: NaN, must not leak
    qw = bf16_bits_from_torch((0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16))
    kw = bf16_bits_from_torch((0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16))
    r = oracle.qk_norm_gate(x, stride, Hq, Hk, D, qw, kw, 1e-6, lib)
    qwv, kwv = bf16_bits_to_f64(qw), bf16_bits_to_f64(kw)
    for m in range(M):
        for h in range(Hq):
            src = bf16_bits_to_f64(x[m, 2 * h * D:(2 * h + 1) * D])
            assert np.array_equal(r["q"][m, h], ref_y_bits(src, qwv, 1e-6, gemma=True)), f"q {m},{h}"
            assert np.array_equal(r["gate"][m, h], x[m, (2 * h + 1) * D:(2 * h + 2) * D]), f"gate {m},{h}"
        for h in range(Hk):
            off = 2 * Hq * D + h * D
            src = bf16_bits_to_f64(x[m, off:off + D])
            assert np.array_equal(r["k"][m, h], ref_y_bits(src, kwv, 1e-6, gemma=True)), f"k {m},{h}"


ALL_PINS = [pin_e4m3_decode, pin_e4m3_encode, pin_e2m1, pin_bf16_rounding, pin_mx_scale,
            pin_worked_rows, pin_rstd_closed_form, pin_quant_stage_random,
            pin_full_path_bruteforce, pin_partial_sum_order, pin_qk_layout]


def pin_scale_layouts(lib):
    """The placement of scales in the GEMM layouts: the 32x4x4 swizzle against
    a library's own implementation of that layout (quack.mx_utils.to_blocked),
    the M-major layout against a plain transpose."""
    from quack.mx_utils import to_blocked
    rng = np.random.default_rng(3)
    for M, G in ((1, 1), (5, 7), (128, 4), (130, 9), (300, 224), (257, 56)):
        a = rng.integers(0, 255, (M, G)).astype(np.uint8)
        mine = oracle.place_scales(a, oracle.SCALE_SWIZZLE_32_4_4)
        ref = to_blocked(torch.from_numpy(a)).numpy().reshape(-1)
        assert np.array_equal(mine, ref), f"swizzled layout {M}x{G}"
        f = rng.standard_normal((M, G)).astype(np.float32)
        mm = oracle.place_scales(f, oracle.SCALE_MN_MAJOR).reshape(G, -1)
        assert mm.shape[1] == (M + 3) // 4 * 4
        assert np.array_equal(mm[:, :M], f.T) and np.all(mm[:, M:] == 0), f"M-major {M}x{G}"


ALL_PINS.append(pin_scale_layouts)


def pin_qk_fp8(lib):
    """The FP8 QK prologue is the bf16 prologue followed by the per-token FP8
    quantization of each head vector (two pinned pieces composed), and its
    gate is the same bit copy."""
    M, Hq, Hk, D = 3, 4, 2, 64
    stride = (2 * Hq + 2 * Hk) * D
    g = torch.Generator().manual_seed(8)
    x = bf16_bits_from_torch((torch.randn((M, stride), generator=g) *
                              torch.pow(10.0, torch.rand((M, 1), generator=g) * 4 - 2)).to(torch.bfloat16))
    x[1, 2 * D:3 * D] = 0  # an all-zero q head: scale 1, codes 0
    qw = bf16_bits_from_torch((0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16))
    kw = bf16_bits_from_torch((0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16))
    base = oracle.qk_norm_gate(x, stride, Hq, Hk, D, qw, kw, 1e-6, lib)
    f8 = oracle.qk_norm_gate_fp8(x, stride, Hq, Hk, D, qw, kw, 1e-6, lib)
    for name, H in (("q", Hq), ("k", Hk)):
        y = base[name].reshape(M * H, D)
        assert np.array_equal(f8[name].reshape(M * H, D), y)
        rq, rs = oracle.quant_rows(y, oracle.FP8_PER_TOKEN, lib)
        assert np.array_equal(f8[name + "8"].reshape(M * H, D), rq), f"{name} codes"
        assert np.array_equal(f8[name + "s"].reshape(-1), rs), f"{name} scales"
    assert np.array_equal(f8["gate"], base["gate"])
    assert f8["qs"][1, 1] == 1.0 and np.all(f8["q8"][1, 1] == 0)


ALL_PINS.append(pin_qk_fp8)


# ----------------------------------------------------------------------------
# binary16 input/output
# ----------------------------------------------------------------------------


def fp16_bits_to_f64(bits):
    """binary16 bit patterns -> values, by numpy's own half-precision type."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def nearest_fp16_decimal(x: Decimal) -> int:
    """binary16 bit pattern nearest to a high-precision value (ties to even;
    finite values only)."""
    if x == 0:
        return 0x8000 if x.is_signed() else 0
    neg = x < 0
    ax = -x if neg else x
    base = int(np.array([np.float16(float(ax))]).view(np.uint16)[0])
    best = None
    for b in range(max(base - 2, 0), min(base + 3, 0x7C00)):
        d = abs(Decimal(float(fp16_bits_to_f64([b])[0])) - ax)
        key = (d, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1] | 0x8000 if neg else best[1]


def pin_fp16_format(lib):
    """binary16 decode and rounding against numpy's float16 and exact
    Fraction arithmetic: every pattern, random values, ties, overflow and
    subnormals."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = fp16_bits_to_f64(bits)
    mine = oracle.fp16_to_double(bits, lib)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan), "binary16 NaN patterns"
    assert np.array_equal(mine[~nan], ref[~nan]), "binary16 decode vs numpy"
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(ref[~nan])), "binary16 signed zero"
    assert np.array_equal(oracle.fp16_from_double(ref[~nan], lib), bits[~nan]), "round trip"
    # binary32 inputs (so numpy's conversion rounds once) across the range
    rng = np.random.default_rng(17)
    f = (rng.standard_normal(40000) * np.exp2(rng.uniform(-30, 18, 40000))).astype(np.float32)
    with np.errstate(over="ignore"):  # beyond 65520 numpy gives infinity, as it should
        ref16 = f.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.fp16_from_double(f.astype(np.float64), lib), ref16), \
        "binary16 rounding vs numpy"
    # midpoints between neighbours: ties to the even pattern, exactly
    for b in list(rng.integers(0, 0x7BFF, 300)) + [0, 1, 0x3FF, 0x400, 0x3BFF, 0x7BFE]:
        b = int(b)
        lo, hi = fp16_bits_to_f64([b, b + 1])
        mid = (lo + hi) / 2
        assert Fraction(mid) == (Fraction(lo) + Fraction(hi)) / 2
        want_tie = b if b % 2 == 0 else b + 1
        for sgn, sb in ((1.0, 0), (-1.0, 0x8000)):
            assert lib.orc_fp16_from_double(sgn * mid) == want_tie | sb, f"tie above {b:#x}"
            assert lib.orc_fp16_from_double(sgn * np.nextafter(mid, 0)) == b | sb
            assert lib.orc_fp16_from_double(sgn * np.nextafter(mid, np.inf)) == (b + 1) | sb
    # overflow: 65520 is the midpoint between 65504 (odd) and 2^16: infinity
    assert lib.orc_fp16_from_double(65520.0) == 0x7C00
    assert lib.orc_fp16_from_double(np.nextafter(65520.0, 0)) == 0x7BFF
    assert lib.orc_fp16_from_double(-1e9) == 0xFC00
    # subnormals: 2^-25 ties to 0, 3 2^-25 ties to 2 2^-24
    assert lib.orc_fp16_from_double(2.0 ** -25) == 0
    assert lib.orc_fp16_from_double(-(2.0 ** -25)) == 0x8000
    assert lib.orc_fp16_from_double(np.nextafter(2.0 ** -25, 1)) == 1
    assert lib.orc_fp16_from_double(3 * 2.0 ** -25) == 2


def _small_case_fp16(seed, M, H, P, residual):
    g = torch.Generator().manual_seed(seed)
    as_bits = lambda t: t.to(torch.float16).contiguous().view(torch.int16).numpy().view(np.uint16)
    parts = [as_bits(torch.randn((M, H), generator=g) * (torch.rand((M, 1), generator=g) * 8 + 0.1))
             for _ in range(P)]
    res = as_bits(torch.randn((M, H), generator=g)) if residual else None
    w = as_bits(1 + 0.3 * torch.randn((H,), generator=g))
    return parts, res, w


def pin_fp16_path(lib):
    """io = binary16: the whole unfused sequence recomputed independently
    (numpy fp32 sums rounded once by numpy, the norm in 60-digit decimal
    rounded to the nearest binary16, the quantization by the library and
    brute formulations), the constant-row closed form of W1, and the
    quantization of binary16 rows with subnormal and near-overflow values."""
    F16 = oracle.IO_FP16
    cases = [(1, 2, 32, 1, True, oracle.FP8_PER_TOKEN), (2, 2, 64, 3, True, oracle.MXFP4),
             (3, 2, 128, 2, False, oracle.FP8_PER_GROUP128), (4, 1, 96, 4, True, oracle.MXFP4)]
    getcontext().prec = 60
    for seed, M, H, P, has_res, mode in cases:
        parts, res, w = _small_case_fp16(seed, M, H, P, has_res)
        eps = 1e-6 if seed % 2 else 1e-5
        r = oracle.rmsnorm_quant(parts, res, w, eps, mode, lib, io=F16)
        acc = fp16_bits_to_f64(parts[0]).astype(np.float32)
        for p in parts[1:] + ([res] if has_res else []):
            acc = (acc + fp16_bits_to_f64(p).astype(np.float32)).astype(np.float32)
        h = acc.astype(np.float16).view(np.uint16)
        assert np.array_equal(r["residual_out"], h), f"fp16 residual case {seed}"
        wv = fp16_bits_to_f64(w)
        y = np.zeros((M, H), dtype=np.uint16)
        for m in range(M):
            hv = fp16_bits_to_f64(h[m])
            rs = decimal_rstd(hv, np.float32(eps))
            y[m] = [nearest_fp16_decimal(Decimal(float(a)) * rs * Decimal(float(b)))
                    for a, b in zip(hv, wv)]
        assert np.array_equal(r["y"], y), f"fp16 y case {seed}"
        if mode == oracle.MXFP4:
            rq, rsc = ref_quant_mx(y, fp16_bits_to_f64)
        else:
            rq, rsc = ref_quant_fp8(y, H if mode == oracle.FP8_PER_TOKEN else 128, fp16_bits_to_f64)
        assert np.array_equal(r["q"], rq), f"fp16 codes case {seed}"
        assert np.array_equal(r["scale"].reshape(rsc.shape), rsc), f"fp16 scales case {seed}"
    # W1 with binary16 storage: y = 1 exactly, so the same codes and scales
    w1 = {c["id"]: c for c in json.load(open(os.path.join(GOLDEN, "worked_rows.json")))["cases"]}["W1"]
    H = w1["H"]
    x = np.full((1, H), np.float16(w1["x_value"])).view(np.uint16)
    wt = np.full((H,), np.float16(w1["w_value"])).view(np.uint16)
    r = oracle.rmsnorm_quant([x], None, wt, w1["eps"], oracle.FP8_PER_TOKEN, lib, io=F16)
    assert np.all(fp16_bits_to_f64(r["y"]) == w1["y_value"]), "W1 fp16 y"
    assert r["scale"][0] == np.float32(w1["fp8_per_token"]["scale"])
    assert np.all(r["q"] == int(w1["fp8_per_token"]["code"], 16))
    r = oracle.rmsnorm_quant([x], None, wt, w1["eps"], oracle.MXFP4, lib, io=F16)
    assert np.all(r["scale"] == w1["mxfp4"]["scale_code"])
    assert np.all(r["q"] == int(w1["mxfp4"]["byte"], 16))
    # quantization of binary16 rows over the format's whole range
    rng = np.random.default_rng(23)
    y = (rng.standard_normal((4, 256)) * np.exp2(rng.integers(-20, 12, (4, 1)))).astype(np.float16)
    y[1, :32] = np.float16(2.0 ** -24) * rng.integers(-3, 4, 32)  # subnormal block
    y[2, 7] = np.float16(65504.0)
    y[3, 100:140] = 0
    yb = y.view(np.uint16)
    for mode, group in ((oracle.FP8_PER_TOKEN, 256), (oracle.FP8_PER_GROUP128, 128)):
        q, sc = oracle.quant_rows(yb, mode, lib, io=F16)
        rq, rsc = ref_quant_fp8(yb, group, fp16_bits_to_f64)
        assert np.array_equal(q, rq) and np.array_equal(sc.reshape(rsc.shape), rsc), f"fp16 FP8 {mode}"
    q, sc = oracle.quant_rows(yb, oracle.MXFP4, lib, io=F16)
    rq, rsc = ref_quant_mx(yb, fp16_bits_to_f64)
    assert np.array_equal(q, rq) and np.array_equal(sc, rsc), "fp16 MXFP4"
    assert sc[2, 0] == 15 - 2 + 127  # amax 65504: floor(log2) = 15


ALL_PINS += [pin_fp16_format, pin_fp16_path]


# ----------------------------------------------------------------------------
# hc_mix: the low-rank gate over the hyper-state (reading A19)
# ----------------------------------------------------------------------------


def _bf16_bits_f64(a):
    """float64 values that are exact in bf16 -> their bit patterns."""
    return f32_to_bf16_bits_torch(np.asarray(a, dtype=np.float32))


def _hc_case(seed, M, hc, C, r, wd_std=None, wu_std=None):
    rng = np.random.default_rng(seed)
    K = hc * C
    x = f32_to_bf16_bits_torch(rng.standard_normal((M, K)).astype(np.float32))
    wd = f32_to_bf16_bits_torch((rng.standard_normal((r, K)) * (wd_std or K ** -0.5)).astype(np.float32))
    wu = f32_to_bf16_bits_torch((rng.standard_normal((K, r)) * (wu_std or r ** -0.5)).astype(np.float32))
    return x, wd, wu


def pin_hc_mix_worked(lib):
    """The hand-worked row of tests/golden/hc_mix_worked.json."""
    d = json.load(open(os.path.join(GOLDEN, "hc_mix_worked.json")))
    x = _bf16_bits_f64([d["x"]])
    wd, wu = _bf16_bits_f64(d["w_down"]), _bf16_bits_f64(d["w_up"])
    u, ub = oracle.hc_mix(x, wd, wu, d["hc"], d["C"], d["r"], lib)
    assert np.allclose(u[0], d["u"], rtol=0, atol=1e-15), f"hc_mix worked u {u[0]}"
    assert list(bf16_bits_to_f64(ub[0])) == d["u_bf16"], f"hc_mix worked bf16 {ub[0]}"


def pin_hc_mix_closed_forms(lib):
    """Closed forms and invariants of the gated mix on random rows:
    zero up-factor -> every gate 1/2 and u = (sum of the streams) / 2, exactly;
    negated up-factor -> gates 1 - g, so u + u' = sum of the streams;
    logits of +-40 built through both factors select stream 0 alone;
    a permutation of the streams (applied to x, to W_down's column blocks and
    to W_up's row blocks) leaves u unchanged; a permutation of the channels
    permutes u."""
    hc, C, r, M = 4, 24, 8, 3
    K = hc * C
    x, wd, wu = _hc_case(11, M, hc, C, r)
    xv = bf16_bits_to_f64(x).reshape(M, hc, C)
    streams = xv.sum(axis=1)
    u0, _ = oracle.hc_mix(x, wd, np.zeros_like(wu), hc, C, r, lib)
    assert np.array_equal(u0, 0.5 * streams), "zero up-factor: u = sum/2"
    u, _ = oracle.hc_mix(x, wd, wu, hc, C, r, lib)
    un, _ = oracle.hc_mix(x, wd, wu ^ np.uint16(0x8000), hc, C, r, lib)
    assert np.allclose(u + un, streams, rtol=0, atol=1e-12), "negated up-factor"
    # selection: t0 = x[0] = 1 through a one-hot down row; z = +-40 per stream
    xs = x.copy()
    xs[:, 0] = 0x3F80  # 1.0
    wds = np.zeros_like(wd)
    wds[0, 0] = 0x3F80
    wus = np.zeros_like(wu)
    wus[:, 0] = 0xC220  # -40
    wus[:C, 0] = 0x4220  # +40 on stream 0
    us, _ = oracle.hc_mix(xs, wds, wus, hc, C, r, lib)
    xsv = bf16_bits_to_f64(xs).reshape(M, hc, C)
    assert np.allclose(us, xsv[:, 0, :], rtol=0, atol=1e-15), "selection of stream 0"
    # stream permutation
    perm = [2, 0, 3, 1]
    cols = np.concatenate([np.arange(s * C, (s + 1) * C) for s in perm])
    up, _ = oracle.hc_mix(x[:, cols], wd[:, cols], wu[cols, :], hc, C, r, lib)
    assert np.allclose(up, u, rtol=0, atol=1e-12), "stream permutation"
    # channel permutation
    cp = np.random.default_rng(5).permutation(C)
    ccols = np.concatenate([s * C + cp for s in range(hc)])
    uc, _ = oracle.hc_mix(x[:, ccols], wd[:, ccols], wu[ccols, :], hc, C, r, lib)
    assert np.allclose(uc, u[:, cp], rtol=0, atol=1e-12), "channel permutation"
    assert K == x.shape[1]


def pin_hc_mix_library(lib):
    """The whole mix recomputed with library routines on tiny random cases:
    numpy fp64 matrix products for the two factors, scipy's logistic function
    for the gate, a sum over the reshaped streams, and the bf16 output by the
    60-digit nearest search."""
    from scipy.special import expit
    for seed, (M, hc, C, r) in enumerate([(1, 4, 8, 8), (5, 4, 16, 4), (3, 2, 40, 16),
                                          (2, 4, 64, 64)]):
        x, wd, wu = _hc_case(100 + seed, M, hc, C, r, wd_std=2.0 / (hc * C) ** 0.5,
                             wu_std=2.0 / r ** 0.5)
        xv, wdv, wuv = bf16_bits_to_f64(x), bf16_bits_to_f64(wd), bf16_bits_to_f64(wu)
        g = expit((xv @ wdv.T) @ wuv.T)
        want = (g * xv).reshape(M, hc, C).sum(axis=1)
        u, ub = oracle.hc_mix(x, wd, wu, hc, C, r, lib)
        assert np.allclose(u, want, rtol=1e-12, atol=1e-12), f"hc_mix library case {seed}"
        getcontext().prec = 60
        wb = np.array([[nearest_bf16_decimal(Decimal(float(v))) for v in row] for row in u],
                      dtype=np.uint16)
        assert np.array_equal(ub, wb), f"hc_mix bf16 output case {seed}"


ALL_PINS += [pin_hc_mix_worked, pin_hc_mix_closed_forms, pin_hc_mix_library]
