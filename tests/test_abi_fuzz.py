"""Property tests of the argument checks of fn_rmsnorm_quant, fn_hc_mix and
fn_hc_mix_noalloc (no GPU).

Random calls over fake, far-apart device addresses, with sizes, modes, flags,
alignments and overlaps drawn to hit every rule of include/fusednorm.h.  The
rules are restated here from the header, independently of the C code: a call
that breaks no rule must pass every check (on this CPU-only machine it then
fails at the launch with FN_ERR_CUDA, proving it got that far), and a call
that breaks rules must return one of the statuses those rules name, having
launched nothing.
"""
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

SPACE = 1 << 36  # distance between the fake buffers


@pytest.fixture(scope="module")
def fnb():
    from mxfp4_quantization_b200.build import build_library
    build_library()
    from mxfp4_quantization_b200 import fusednorm
    return fusednorm


def _round_up(x, m):
    return (x + m - 1) // m * m


def expected(fnb, a):
    """The set of statuses the header allows for call `a` ({FN_ERR_CUDA}
    when no rule is broken: the call reaches the launch)."""
    E, A, U, OK = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED, fnb.FN_OK
    bad = set()
    P, M, H, mode = a["P"], a["M"], a["H"], a["mode"]
    q, flags = mode & 0xFF, mode & ~0xFF
    SW, MN, F16 = fnb.FN_SCALE_SWIZZLE_32_4_4, fnb.FN_SCALE_MN_MAJOR, fnb.FN_IO_FP16
    if not 1 <= P <= 8:
        return {E}
    layout = flags & ~F16
    if q not in (0, 1, 2) or layout not in (0, SW, MN) or (layout == SW and q != 2) or \
            (layout == MN and q != 1):
        return {E}
    if M < 0 or H <= 0 or H % 8 or (q == 1 and H % 128) or (q == 2 and H % 32):
        return {E}
    if H > 32768:
        return {U}
    if a["eps"] != a["eps"] or a["eps"] < 0:
        return {E}
    if M == 0:
        return {OK}
    ptr = a["ptr"]
    if ptr["weight"] is None or ptr["out_q"] is None or ptr["out_scale"] is None:
        bad.add(E)
    if ptr["residual"] is not None and ptr["out_residual"] is None:
        bad.add(E)
    if any(p is None for p in ptr["parts"]):
        bad.add(E)
    for p in ptr["parts"]:
        if p is not None and p % 16:
            bad.add(A)
    for k in ("weight", "residual", "out_residual", "out_y"):
        if ptr[k] is not None and ptr[k] % 16:
            bad.add(A)
    if ptr["out_q"] is not None and ptr["out_q"] % (4 if q == 2 else 8):
        bad.add(A)
    if q != 2 and ptr["out_scale"] is not None and ptr["out_scale"] % 4:
        bad.add(A)
    if bad:
        return bad
    rows = M * H * 2
    codes = M * H // 2 if q == 2 else M * H
    if q == 0:
        scales = M * 4
    elif q == 1:
        scales = (_round_up(M, 4) if layout == MN else M) * (H // 128) * 4
    else:
        scales = _round_up(M, 128) * _round_up(H // 32, 4) if layout == SW else M * (H // 32)
    outs = [("out_q", codes), ("out_scale", scales)]
    outs += [(k, rows) for k in ("out_residual", "out_y") if ptr[k] is not None]
    ins = [(p, rows) for p in ptr["parts"]] + [(ptr["weight"], H * 2)]
    hit = lambda a0, n0, a1, n1: a0 < a1 + n1 and a1 < a0 + n0  # noqa: E731
    for i, (k, n) in enumerate(outs):
        for k2, n2 in outs[i + 1:]:
            if hit(ptr[k], n, ptr[k2], n2):
                bad.add(E)
        for p, n2 in ins:
            if hit(ptr[k], n, p, n2):
                bad.add(E)
        if ptr["residual"] is not None and hit(ptr[k], n, ptr["residual"], rows) and \
                not (k == "out_residual" and ptr[k] == ptr["residual"]):
            bad.add(E)
    return bad or {fnb.FN_ERR_CUDA}


@st.composite
def calls(draw):
    # mostly well-formed modes and shapes, so that the pointer rules get exercised
    rare = draw(st.integers(0, 9)) == 0
    P = draw(st.sampled_from([0, 9, 5])) if rare else draw(st.sampled_from([1, 2, 3, 4, 8]))
    q = draw(st.sampled_from([0, 1, 2]))
    if draw(st.integers(0, 9)) == 0:
        flags = draw(st.sampled_from([0x400, 0x300, 0x2000, 0x100, 0x200]))
        q = draw(st.sampled_from([q, 3, -1]))
    else:
        flags = draw(st.sampled_from([0, 0x1000] + ([0x100, 0x1100] if q == 2 else []) +
                                     ([0x200, 0x1200] if q == 1 else [])))
    M = draw(st.sampled_from([0, -1])) if draw(st.integers(0, 9)) == 0 else \
        draw(st.sampled_from([1, 3, 16, 129, 1000]))
    if draw(st.integers(0, 9)) == 0:
        H = draw(st.sampled_from([0, 12, 96, 32776, 40960]))
    else:
        H = draw(st.sampled_from([128, 256, 2048, 7168, 8192, 32768] + ([8, 24] if q == 0 else [])))
    eps = draw(st.sampled_from([-1.0, float("nan")])) if draw(st.integers(0, 19)) == 0 else \
        draw(st.sampled_from([1e-6, 0.0]))
    slot = iter(range(1, 32))

    def addr(null_ok=True):
        if null_ok and draw(st.integers(0, 49)) == 0:
            return None
        base = next(slot) * SPACE
        if draw(st.integers(0, 14)) == 0:
            return base + draw(st.sampled_from([4, 8, 2, 1]))  # misaligned for some rules
        return base + draw(st.sampled_from([0, 16, 256]))

    ptr = {"parts": [addr() for _ in range(max(P, 0))], "weight": addr(),
           "residual": addr() if draw(st.booleans()) else None, "out_q": addr(),
           "out_scale": addr(), "out_residual": addr() if draw(st.booleans()) else None,
           "out_y": addr() if draw(st.booleans()) else None}
    # sometimes place one output on or next to an input, or on another output
    kind = draw(st.integers(0, 5))
    if kind == 1 and ptr["residual"] is not None:
        ptr["out_residual"] = ptr["residual"]  # the allowed in-place form
    elif kind == 2 and ptr["parts"] and ptr["parts"][0] is not None:
        ptr[draw(st.sampled_from(["out_q", "out_y", "out_scale"]))] = ptr["parts"][0] + 64
    elif kind == 3 and ptr["out_q"] is not None:
        ptr["out_scale"] = ptr["out_q"] + 512
    elif kind == 4 and ptr["residual"] is not None:
        ptr[draw(st.sampled_from(["out_y", "out_q"]))] = ptr["residual"] + 16
    return {"P": P, "M": M, "H": H, "mode": q | flags if q >= 0 else q, "eps": eps, "ptr": ptr}


@settings(max_examples=600, deadline=None, suppress_health_check=list(HealthCheck))
@given(a=calls())
def test_status_follows_the_documented_rules(fnb, a):
    ptr = a["ptr"]
    parts = ptr["parts"] if a["P"] > 0 else [0x10]
    got = fnb.fn_rmsnorm_quant(parts, a["P"], ptr["residual"], ptr["weight"], a["eps"], a["mode"],
                               a["M"], a["H"], ptr["out_q"], ptr["out_scale"], ptr["out_residual"],
                               ptr["out_y"], None)
    want = expected(fnb, a)
    assert got in want, (got, want, a)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE


# ---- fn_hc_mix and fn_hc_mix_noalloc -------------------------------------------------


def expected_hc(fnb, a, noalloc=False):
    """The statuses include/fusednorm.h allows for hc_mix call `a`
    ({FN_ERR_CUDA} when no rule is broken: the call reaches the launch)."""
    E, A, U, OK = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED, fnb.FN_OK
    M, hc, C, r = a["M"], a["hc"], a["C"], a["r"]
    if M < 0 or hc < 1 or C <= 0 or r <= 0:
        return {E}
    if hc != 4 or M > 16 or C % 16 or hc * C > 16384 or r % 8 or r > 128:
        return {U}
    if M == 0:
        return {OK}
    ptr = a["ptr"]
    names = ("x", "w_down", "w_up", "out") + (() if noalloc else ("workspace",))
    bad = set()
    for k in names:
        if ptr[k] is None:
            bad.add(E)
        elif ptr[k] % 16:
            bad.add(A)
    if bad:
        return bad
    if noalloc and M * r > 16 * 128:
        return {U}
    K = hc * C
    ins = [(ptr["x"], M * K * 2), (ptr["w_down"], r * K * 2), (ptr["w_up"], K * r * 2)]
    outs = [(ptr["out"], M * C * 2)] + ([] if noalloc else [(ptr["workspace"], M * r * 4)])
    hit = lambda a0, n0, a1, n1: a0 < a1 + n1 and a1 < a0 + n0  # noqa: E731
    for i, (p, n) in enumerate(outs):
        for p2, n2 in outs[i + 1:]:
            if hit(p, n, p2, n2):
                bad.add(E)
        for p2, n2 in ins:
            if hit(p, n, p2, n2):
                bad.add(E)
    return bad or {fnb.FN_ERR_CUDA}


@st.composite
def hc_calls(draw):
    rare = lambda: draw(st.integers(0, 9)) == 0  # noqa: E731
    M = draw(st.sampled_from([-1, 0, 17, 40])) if rare() else draw(st.sampled_from([1, 3, 8, 16]))
    hc = draw(st.sampled_from([0, 2, 8])) if rare() else 4
    C = draw(st.sampled_from([0, 24, 4112, 8192])) if rare() else \
        draw(st.sampled_from([16, 512, 2560, 4096]))
    r = draw(st.sampled_from([0, 12, 136])) if rare() else draw(st.sampled_from([8, 64, 128]))
    slot = iter(range(1, 16))

    def addr():
        if draw(st.integers(0, 39)) == 0:
            return None
        base = next(slot) * SPACE
        if draw(st.integers(0, 14)) == 0:
            return base + draw(st.sampled_from([4, 8, 2]))
        return base + draw(st.sampled_from([0, 16, 256]))

    ptr = {k: addr() for k in ("x", "w_down", "w_up", "out", "workspace")}
    kind = draw(st.integers(0, 5))
    if kind == 1 and ptr["x"] is not None:
        ptr[draw(st.sampled_from(["out", "workspace"]))] = ptr["x"] + 64
    elif kind == 2 and ptr["out"] is not None:
        ptr["workspace"] = ptr["out"] + 32
    elif kind == 3 and ptr["w_up"] is not None:
        ptr["out"] = ptr["w_up"] + 16
    return {"M": M, "hc": hc, "C": C, "r": r, "ptr": ptr}


@settings(max_examples=400, deadline=None, suppress_health_check=list(HealthCheck))
@given(a=hc_calls())
def test_hc_mix_status_follows_the_documented_rules(fnb, a):
    p = a["ptr"]
    got = fnb.fn_hc_mix(p["x"], p["w_down"], p["w_up"], a["M"], a["hc"], a["C"], a["r"], p["out"],
                        p["workspace"], None)
    want = expected_hc(fnb, a)
    assert got in want, (got, want, a)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE


@settings(max_examples=300, deadline=None, suppress_health_check=list(HealthCheck))
@given(a=hc_calls())
def test_hc_mix_noalloc_status_follows_the_documented_rules(fnb, a):
    p = a["ptr"]
    got = fnb.fn_hc_mix_noalloc(p["x"], p["w_down"], p["w_up"], a["M"], a["hc"], a["C"], a["r"],
                                p["out"], None)
    want = expected_hc(fnb, a, noalloc=True)
    assert got in want, (got, want, a)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE
