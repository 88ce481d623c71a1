"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/fusednorm.h declares, and rejects bad arguments before any CUDA
call.  Pointers here are fake addresses: a rejected call never dereferences
or launches anything, and a call that wrongly got through would reach the CUDA
runtime, find no device and return FN_ERR_CUDA, failing the test."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fusednorm.h")


@pytest.fixture(scope="module")
def fnb():
    from mxfp4_quantization_b200.build import build_library
    build_library()
    from mxfp4_quantization_b200 import fusednorm
    return fusednorm


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"FN_API\s+[\w\s\*]+?\b(fn_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    assert declared_symbols() == sorted(["fn_rmsnorm_quant", "fn_ar_rmsnorm_quant", "fn_quant",
                                         "fn_qk_norm_gate",
                                         "fn_qk_norm_gate_fp8", "fn_hc_mix",
                                         "fn_hc_mix_workspace_bytes", "fn_hc_mix_noalloc",
                                         "fn_status_string", "fn_last_variant",
                                         "fn_last_launch", "fn_prefer_variant",
                                         "fn_programmatic_launch", "fn_version"])


def test_library_exports_every_declared_symbol(fnb):
    out = subprocess.run(["nm", "-D", "--defined-only", fnb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fn_\w+)", out))
    missing = set(declared_symbols()) - exported
    assert not missing, f"not exported: {missing}"
    assert set(fnb.ABI_SYMBOLS) == set(declared_symbols())
    # nothing but the ABI leaks out with default visibility
    assert exported == set(declared_symbols())


def test_header_constants_match_binding(fnb):
    src = open(HEADER).read()
    for name in ("FN_FP8_PER_TOKEN", "FN_FP8_PER_GROUP128", "FN_MXFP4", "FN_ERR_INVALID",
                 "FN_ERR_ALIGN", "FN_ERR_UNSUPPORTED", "FN_ERR_CUDA", "FN_VARIANT_ROW_CTA",
                 "FN_VARIANT_ROW_CLUSTER", "FN_VARIANT_QUANT_ONLY", "FN_VARIANT_QK_WARP",
                 "FN_VARIANT_QK_WARP_FP8", "FN_VARIANT_ROW_ALLREDUCE", "FN_VARIANT_HC_MIX"):
        m = re.search(rf"\b{name}\s*=\s*(-?\d+)", src)
        assert m and int(m.group(1)) == getattr(fnb, name), name
    for name in ("FN_MAX_PARTS", "FN_MAX_H", "FN_MAX_HEAD_DIM"):
        m = re.search(rf"#define {name} (\d+)", src)
        assert int(m.group(1)) == getattr(fnb, name), name


def test_status_strings(fnb):
    assert fnb.fn_status_string(0) == "ok"
    for s in (-1, -2, -3, -4):
        assert fnb.fn_status_string(s) and fnb.fn_status_string(s) != "unknown status"
    assert fnb.fn_status_string(17) == "unknown status"
    assert fnb.fn_status_string(-5) == "unknown status"
    assert fnb.fn_version() >= 100


BASE = 0x7F0000000000


def rq(fnb, **kw):
    a = dict(x_parts=[BASE], num_parts=1, residual=BASE + (1 << 32), weight=BASE + (2 << 32),
             eps=1e-6, mode=0, M=4, H=256, out_q=BASE + (3 << 32), out_scale=BASE + (4 << 32),
             out_residual=BASE + (5 << 32), out_y=None, stream=None)
    a.update(kw)
    return fnb.fn_rmsnorm_quant(a["x_parts"], a["num_parts"], a["residual"], a["weight"],
                                a["eps"], a["mode"], a["M"], a["H"], a["out_q"], a["out_scale"],
                                a["out_residual"], a["out_y"], a["stream"])


def test_rmsnorm_quant_rejects_bad_arguments(fnb):
    E, A, U = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED
    cases = [
        (dict(num_parts=0), E), (dict(num_parts=9, x_parts=[BASE] * 9), E),
        (dict(mode=3), E), (dict(mode=-1), E), (dict(M=-1), E), (dict(H=0), E),
        (dict(H=12), E), (dict(mode=1, H=192), E), (dict(mode=2, H=48), E),
        (dict(H=32776), U), (dict(eps=float("nan")), E), (dict(eps=-1.0), E),
        (dict(weight=None), E), (dict(out_q=None), E), (dict(out_scale=None), E),
        (dict(out_residual=None), E), (dict(x_parts=[None]), E),
        (dict(x_parts=[BASE + 8]), A), (dict(weight=BASE + (2 << 32) + 2), A),
        (dict(out_q=BASE + (3 << 32) + 4), A), (dict(out_scale=BASE + (4 << 32) + 2), A),
        (dict(out_y=BASE + (6 << 32) + 8), A),
        # outputs overlapping inputs or each other
        (dict(out_q=BASE + 64), E), (dict(out_y=BASE + (1 << 32)), E),
        (dict(out_scale=BASE + (3 << 32) + 256), E),
        (dict(out_residual=BASE + (1 << 32) + 16), E),
    ]
    for kw, want in cases:
        assert rq(fnb, **kw) == want, kw
        assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE


def test_rmsnorm_quant_accepts_empty_and_in_place(fnb):
    assert rq(fnb, M=0) == fnb.FN_OK
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE
    # in-place residual is the one allowed overlap; mxfp4 codes need 4-byte alignment only
    assert rq(fnb, M=0, out_residual=BASE + (1 << 32)) == fnb.FN_OK
    assert rq(fnb, M=0, mode=2, out_q=BASE + (3 << 32) + 4, out_scale=BASE + (4 << 32) + 1) == 0
    assert rq(fnb, M=0, residual=None, out_residual=None) == fnb.FN_OK


def test_quant_rejects_bad_arguments(fnb):
    q = fnb.fn_quant
    assert q(BASE, 0, 0, 256, BASE + (1 << 32), BASE + (2 << 32), None) == fnb.FN_OK
    assert q(None, 0, 4, 256, BASE + (1 << 32), BASE + (2 << 32), None) == fnb.FN_ERR_INVALID
    assert q(BASE + 8, 0, 4, 256, BASE + (1 << 32), BASE + (2 << 32), None) == fnb.FN_ERR_ALIGN
    assert q(BASE, 1, 4, 64, BASE + (1 << 32), BASE + (2 << 32), None) == fnb.FN_ERR_INVALID
    assert q(BASE, 0, 4, 256, BASE + 512, BASE + (2 << 32), None) == fnb.FN_ERR_INVALID


def qk(fnb, **kw):
    a = dict(qkv=BASE, M=4, row_stride=18432, Hq=32, Hk=4, D=256, q_weight=BASE + (1 << 32),
             k_weight=BASE + (2 << 32), eps=1e-6, out_q=BASE + (3 << 32),
             out_k=BASE + (4 << 32), out_gate=BASE + (5 << 32), stream=None)
    a.update(kw)
    return fnb.fn_qk_norm_gate(a["qkv"], a["M"], a["row_stride"], a["Hq"], a["Hk"], a["D"],
                               a["q_weight"], a["k_weight"], a["eps"], a["out_q"], a["out_k"],
                               a["out_gate"], a["stream"])


def test_qk_norm_gate_rejects_bad_arguments(fnb):
    E, A, U = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED
    cases = [
        (dict(M=-1), E), (dict(D=12), E), (dict(D=0), E), (dict(D=2048, row_stride=1 << 20), U),
        (dict(row_stride=18436), E), (dict(row_stride=8192), E), (dict(Hq=0, Hk=0), E),
        (dict(q_weight=None), E), (dict(out_k=None), E), (dict(eps=float("inf")), E),
        (dict(qkv=BASE + 8), A), (dict(out_gate=BASE + (5 << 32) + 4), A),
        (dict(out_q=BASE + 1024), E), (dict(out_k=BASE + (3 << 32) + 16), E),
    ]
    for kw, want in cases:
        assert qk(fnb, **kw) == want, kw
    assert qk(fnb, M=0) == fnb.FN_OK
    assert qk(fnb, M=0, Hk=0, k_weight=None, out_k=None) == fnb.FN_OK


def test_prefer_variant_is_thread_local_and_returns_previous(fnb):
    import threading
    assert fnb.fn_prefer_variant(fnb.FN_VARIANT_ROW_CLUSTER) == fnb.FN_VARIANT_NONE
    seen = []
    th = threading.Thread(target=lambda: seen.append(fnb.fn_prefer_variant(0)))
    th.start()
    th.join()
    assert seen == [fnb.FN_VARIANT_NONE]
    assert fnb.fn_prefer_variant(fnb.FN_VARIANT_NONE) == fnb.FN_VARIANT_ROW_CLUSTER


def test_scale_layout_flags(fnb):
    E = fnb.FN_ERR_INVALID
    SW, MN = fnb.FN_SCALE_SWIZZLE_32_4_4, fnb.FN_SCALE_MN_MAJOR
    # each flag only with its mode, no unknown flags, no two flags
    assert rq(fnb, M=0, mode=fnb.FN_MXFP4 | SW) == fnb.FN_OK
    assert rq(fnb, M=0, mode=fnb.FN_FP8_PER_GROUP128 | MN) == fnb.FN_OK
    assert rq(fnb, M=0, mode=fnb.FN_FP8_PER_TOKEN | SW) == E
    assert rq(fnb, M=0, mode=fnb.FN_MXFP4 | MN) == E
    assert rq(fnb, M=0, mode=fnb.FN_MXFP4 | SW | MN) == E
    assert rq(fnb, M=0, mode=fnb.FN_MXFP4 | 0x400) == E
    # the padded scale buffer counts in the overlap check: M=4, H=256 swizzled
    # needs 128 * 8 bytes of scales, so codes 512 bytes after it overlap
    assert rq(fnb, mode=fnb.FN_MXFP4 | SW, out_q=BASE + (4 << 32) + 512) == E
    assert fnb.fn_quant(BASE, fnb.FN_FP8_PER_TOKEN | MN, 4, 256, BASE + (1 << 32),
                        BASE + (2 << 32), None) == E


def test_qk_fp8_rejects_bad_arguments(fnb):
    def q8(**kw):
        a = dict(qkv=BASE, M=4, row_stride=18432, Hq=32, Hk=4, D=256, qw=BASE + (1 << 32),
                 kw=BASE + (2 << 32), eps=1e-6, q8=BASE + (3 << 32), qs=BASE + (4 << 32),
                 k8=BASE + (5 << 32), ks=BASE + (6 << 32), g=BASE + (7 << 32), q=None, k=None)
        a.update(kw)
        return fnb.fn_qk_norm_gate_fp8(a["qkv"], a["M"], a["row_stride"], a["Hq"], a["Hk"],
                                       a["D"], a["qw"], a["kw"], a["eps"], a["q8"], a["qs"],
                                       a["k8"], a["ks"], a["g"], a["q"], a["k"], None)
    E, A = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN
    assert q8(M=0) == fnb.FN_OK
    assert q8(q8=None) == E and q8(ks=None) == E and q8(g=None) == E
    assert q8(q8=BASE + (3 << 32) + 4) == A and q8(qs=BASE + (4 << 32) + 2) == A
    assert q8(qs=BASE + (3 << 32) + 64) == E          # scales inside the q codes
    assert q8(k8=BASE + 100 * 2 * 256) == E           # codes inside qkv


def test_fp16_row_flag(fnb):
    """FN_IO_FP16 combines with every mode and layout flag; unknown bits next
    to it are still rejected; its value matches the header."""
    m = re.search(r"#define FN_IO_FP16 (0x[0-9A-Fa-f]+)", open(HEADER).read())
    assert m and int(m.group(1), 16) == fnb.FN_IO_FP16
    F = fnb.FN_IO_FP16
    for mode in (fnb.FN_FP8_PER_TOKEN, fnb.FN_FP8_PER_GROUP128, fnb.FN_MXFP4,
                 fnb.FN_MXFP4 | fnb.FN_SCALE_SWIZZLE_32_4_4,
                 fnb.FN_FP8_PER_GROUP128 | fnb.FN_SCALE_MN_MAJOR):
        assert rq(fnb, M=0, mode=mode | F) == fnb.FN_OK
        assert fnb.fn_quant(BASE, mode | F, 0, 256, BASE + (1 << 32), BASE + (2 << 32),
                            None) == fnb.FN_OK
    assert rq(fnb, M=0, mode=fnb.FN_MXFP4 | F | 0x2000) == fnb.FN_ERR_INVALID
    assert rq(fnb, M=0, mode=fnb.FN_FP8_PER_TOKEN | F | fnb.FN_SCALE_SWIZZLE_32_4_4) == \
        fnb.FN_ERR_INVALID
    # the same argument checks apply (here: H not a multiple of 8)
    assert rq(fnb, mode=fnb.FN_MXFP4 | F, H=12) == fnb.FN_ERR_INVALID


def test_programmatic_launch_is_thread_local_and_returns_previous(fnb):
    import threading
    assert fnb.fn_programmatic_launch(1) == 0
    seen = []
    t = threading.Thread(target=lambda: seen.append(fnb.fn_programmatic_launch(0)))
    t.start()
    t.join()
    assert seen == [0]
    with fnb.programmatic_launch(False):
        assert fnb.fn_programmatic_launch(0) == 0
    assert fnb.fn_programmatic_launch(0) == 1


def ar(fnb, n=2, rank=0, **kw):
    """fn_ar_rmsnorm_quant on fake, disjoint addresses (rank d's buffers at
    BASE + d << 40); a rejected call never touches them."""
    a = dict(x_parts=[BASE + (d << 40) for d in range(n)], num_ranks=n, rank=rank,
             residual=BASE + (1 << 32), weight=BASE + (2 << 32), eps=1e-6, mode=2, M=4, H=256,
             out_q=[BASE + (d << 40) + (3 << 32) for d in range(n)],
             out_scale=[BASE + (d << 40) + (4 << 32) for d in range(n)],
             out_residual=[BASE + (d << 40) + (5 << 32) for d in range(n)], out_y=None,
             stream=None)
    a.update(kw)
    return fnb.fn_ar_rmsnorm_quant(a["x_parts"], a["num_ranks"], a["rank"], a["residual"],
                                   a["weight"], a["eps"], a["mode"], a["M"], a["H"], a["out_q"],
                                   a["out_scale"], a["out_residual"], a["out_y"], a["stream"])


def test_allreduce_rejects_bad_arguments(fnb):
    E, A, U = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED
    for kw, want in [
        (dict(n=1), E), (dict(n=9), E), (dict(rank=2), E), (dict(rank=-1), E),
        (dict(mode=3), E), (dict(H=12), E), (dict(mode=1, H=192), E), (dict(eps=-1.0), E),
        (dict(mode=2 | fnb.FN_IO_FP16), U), (dict(weight=None), E),
        (dict(out_residual=None), E),  # a residual needs residual_out on every rank
        (dict(x_parts=[BASE, None]), E), (dict(x_parts=[BASE, BASE + 8]), A),
        (dict(out_q=[BASE + (3 << 32), BASE + (3 << 32)]), E),  # two ranks' codes overlap
        (dict(out_q=[BASE + (3 << 32) + 2, BASE + (1 << 40) + (3 << 32)]), A),
        # another rank's residual_out on this rank's residual: only the own entry may alias
        (dict(out_residual=[BASE + (5 << 32), BASE + (1 << 32)]), E),
        (dict(out_q=[BASE, BASE + (1 << 40) + (3 << 32)]), E),  # codes over a partial
    ]:
        n = kw.pop("n", 2)
        assert ar(fnb, n=n, **kw) == want, (kw, n)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE


def test_allreduce_empty_shard_and_in_place(fnb):
    # M=1 over 2 ranks: rank 0's shard is empty, nothing is launched
    assert ar(fnb, rank=0, M=1) == fnb.FN_OK
    assert ar(fnb, M=0) == fnb.FN_OK
    # in place on the own replica passes every check and reaches the launch,
    # which fails here for want of a device
    assert ar(fnb, out_residual=[BASE + (1 << 32), BASE + (1 << 40) + (5 << 32)]) == \
        fnb.FN_ERR_CUDA


def hc(fnb, **kw):
    a = dict(x=BASE, w_down=BASE + (1 << 32), w_up=BASE + (2 << 32), M=4, hc=4, C=2560, r=64,
             out=BASE + (3 << 32), workspace=BASE + (4 << 32), stream=None)
    a.update(kw)
    return fnb.fn_hc_mix(a["x"], a["w_down"], a["w_up"], a["M"], a["hc"], a["C"], a["r"],
                         a["out"], a["workspace"], a["stream"])


def test_hc_mix_rejects_bad_arguments(fnb):
    """Every rule of fn_hc_mix's contract is checked on the host before any
    launch (the pointers here are never dereferenced)."""
    E, A, U = fnb.FN_ERR_INVALID, fnb.FN_ERR_ALIGN, fnb.FN_ERR_UNSUPPORTED
    cases = [
        (dict(M=-1), E), (dict(C=0), E), (dict(r=0), E), (dict(hc=0), E),
        (dict(M=17), U), (dict(hc=2), U), (dict(C=2568), U), (dict(C=4112), U),
        (dict(r=12), U), (dict(r=136), U),
        (dict(x=None), E), (dict(w_down=None), E), (dict(w_up=None), E), (dict(out=None), E),
        (dict(workspace=None), E),
        (dict(x=BASE + 8), A), (dict(w_up=BASE + (2 << 32) + 2), A),
        (dict(out=BASE + (3 << 32) + 4), A), (dict(workspace=BASE + (4 << 32) + 8), A),
        # outputs overlapping the inputs or each other
        (dict(out=BASE + 4096), E), (dict(workspace=BASE + (1 << 32) + 64), E),
        (dict(workspace=BASE + (3 << 32) + 32), E),
    ]
    for kw, want in cases:
        assert hc(fnb, **kw) == want, kw
        assert fnb.fn_last_variant() == fnb.FN_VARIANT_NONE
    assert hc(fnb, M=0) == fnb.FN_OK
    assert hc(fnb, M=0, x=None, out=None, workspace=None) == fnb.FN_OK
    assert fnb.fn_hc_mix_workspace_bytes(16, 64) == 16 * 64 * 4
    assert fnb.fn_hc_mix_workspace_bytes(0, 64) == 0
    assert fnb.fn_hc_mix_workspace_bytes(-1, 64) == -1 and fnb.fn_hc_mix_workspace_bytes(4, 0) == -1
