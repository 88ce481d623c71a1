"""Negative controls for the parity harness (tests/parity.py), on the CPU.

The GPU parity tests are only as good as the comparison they run.  Here the
oracle's own outputs stand in for a kernel's: unchanged they must pass, and
each planted fault — one flipped code bit, a wrong scale, y off by two ulps,
a residual off by one ulp, a code two steps away, a code that moved where y
did not — must make the comparison fail."""
import numpy as np
import pytest

import oracle
from mxfp4_quantization_b200 import synth
from tests import parity


def _case(mode, seed=5, M=12, H=1024, P=2, io=oracle.IO_BF16):
    import torch
    wl = synth.RowWorkload("ctl", M=M, H=H, P=P, mode=mode, eps=1e-6, seed=seed,
                           outlier_frac=0.01,
                           dtype=torch.float16 if io == oracle.IO_FP16 else torch.bfloat16)
    inp = wl.inputs(device="cpu")
    parts = [synth.to_bits(p) for p in inp["parts"]]
    res, w = synth.to_bits(inp["residual"]), synth.to_bits(inp["weight"])
    orc = oracle.rmsnorm_quant(parts, res, w, wl.eps, mode, io=io)
    gpu = {"q": orc["q"].copy(), "scale": orc["scale"].copy(),
           "residual_out": orc["residual_out"].copy(), "y": orc["y"].copy()}
    return wl, parts, res, w, gpu


def _check(wl, parts, res, w, gpu, io=oracle.IO_BF16):
    return parity.check_rmsnorm(wl.mode, wl.eps, parts, res, w, gpu, io)


MODES = [oracle.FP8_PER_TOKEN, oracle.FP8_PER_GROUP128, oracle.MXFP4]


@pytest.mark.parametrize("io", [oracle.IO_BF16, oracle.IO_FP16])
@pytest.mark.parametrize("mode", MODES)
def test_exact_outputs_pass(mode, io):
    wl, parts, res, w, gpu = _case(mode, io=io)
    stats = _check(wl, parts, res, w, gpu, io)
    assert stats["codes_diff"] == 0 and stats["scale_diff"] == 0


@pytest.mark.parametrize("mode", MODES)
def test_flipped_code_bit_fails(mode):
    wl, parts, res, w, gpu = _case(mode)
    gpu["q"][3, 17] ^= 0x01
    with pytest.raises(AssertionError):
        _check(wl, parts, res, w, gpu)


@pytest.mark.parametrize("mode", MODES)
def test_wrong_scale_fails(mode):
    wl, parts, res, w, gpu = _case(mode)
    s = gpu["scale"].reshape(wl.M, -1)
    if mode == oracle.MXFP4:
        s[2, 1] = s[2, 1] + 1
    else:
        s[2, 0] = np.float32(s[2, 0]) * np.float32(1.0 + 2 ** -20)
    with pytest.raises(AssertionError):
        _check(wl, parts, res, w, gpu)


def test_y_two_ulps_off_fails():
    wl, parts, res, w, gpu = _case(oracle.MXFP4)
    y = gpu["y"]
    i = int(np.argmax((y & 0x7FFF) > 0x3000))  # a normal, nonzero element of row 0
    y[0, i] = y[0, i] + 2
    with pytest.raises(AssertionError):
        _check(wl, parts, res, w, gpu)


def test_residual_one_ulp_off_fails():
    wl, parts, res, w, gpu = _case(oracle.FP8_PER_TOKEN)
    gpu["residual_out"][5, 9] += 1
    with pytest.raises(AssertionError):
        _check(wl, parts, res, w, gpu)


def test_code_two_steps_away_fails_end_to_end():
    """A kernel whose y moved by one ulp but whose code moved by two steps."""
    wl, parts, res, w, gpu = _case(oracle.FP8_PER_GROUP128)
    orc = oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)
    q, y = gpu["q"], gpu["y"]
    j = 40
    y[1, j] += 1
    q[1, j] = (q[1, j] & 0x80) | ((q[1, j] & 0x7F) + 2)
    with pytest.raises(AssertionError):
        parity.compare_end_to_end(wl.mode, wl.H, y, q, gpu["scale"], orc["y"], orc["q"],
                                  orc["scale"])


def test_code_moved_where_y_did_not_fails_end_to_end():
    wl, parts, res, w, gpu = _case(oracle.MXFP4)
    orc = oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)
    q = gpu["q"]
    lo = q[4, 3] & 0x0F
    q[4, 3] = (q[4, 3] & 0xF0) | ((lo & 0x8) | min((lo & 0x7) + 1, 7) if (lo & 0x7) < 7
                                  else (lo & 0x8) | 6)
    with pytest.raises(AssertionError):
        parity.compare_end_to_end(wl.mode, wl.H, gpu["y"], q, gpu["scale"], orc["y"], orc["q"],
                                  orc["scale"])


def test_all_rows_runner_passes_exact_and_catches_a_fault_in_a_late_chunk():
    """The row-parallel runner of the full-size tests (spawned processes over
    chunks of rows) sums the statistics of every chunk, and a fault planted in
    the last chunk only still fails the comparison."""
    wl, parts, res, w, gpu = _case(oracle.FP8_PER_GROUP128, M=70, H=1024)
    st = parity.check_rmsnorm_all_rows(wl.mode, wl.eps, parts, res, w, gpu, chunk=16, procs=3)
    assert st["rows"] == 70 and st["codes"] == 70 * 1024 and st["codes_diff"] == 0
    assert st["groups"] == 70 * 8
    gpu["q"][69, 5] ^= 0x01
    with pytest.raises(AssertionError):
        parity.check_rmsnorm_all_rows(wl.mode, wl.eps, parts, res, w, gpu, chunk=16, procs=3)


# ---- hc_mix ------------------------------------------------------------------------
#
# The criterion of the hc_mix GPU tests (parity.check_hc_mix) must pass the
# oracle's own bf16 result and fail a kernel that made any of the plausible
# mistakes below.  A mistaken kernel is stood in for by a copy of the oracle
# with the mistake planted (built on the CPU, as the oracle's own negative
# controls do), run on the same inputs at the workload's shape.

HC_FAULTS = [
    ("gate_sign", "g[e] = 1.0 / (1.0 + exp(-z));", "g[e] = 1.0 / (1.0 + exp(z));"),
    ("last_stream_dropped", "for (int s = 0; s < hc; ++s)", "for (int s = 0; s < hc - 1; ++s)"),
    ("w_up_transposed", "z += t[j] * orc_bf16_to_double(w_up[e * r + j]);",
     "z += t[j] * orc_bf16_to_double(w_up[(int64_t)j * K + e]);"),
    # the rounding that the gate kernel's three-part split of t avoids
    ("t_rounded_to_bf16", "t[j] = acc;", "t[j] = orc_bf16_to_double(orc_bf16_from_double(acc));"),
]


def _hc_case(M=4, C=512, r=64, seed=21):
    wl = synth.HCWorkload("ctl", M=M, C=C, r=r, seed=seed)
    inp = wl.inputs(device="cpu")
    bits = {k: synth.to_bits(inp[k]) for k in ("x", "w_down", "w_up")}
    u, ub = oracle.hc_mix(bits["x"], bits["w_down"], bits["w_up"], wl.hc, wl.C, wl.r)
    return wl, bits, u, ub


def test_hc_exact_outputs_pass():
    _, _, u, ub = _hc_case()
    st = parity.check_hc_mix(u, ub, ub)
    assert st["bf16_equal_frac"] == 1.0


def test_hc_two_ulps_off_fails():
    _, _, u, ub = _hc_case()
    bad = ub.copy()
    i = np.unravel_index(np.argmax(np.abs(u)), u.shape)
    bad[i] = np.uint16(int(bad[i]) + 2)
    with pytest.raises(AssertionError):
        parity.check_hc_mix(u, ub, bad)


@pytest.mark.parametrize("name,old,new", HC_FAULTS, ids=[f[0] for f in HC_FAULTS])
def test_hc_planted_mistake_fails(tmp_path, name, old, new):
    import os
    from oracle.build import SRC, build_oracle
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} missing"
    mut = os.path.join(tmp_path, "orc_fault.c")
    with open(mut, "w") as fh:
        fh.write(src.replace(old, new))
    lib = oracle.load(build_oracle(src=mut, out=os.path.join(tmp_path, "liborc_fault.so"),
                                   extra_flags=("-Wno-error",), force=True))
    wl, bits, u, ub = _hc_case()
    _, wrong = oracle.hc_mix(bits["x"], bits["w_down"], bits["w_up"], wl.hc, wl.C, wl.r, lib=lib)
    with pytest.raises(AssertionError):
        parity.check_hc_mix(u, ub, wrong)
