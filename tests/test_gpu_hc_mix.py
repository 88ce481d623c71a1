"""hc_mix (the low-rank gate over the hyper-state) on the GPU against the
float64 oracle.

Criteria, per output element, with u the oracle's float64 value
(tests/parity.py, check_hc_mix; its negative controls run on the CPU):
  the page's:   |gpu - u| <= 4e-3 + 1e-2 |u|   (sglang PR #41880, "Accuracy
                Tests": the float64 reference at atol 4e-3, rtol 1e-2);
  derived:      |gpu - u| <= 2^-8 |u| + 2e-5    (the one bf16 rounding, at most
                half an ulp: 8 significant bits, so 2^-8 relative; plus the
                fp32 path: products of bf16 are exact, the gate logits take t
                as three bf16 parts exact to 2^-24, sums of 10240 terms of
                ~1e-2 and of 64 terms of ~1e-1 in fp32 carry ~1e-6 absolute,
                the sigmoid ~1e-7, bounded here with margin by 2e-5).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_quantization_b200 import synth
from tests import gpu_util, parity

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module")
def fnb():
    return gpu_util.lib()


def bf16_vals(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def run(fnb, wl, M=None, workspace=None, out=None):
    inp = wl.inputs(device="cpu", M=M)
    x, wd, wu = (inp[k].cuda() for k in ("x", "w_down", "w_up"))
    M = x.shape[0]
    go = gpu_util.Guarded((M, wl.C), torch.bfloat16) if out is None else None
    gw = gpu_util.Guarded((max(1, M * wl.r),), torch.float32) if workspace is None else None
    o = fnb.hc_mix(x, wd, wu, hc=wl.hc, out=go.t if go else out,
                   workspace=gw.t if gw else workspace)
    launch = fnb.fn_last_launch()
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_HC_MIX
    torch.cuda.synchronize()
    for g in (go, gw):
        assert g is None or g.intact(), "write outside an output"
    return inp, gpu_util.bits(o), launch


def check(wl, inp, got_bits, logit_scale=1.0):
    """Both criteria; the fp32 term of the derived bound grows with the size
    of the logits (`logit_scale` times the unit-variance recipe)."""
    u, ub = oracle.hc_mix(gpu_util.bits(inp["x"]), gpu_util.bits(inp["w_down"]),
                          gpu_util.bits(inp["w_up"]), wl.hc, wl.C, wl.r)
    return parity.check_hc_mix(u, ub, got_bits, logit_scale)


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_workload_every_decode_m(fnb, M):
    """The workload's shape (hc = 4, C = 2560, rank 64) at every M <= 16."""
    wl = synth.hc_mix(M)
    inp, got, launch = run(fnb, wl)
    st = check(wl, inp, got)
    # 16 clusters of 8 blocks (4 weight rows of W_down each; 160 threads per
    # row group of at most 4 rows, for M padded to 1, 2, 4, 8 or 16), then 128
    # gate-and-mix blocks of 20 channels (a warp per 8 of their 80 W_up rows)
    mm = next(b for b in (1, 2, 4, 8, 16) if b >= M)
    assert list(launch) == [128, 160 * max(1, mm // 4), 128, 320], launch
    assert st["bf16_equal_frac"] > 0.99, st


SHAPES = [  # (M, C, r): ranks 8..128, C from one block of channels to the largest
    (1, 16, 8), (3, 32, 16), (5, 64, 24), (16, 16, 128), (2, 1024, 32), (7, 4096, 64),
    (16, 4096, 128), (9, 2560, 40), (4, 48, 56), (12, 512, 8), (16, 2560, 128),
    (3, 2384, 64),  # 2384 = 16 * 149: no divisor of C in steps of 4 keeps blocks <= SMs
]


@pytest.mark.parametrize("M,C,r", SHAPES, ids=[f"M{s[0]}_C{s[1]}_r{s[2]}" for s in SHAPES])
def test_shapes(fnb, M, C, r):
    wl = synth.HCWorkload("shape", M=M, C=C, r=r, seed=M * 7 + C + r)
    inp, got, _ = run(fnb, wl)
    check(wl, inp, got)


def test_saturated_and_balanced_gates(fnb):
    """Logits far out on both sides (gates at 0 and 1 within fp32) and exactly
    zero (zero up-factor: every gate 1/2, u = sum of the streams / 2)."""
    wl = synth.HCWorkload("sat", M=6, C=256, r=32, seed=3)
    inp = wl.inputs(device="cpu")
    big = dict(inp, w_up=(inp["w_up"].float() * 60).to(torch.bfloat16))
    _, got, _ = run_inputs(fnb, wl, big)
    check(wl, big, got, logit_scale=60.0)
    zero = dict(inp, w_up=torch.zeros_like(inp["w_up"]))
    _, got, _ = run_inputs(fnb, wl, zero)
    check(wl, zero, got)
    # the kernel's order: u = fl(u + x_s / 2) for s = 0..3 (every product exact)
    xv = bf16_vals(gpu_util.bits(inp["x"])).astype(np.float32).reshape(wl.M, wl.hc, wl.C)
    u = np.zeros((wl.M, wl.C), dtype=np.float32)
    for s in range(wl.hc):
        u = (u + np.float32(0.5) * xv[:, s, :]).astype(np.float32)
    want = gpu_util.bits(torch.from_numpy(u).to(torch.bfloat16))
    assert np.array_equal(got, want)


def run_inputs(fnb, wl, inp):
    x, wd, wu = (inp[k].cuda() for k in ("x", "w_down", "w_up"))
    o = fnb.hc_mix(x, wd, wu, hc=wl.hc)
    torch.cuda.synchronize()
    return inp, gpu_util.bits(o), fnb.fn_last_launch()


def test_replays_and_graph_are_bit_identical(fnb):
    """Repeated calls, a CUDA graph of calls and a chain of programmatic
    launches all give the first call's bits."""
    wl = synth.hc_mix(16)
    inp = wl.inputs(device="cuda")
    x, wd, wu = inp["x"], inp["w_down"], inp["w_up"]
    ref = fnb.hc_mix(x, wd, wu).clone()
    outs = [fnb.hc_mix(x, wd, wu) for _ in range(5)]
    with fnb.programmatic_launch(True):
        outs += [fnb.hc_mix(x, wd, wu) for _ in range(5)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ws = torch.empty(wl.M * wl.r, dtype=torch.float32, device="cuda")
        gout = [torch.empty((wl.M, wl.C), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
        g = torch.cuda.CUDAGraph()
        with fnb.programmatic_launch(True):
            with torch.cuda.graph(g, stream=s):
                for o in gout:
                    fnb.hc_mix(x, wd, wu, out=o, workspace=ws)
        g.replay()
        g.replay()
    torch.cuda.synchronize()
    for o in outs + gout:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))


def test_consecutive_calls_share_a_workspace(fnb):
    """Calls on one stream that share one workspace and feed each other (the
    output of one becomes stream 0 of the next row set) match the oracle run
    on the same chain: each call's second kernel reads the t its own first
    kernel wrote."""
    wl = synth.HCWorkload("chain", M=4, C=512, r=32, seed=8)
    inp = wl.inputs(device="cuda")
    x, wd, wu = inp["x"].clone(), inp["w_down"], inp["w_up"]
    ws = torch.empty(wl.M * wl.r, dtype=torch.float32, device="cuda")
    xs, outs = [], []
    for i in range(4):
        xs.append(x.clone())
        o = fnb.hc_mix(x, wd, wu, workspace=ws)
        outs.append(o)
        x = x.clone()
        x[:, :wl.C] = o
    torch.cuda.synchronize()
    for xi, o in zip(xs, outs):
        check(wl, {"x": xi.cpu(), "w_down": wd.cpu(), "w_up": wu.cpu()}, gpu_util.bits(o))


def test_rejected_calls_touch_nothing(fnb):
    wl = synth.hc_mix(4)
    inp = wl.inputs(device="cuda")
    go = gpu_util.Guarded((4, wl.C), torch.bfloat16)
    gw = gpu_util.Guarded((4 * wl.r,), torch.float32)
    args = [inp["x"].data_ptr(), inp["w_down"].data_ptr(), inp["w_up"].data_ptr()]
    st = fnb.fn_hc_mix(*args, 17, 4, wl.C, wl.r, go.t.data_ptr(), gw.t.data_ptr(), None)
    assert st == fnb.FN_ERR_UNSUPPORTED
    st = fnb.fn_hc_mix(*args, 4, 4, wl.C, wl.r, go.t.data_ptr() + 2, gw.t.data_ptr(), None)
    assert st == fnb.FN_ERR_ALIGN
    st = fnb.fn_hc_mix(*args, 4, 4, wl.C, wl.r, go.t.data_ptr(), go.t.data_ptr() + 64, None)
    assert st == fnb.FN_ERR_INVALID
    # the tensor API refuses a workspace smaller than fn_hc_mix_workspace_bytes
    with pytest.raises(ValueError):
        fnb.hc_mix(inp["x"], inp["w_down"], inp["w_up"], out=go.t, workspace=gw.t[:-1])
    torch.cuda.synchronize()
    assert go.untouched() and gw.untouched()
