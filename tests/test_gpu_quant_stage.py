"""fn_quant (the quantization stage alone) against the oracle, bit for bit,
over every finite bf16 value and the rounding corner cases of E4M3 / E2M1 /
E8M0.  The fused kernel runs the same device code for its quantization stage."""
import os

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util, parity
from tests.oracle_pins import all_finite_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fnb():
    return gpu_util.lib()


def exhaustive_rows(H, seed):
    """All finite bf16 patterns, shuffled into rows of H, plus corner rows."""
    b, _ = all_finite_bf16()
    rng = np.random.default_rng(seed)
    shuffled = rng.permutation(b)
    sorted_runs = np.sort(b)  # consecutive patterns share a group: many near-ties
    rows = [shuffled, sorted_runs]
    # MX tie blocks: amax 5 * 2^k puts the E2M1 midpoints at 0.25..5 * 2^k
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5,
                     -3.5, -5.0, 0.1, -0.1, 6.0, 7.0, -7.5, 0.0], dtype=np.float64)
    tie_blocks = []
    for k in range(-124, 124, 3):
        blk = np.zeros(32)
        blk[:ties.size] = ties * 2.0 ** k
        tie_blocks.append(blk)
    tb = torch.from_numpy(np.concatenate(tie_blocks).astype(np.float32)).to(torch.bfloat16)
    rows.append(tb.view(torch.int16).numpy().view(np.uint16))
    rows.append(np.zeros(H * 2, dtype=np.uint16))                    # zero groups
    rows.append(np.full(H, 0x8000, dtype=np.uint16))                 # -0 everywhere
    rows.append(rng.integers(1, 0x80, H * 2).astype(np.uint16))      # subnormals only
    rows.append((rng.integers(1, 0x80, H) | 0x8000).astype(np.uint16))
    flat = np.concatenate(rows)
    pad = (-flat.size) % H
    flat = np.concatenate([flat, np.zeros(pad, dtype=np.uint16)])
    return flat.reshape(-1, H)


@pytest.mark.parametrize("mode", [oracle.FP8_PER_TOKEN, oracle.FP8_PER_GROUP128, oracle.MXFP4])
@pytest.mark.parametrize("H", [128, 4096])
def test_quant_stage_exhaustive(fnb, mode, H):
    y = exhaustive_rows(H, seed=H + mode)
    yt = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).cuda()
    M = y.shape[0]
    q_shape = (M, H // 2) if mode == oracle.MXFP4 else (M, H)
    s_shape = oracle.scale_shape(mode, M, H)
    gq = gpu_util.Guarded(q_shape, torch.uint8)
    gs = gpu_util.Guarded(s_shape, torch.uint8 if mode == oracle.MXFP4 else torch.float32)
    fnb.quant(yt, mode, out_q=gq.t, out_scale=gs.t)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_QUANT_ONLY
    torch.cuda.synchronize()
    assert gq.intact() and gs.intact(), "write outside an output"
    parity.compare_quant_stage(y, gpu_util.u8(gq.t), gpu_util.scale_np(gs.t, mode), mode)


def test_negative_tiny_values_keep_their_sign(fnb):
    """A negative value that rounds to zero gives the -0 code (0x80 / 0x8)."""
    y = np.zeros((1, 128), dtype=np.float32)
    y[0, 0] = 448.0
    y[0, 1:8] = -1e-6
    y[0, 8] = -0.0
    yb = torch.from_numpy(y).to(torch.bfloat16)
    yt = yb.cuda()
    for mode in (oracle.FP8_PER_GROUP128, oracle.MXFP4):
        q, s = fnb.quant(yt, mode)
        torch.cuda.synchronize()
        parity.compare_quant_stage(gpu_util.bits(yb), gpu_util.u8(q), gpu_util.scale_np(s, mode),
                                   mode)
    q, _ = fnb.quant(yt, oracle.FP8_PER_GROUP128)
    assert np.all(gpu_util.u8(q)[0, 1:9] == 0x80)


@pytest.mark.parametrize("mode", [oracle.FP8_PER_TOKEN, oracle.FP8_PER_GROUP128, oracle.MXFP4])
def test_quant_stage_random_scales(fnb, mode):
    """Many groups, each with its own magnitude 2^U(-130, 120): the FP8
    quotient's fast path (reciprocal multiply) and its exact fallbacks
    (near-midpoint, E4M3-subnormal, tiny scale) all against IEEE division."""
    g = torch.Generator().manual_seed(77 + mode)
    M, H = 4096, 1024
    mag = torch.pow(2.0, torch.randint(-130, 120, (M, H // 128, 1), generator=g).float())
    y = (torch.randn((M, H // 128, 128), generator=g) * mag).reshape(M, H)
    y[::7, 5] = 0.0
    y[::11, 9] = -0.0
    yb = y.to(torch.bfloat16)
    q, s = fnb.quant(yb.cuda(), mode)
    torch.cuda.synchronize()
    parity.compare_quant_stage(gpu_util.bits(yb), gpu_util.u8(q), gpu_util.scale_np(s, mode), mode)


def test_scale_and_reciprocal_arithmetic_exhaustive(tmp_path):
    """The kernels' FP8 scale (division-free) equals CUDA's IEEE quotient, and
    their reciprocal is CUDA's IEEE reciprocal or one ulp below it and never
    above 1/s, for every positive finite bf16 and binary16 amax
    (tests/recip_check.cu)."""
    import subprocess
    here = os.path.dirname(os.path.abspath(__file__))
    csrc = os.path.join(os.path.dirname(here), "mxfp4_quantization_b200", "csrc")
    exe = os.path.join(tmp_path, "recip_check")
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-I", csrc, "-o", exe,
                    os.path.join(here, "recip_check.cu")], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("scale mismatches 0") == 2 and r.stdout.count("bad reciprocals 0") == 2
