"""QK Gemma-RMSNorm + gate extraction on the GPU against the oracle: q and k
within 1 bf16 ulp, gate bit-exact, nothing read past the k heads."""
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


def check_qk(fnb, M, Hq, Hk, D, stride, seed, eps=1e-6, poison_tail=True):
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn((M, stride), generator=g).to(torch.bfloat16)
    if poison_tail:  # v heads and padding: NaN, must not leak into any output
        qkv[:, (2 * Hq + Hk) * D:] = float("nan")
    qw = (0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16)
    kw = (0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16)
    dev = qkv.cuda()
    outs = [gpu_util.Guarded(s, torch.bfloat16) for s in ((M, Hq, D), (M, Hk, D), (M, Hq, D))]
    o = fnb.qk_norm_gate(dev, Hq, Hk, D, qw.cuda(), kw.cuda(), eps,
                         out=fnb.QKOutput(*[x.t for x in outs]))
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_QK_WARP
    torch.cuda.synchronize()
    assert all(x.intact() for x in outs), "write outside an output"
    ref = oracle.qk_norm_gate(gpu_util.bits(qkv), stride, Hq, Hk, D, gpu_util.bits(qw),
                              gpu_util.bits(kw), eps)
    gq, gk, gg = gpu_util.bits(o.q), gpu_util.bits(o.k), gpu_util.bits(o.gate)
    assert np.array_equal(gg, ref["gate"]), "gate is not a bit copy"
    for name, a, b in (("q", gq, ref["q"]), ("k", gk, ref["k"])):
        d = parity.ulp_diff(a, b)
        assert d.max(initial=0) <= 1, f"{name} differs by {d.max()} ulp"
    return o


@pytest.mark.parametrize("M", synth.QK_M)
def test_qk_prologue_config(fnb, M):
    wl = synth.qk_prologue(M)
    inp = wl.inputs(device="cpu")
    dev = inp["qkv"].cuda()
    o = fnb.qk_norm_gate(dev, wl.Hq, wl.Hk, wl.D, inp["q_weight"].cuda(),
                         inp["k_weight"].cuda(), wl.eps)
    torch.cuda.synchronize()
    ref = oracle.qk_norm_gate(gpu_util.bits(inp["qkv"]), wl.row_stride, wl.Hq, wl.Hk, wl.D,
                              gpu_util.bits(inp["q_weight"]), gpu_util.bits(inp["k_weight"]),
                              wl.eps)
    assert np.array_equal(gpu_util.bits(o.gate), ref["gate"])
    assert parity.ulp_diff(gpu_util.bits(o.q), ref["q"]).max() <= 1
    assert parity.ulp_diff(gpu_util.bits(o.k), ref["k"]).max() <= 1


@pytest.mark.parametrize("M,Hq,Hk,D,pad", [
    (4, 32, 4, 256, 4 * 256), (64, 32, 4, 256, 4 * 256), (3, 2, 1, 8, 8), (5, 3, 2, 64, 24),
    (7, 8, 2, 128, 0), (2, 4, 4, 512, 64), (3, 2, 2, 1024, 8), (9, 5, 0, 256, 0),
    (6, 0, 3, 256, 16), (1000, 4, 1, 256, 256), (2, 3, 1, 264, 40),
])
def test_qk_shapes(fnb, M, Hq, Hk, D, pad):
    check_qk(fnb, M, Hq, Hk, D, (2 * Hq + Hk) * D + pad, seed=M + Hq + D)


def test_qk_empty(fnb):
    z = torch.zeros((0, 18432), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(256, dtype=torch.bfloat16, device="cuda")
    o = fnb.qk_norm_gate(z, 32, 4, 256, w, w, 1e-6)
    assert o.q.shape == (0, 32, 256) and fnb.fn_last_variant() == fnb.FN_VARIANT_NONE


@pytest.mark.parametrize("M,Hq,Hk,D", [(4, 32, 4, 256), (64, 32, 4, 256), (5, 3, 2, 64),
                                       (3, 2, 2, 1024), (9, 5, 0, 256), (6, 0, 3, 256),
                                       (700, 4, 1, 264)])
def test_qk_fp8_epilogue(fnb, M, Hq, Hk, D):
    """E4M3 q and k with one scale per (token, head): the quantization of the
    GPU's own normed heads is bit-exact against the oracle, the end-to-end
    codes meet the criterion of the row kernels, gate and bf16 heads as in the
    bf16 prologue, and the codes do not depend on whether bf16 heads are asked
    for."""
    stride = (2 * Hq + 2 * Hk) * D + 16
    g = torch.Generator().manual_seed(M * 7 + D)
    qkv = (torch.randn((M, stride), generator=g) *
           torch.pow(10.0, torch.rand((M, 1), generator=g) * 3 - 1.5)).to(torch.bfloat16)
    qkv[:, (2 * Hq + Hk) * D:] = float("nan")
    qw = (0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16)
    kw = (0.1 * torch.randn((D,), generator=g)).to(torch.bfloat16)
    dev, qwd, kwd = qkv.cuda(), qw.cuda(), kw.cuda()
    o = fnb.qk_norm_gate_fp8(dev, Hq, Hk, D, qwd, kwd, 1e-6, emit_bf16=True)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_QK_WARP_FP8
    o2 = fnb.qk_norm_gate_fp8(dev, Hq, Hk, D, qwd, kwd, 1e-6, emit_bf16=False)
    torch.cuda.synchronize()
    ref = oracle.qk_norm_gate_fp8(gpu_util.bits(qkv), stride, Hq, Hk, D, gpu_util.bits(qw),
                                  gpu_util.bits(kw), 1e-6)
    assert np.array_equal(gpu_util.bits(o.gate), ref["gate"])
    for name, H in (("q", Hq), ("k", Hk)):
        if H == 0:
            continue
        y = gpu_util.bits(getattr(o, name)).reshape(M * H, D)
        assert parity.ulp_diff(y, ref[name].reshape(M * H, D)).max() <= 1
        codes = gpu_util.u8(getattr(o, name + "8")).reshape(M * H, D)
        scales = getattr(o, name + "_scale").cpu().numpy().reshape(M * H)
        assert torch.equal(getattr(o, name + "8").view(torch.uint8),
                           getattr(o2, name + "8").view(torch.uint8))
        parity.compare_quant_stage(y, codes, scales, oracle.FP8_PER_TOKEN)
        parity.compare_end_to_end(oracle.FP8_PER_TOKEN, D, y, codes, scales,
                                  ref[name].reshape(M * H, D), ref[name + "8"].reshape(M * H, D),
                                  ref[name + "s"].reshape(M * H))
