"""Scale layouts for the GEMM that consumes the quantized tuple.

The kernels' scales in the 32x4x4 swizzled (MXFP4) and M-major (FP8
per-group-128) layouts against the oracle's row-major scales placed by
oracle.place_scales (pinned against a library's implementation of the
layout); padding stays untouched.  Then the layout is handed to B200's
block-scaled GEMM (torch.nn.functional.scaled_mm, cuBLASLt underneath) as its
consumer: activations quantized by the fused kernel, weights by fn_quant, and
the product must match the product of the dequantized operands (with a
bf16 output: this torch build's fp32 output of that GEMM is not usable).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_quantization_b200 import synth
from tests import gpu_util, parity

pytestmark = pytest.mark.gpu

MX, G128 = synth.MXFP4, synth.FP8_PER_GROUP128


@pytest.fixture(scope="module")
def fnb():
    return gpu_util.lib()


@pytest.mark.parametrize("variant", [0, 1, 2])
@pytest.mark.parametrize("mode,M,H", [(MX, 5, 7168), (MX, 130, 1024), (MX, 300, 224 * 32),
                                      (G128, 7, 8192), (G128, 129, 1024), (G128, 301, 2048)])
def test_layout_matches_oracle(fnb, mode, M, H, variant):
    flag = fnb.FN_SCALE_SWIZZLE_32_4_4 if mode == MX else fnb.FN_SCALE_MN_MAJOR
    wl = synth.RowWorkload("layout", M=M, H=H, P=2, mode=mode, eps=1e-6, seed=M + H)
    inp = wl.inputs(device="cpu")
    q, s = fnb.alloc_outputs(mode | flag, M, H, "cuda")
    with fnb.prefer_variant(variant):
        out = fnb.rmsnorm_quant([p.cuda() for p in inp["parts"]], inp["weight"].cuda(), wl.eps,
                                mode | flag, residual=inp["residual"].cuda(), emit_y=True,
                                out_q=q, out_scale=s)
    torch.cuda.synchronize()
    gpu_rowmajor_codes = gpu_util.u8(out.q)
    y = gpu_util.bits(out.y)
    rq, rs = oracle.quant_rows(y, mode)  # the quantization of the GPU's own y
    assert np.array_equal(gpu_rowmajor_codes.reshape(rq.shape), rq)
    want = oracle.place_scales(rs.reshape(M, -1), oracle.SCALE_SWIZZLE_32_4_4 if mode == MX
                               else oracle.SCALE_MN_MAJOR, fill=0)
    got = gpu_util.scale_np(s, mode).reshape(-1)
    if mode == MX:
        assert np.array_equal(got, want)
    else:
        assert np.array_equal(got.view(np.uint32), want.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("variant", [0, 1])
@pytest.mark.parametrize("mode,M,H", [(MX, 300, 7168), (MX, 5, 2048), (G128, 301, 8192),
                                      (G128, 7, 1024)])
def test_layout_with_fp16_rows(fnb, mode, M, H, variant):
    """The layout flags combined with float16 rows (FN_IO_FP16)."""
    flag = fnb.FN_SCALE_SWIZZLE_32_4_4 if mode == MX else fnb.FN_SCALE_MN_MAJOR
    wl = synth.RowWorkload("layout16", M=M, H=H, P=2, mode=mode, eps=1e-6, seed=M + H + 1,
                           dtype=torch.float16)
    inp = wl.inputs(device="cpu")
    q, s = fnb.alloc_outputs(mode | flag, M, H, "cuda")
    with fnb.prefer_variant(variant):
        out = fnb.rmsnorm_quant([p.cuda() for p in inp["parts"]], inp["weight"].cuda(), wl.eps,
                                mode | flag, residual=inp["residual"].cuda(), emit_y=True,
                                out_q=q, out_scale=s)
    torch.cuda.synchronize()
    assert out.y.dtype == torch.float16 and out.residual_out.dtype == torch.float16
    y = gpu_util.bits(out.y)
    rq, rs = oracle.quant_rows(y, mode, io=oracle.IO_FP16)
    assert np.array_equal(gpu_util.u8(out.q).reshape(rq.shape), rq)
    want = oracle.place_scales(rs.reshape(M, -1), oracle.SCALE_SWIZZLE_32_4_4 if mode == MX
                               else oracle.SCALE_MN_MAJOR, fill=0)
    got = gpu_util.scale_np(s, mode).reshape(-1)
    if mode == MX:
        assert np.array_equal(got, want)
    else:
        assert np.array_equal(got.view(np.uint32), want.astype(np.float32).view(np.uint32))


def _dequant_mx(codes_u8, scales_rowmajor_u8):
    """Dequantized MXFP4 values (float64) from packed codes and E8M0 scales."""
    table = np.array([oracle.e2m1_decode([c])[0] for c in range(16)])
    M = codes_u8.shape[0]
    e = parity.unpack_e2m1(codes_u8)
    vals = table[e]
    scale = np.ldexp(1.0, scales_rowmajor_u8.astype(np.int64) - 127)
    return vals * np.repeat(scale, 32, axis=1)


def test_block_scaled_gemm_consumes_the_swizzled_tuple(fnb):
    F = torch.nn.functional
    if not hasattr(F, "scaled_mm") or not hasattr(F, "ScalingType"):
        pytest.skip("this torch has no block-scaled scaled_mm")
    M, K, N = 256, 1024, 384
    SW = fnb.FN_SCALE_SWIZZLE_32_4_4
    wl = synth.RowWorkload("gemm_a", M=M, H=K, P=1, mode=MX, eps=1e-6, seed=31)
    inp = wl.inputs(device="cuda")
    qa, sa = fnb.alloc_outputs(MX | SW, M, K, "cuda")
    fnb.rmsnorm_quant(inp["parts"], inp["weight"], wl.eps, MX | SW, residual=inp["residual"],
                      out_q=qa, out_scale=sa)
    wb = (torch.randn((N, K), generator=torch.Generator(device="cuda").manual_seed(5),
                      device="cuda") * 0.05).to(torch.bfloat16)
    qb, sb = fnb.alloc_outputs(MX | SW, N, K, "cuda")
    fnb.quant(wb, MX | SW, out_q=qb, out_scale=sb)
    # the same quantizations with row-major scales, to dequantize on the host
    qa2, sa2 = fnb.alloc_outputs(MX, M, K, "cuda")
    fnb.rmsnorm_quant(inp["parts"], inp["weight"], wl.eps, MX, residual=inp["residual"],
                      out_q=qa2, out_scale=sa2)
    qb2, sb2 = fnb.alloc_outputs(MX, N, K, "cuda")
    fnb.quant(wb, MX, out_q=qb2, out_scale=sb2)
    torch.cuda.synchronize()
    assert torch.equal(qa, qa2) and torch.equal(qb, qb2)
    a = qa.view(torch.float4_e2m1fn_x2)
    b = qb.view(torch.float4_e2m1fn_x2)
    try:
        c = F.scaled_mm(a, b.t(), sa.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        sb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                        swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError, TypeError) as e:
        pytest.skip(f"block-scaled scaled_mm unavailable here: {str(e)[:120]}")
    torch.cuda.synchronize()
    da = _dequant_mx(gpu_util.u8(qa2), gpu_util.u8(sa2))
    db = _dequant_mx(gpu_util.u8(qb2), gpu_util.u8(sb2))
    ref = da @ db.T
    got = c.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    # bf16 output rounding (half an ulp, 2^-9 relative) plus fp32 accumulation
    tol = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(da) @ np.abs(db).T + 1e-6
    assert np.all(err <= tol), f"max err {err.max()} (max tol {tol.max()})"
