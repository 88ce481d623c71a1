"""fn_hc_mix_noalloc: hc_mix for callers that cannot allocate device memory.

Such a caller (a loop that reserved all its memory up front, a host callback,
a plugin whose framework owns every allocation) cannot hand fn_hc_mix a
workspace; this entry point keeps the intermediate in a fixed array inside
the library instead.  The test calls it through the C ABI twice in a row, on
two different sets of inputs, and checks each result against fn_hc_mix (with
a workspace) on the same inputs: the criterion of the hc_mix tests, and the
same bits, since both run the same kernels.  The second call must not see
anything of the first.

This file is named to be collected last; it needs nothing that earlier tests
leave behind and runs alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

from mxfp4_quantization_b200 import synth
from tests import gpu_util

pytestmark = pytest.mark.gpu

ATOL, RTOL = 4e-3, 1e-2  # the hc_mix tests' criterion (the page's float64 tolerance)


def bf16_vals(t):
    return (gpu_util.bits(t).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def with_workspace(fnb, wl, inp):
    out = torch.empty((wl.M, wl.C), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((fnb.fn_hc_mix_workspace_bytes(wl.M, wl.r),), dtype=torch.uint8,
                     device="cuda")
    st = fnb.fn_hc_mix(inp["x"].data_ptr(), inp["w_down"].data_ptr(), inp["w_up"].data_ptr(),
                       wl.M, wl.hc, wl.C, wl.r, out.data_ptr(), ws.data_ptr(),
                       torch.cuda.current_stream().cuda_stream)
    assert st == fnb.FN_OK, fnb.fn_status_string(st)
    return out


def without_workspace(fnb, wl, inp):
    out = torch.empty((wl.M, wl.C), dtype=torch.bfloat16, device="cuda")
    st = fnb.fn_hc_mix_noalloc(inp["x"].data_ptr(), inp["w_down"].data_ptr(),
                               inp["w_up"].data_ptr(), wl.M, wl.hc, wl.C, wl.r, out.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == fnb.FN_OK, fnb.fn_status_string(st)
    assert fnb.fn_last_variant() == fnb.FN_VARIANT_HC_MIX
    return out


@pytest.mark.parametrize("M,C,r", [(16, 2560, 64), (5, 512, 128)])
def test_no_alloc_entry_matches_the_workspace_entry_on_two_calls_in_a_row(M, C, r):
    fnb = gpu_util.lib()
    wls = [synth.HCWorkload("noalloc", M=M, C=C, r=r, seed=41 + i) for i in range(2)]
    inps = [wl.inputs(device="cuda") for wl in wls]
    got = [without_workspace(fnb, wl, inp) for wl, inp in zip(wls, inps)]
    want = [with_workspace(fnb, wl, inp) for wl, inp in zip(wls, inps)]
    torch.cuda.synchronize()
    for g, w in zip(got, want):
        gv, wv = bf16_vals(g), bf16_vals(w)
        assert np.all(np.abs(gv - wv) <= ATOL + RTOL * np.abs(wv))
        assert torch.equal(g.view(torch.int16), w.view(torch.int16))
    # the two calls' inputs differ, and so do their results
    assert not torch.equal(got[0].view(torch.int16), got[1].view(torch.int16))


def test_no_alloc_entry_rejects_what_the_scratch_cannot_hold():
    fnb = gpu_util.lib()
    wl = synth.hc_mix(4)
    inp = wl.inputs(device="cuda")
    out = torch.empty((17, wl.C), dtype=torch.bfloat16, device="cuda")
    args = [inp["x"].data_ptr(), inp["w_down"].data_ptr(), inp["w_up"].data_ptr()]
    # 17 rows or rank 136 would not fit the 16 x 128 scratch (nor the kernels)
    assert fnb.fn_hc_mix_noalloc(*args, 17, 4, wl.C, wl.r, out.data_ptr(),
                                 None) == fnb.FN_ERR_UNSUPPORTED
    assert fnb.fn_hc_mix_noalloc(*args, 4, 4, wl.C, 136, out.data_ptr(),
                                 None) == fnb.FN_ERR_UNSUPPORTED
    assert fnb.fn_hc_mix_noalloc(*args, 0, 4, wl.C, wl.r, None, None) == fnb.FN_OK
