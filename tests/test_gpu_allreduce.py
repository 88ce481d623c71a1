"""The fused all-reduce + RMSNorm + quantization (two-stage form) on one GPU.

Virtual ranks: the group's buffers all live on one device and the ranks'
calls run one after another on one stream (stream order stands in for the
group barriers; no kernel waits on another).  Every rank must end with the
same bits, and they must meet the parity criteria against the oracle run on
the summed partials.  Then two processes on the same GPU share their buffers
through CUDA IPC and run the tensor-parallel object with host barriers.
"""
import datetime
import hashlib
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from mxfp4_quantization_b200 import synth
from tests import gpu_util, parity

pytestmark = pytest.mark.gpu

TOKEN, G128, MX = synth.FP8_PER_TOKEN, synth.FP8_PER_GROUP128, synth.MXFP4


@pytest.fixture(scope="module")
def fnb():
    return gpu_util.lib()


def _rank_buffers(fnb, mode, M, H, world, flags=0, emit_y=True):
    bufs = []
    for _ in range(world):
        q, s = fnb.alloc_outputs(mode | flags, M, H, "cuda")
        bufs.append({"q": q, "scale": s, "residual": None,
                     "y": torch.empty((M, H), dtype=torch.bfloat16, device="cuda") if emit_y
                     else None})
    return bufs


@pytest.mark.parametrize("world", [2, 3, 4, 8])
@pytest.mark.parametrize("mode", [TOKEN, G128, MX], ids=["token", "g128", "mxfp4"])
@pytest.mark.parametrize("M,H", [(37, 7168), (150, 2048), (5, 8192)])
def test_virtual_ranks(fnb, world, mode, M, H):
    wl = synth.RowWorkload("ar", M=M, H=H, P=world, mode=mode, eps=1e-6, seed=M + world,
                           channel_decades=1.0)
    inp = wl.inputs(device="cuda")
    parts, res0, w = inp["parts"], inp["residual"], inp["weight"]
    bufs = _rank_buffers(fnb, mode, M, H, world)
    for b in bufs:
        b["residual"] = res0.clone()  # every rank's replica, updated in place
    ptr = lambda key: [b[key].data_ptr() for b in bufs]  # noqa: E731
    for r in range(world):
        st = fnb.fn_ar_rmsnorm_quant([p.data_ptr() for p in parts], world, r,
                                     bufs[r]["residual"].data_ptr(), w.data_ptr(), wl.eps, mode,
                                     M, H, ptr("q"), ptr("scale"), ptr("residual"), ptr("y"), None)
        assert st == fnb.FN_OK, fnb.fn_status_string(st)
        r0, r1 = M * r // world, M * (r + 1) // world
        if r1 > r0:
            assert fnb.fn_last_variant() == fnb.FN_VARIANT_ROW_ALLREDUCE
            assert fnb.fn_last_launch()[0] == r1 - r0
    torch.cuda.synchronize()
    for b in bufs[1:]:
        for key in ("q", "scale", "residual", "y"):
            assert torch.equal(b[key].view(torch.uint8), bufs[0][key].view(torch.uint8)), key
    gpu = {"q": gpu_util.u8(bufs[0]["q"]), "scale": gpu_util.scale_np(bufs[0]["scale"], mode),
           "residual_out": gpu_util.bits(bufs[0]["residual"]), "y": gpu_util.bits(bufs[0]["y"])}
    parity.check_rmsnorm(mode, wl.eps, [gpu_util.bits(p) for p in parts], gpu_util.bits(res0),
                         gpu_util.bits(w), gpu)


def _random_ar_cases(n, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        mode = int(rng.integers(0, 3))
        unit = {TOKEN: 8, G128: 128, MX: 32}[mode]
        H = int(unit * rng.integers(1, max(2, 8192 // unit) + 1))
        out.append((i, mode, int(rng.integers(2, 9)), int(rng.choice([1, 2, 7, 16, 63, 200])), H,
                    bool(rng.integers(0, 4) > 0)))
    return out


@pytest.mark.parametrize("i,mode,world,M,H,has_res", _random_ar_cases(24),
                         ids=[f"r{c[0]}" for c in _random_ar_cases(24)])
def test_virtual_ranks_random(fnb, i, mode, world, M, H, has_res):
    """Seeded random groups (2..8 ranks, shards from empty to many rows, any
    H the mode allows up to 8192, with or without a residual)."""
    wl = synth.RowWorkload("ar_rand", M=M, H=H, P=world, mode=mode, eps=1e-6, seed=500 + i,
                           residual=has_res, channel_decades=1.0)
    inp = wl.inputs(device="cuda")
    parts, res0, w = inp["parts"], inp["residual"], inp["weight"]
    bufs = _rank_buffers(fnb, mode, M, H, world)
    for b in bufs:
        b["residual"] = res0.clone() if has_res else torch.empty((M, H), dtype=torch.bfloat16,
                                                                 device="cuda")
    ptr = lambda key: [b[key].data_ptr() for b in bufs]  # noqa: E731
    for r in range(world):
        st = fnb.fn_ar_rmsnorm_quant([p.data_ptr() for p in parts], world, r,
                                     bufs[r]["residual"].data_ptr() if has_res else None,
                                     w.data_ptr(), wl.eps, mode, M, H, ptr("q"), ptr("scale"),
                                     ptr("residual"), ptr("y"), None)
        assert st == fnb.FN_OK, fnb.fn_status_string(st)
    torch.cuda.synchronize()
    for b in bufs[1:]:
        for key in ("q", "scale", "residual", "y"):
            assert torch.equal(b[key].view(torch.uint8), bufs[0][key].view(torch.uint8)), key
    gpu = {"q": gpu_util.u8(bufs[0]["q"]), "scale": gpu_util.scale_np(bufs[0]["scale"], mode),
           "residual_out": gpu_util.bits(bufs[0]["residual"]), "y": gpu_util.bits(bufs[0]["y"])}
    parity.check_rmsnorm(mode, wl.eps, [gpu_util.bits(p) for p in parts],
                         gpu_util.bits(res0) if has_res else None, gpu_util.bits(w), gpu)


def test_virtual_ranks_swizzled_scales_no_residual(fnb):
    M, H, world = 130, 7168, 4
    SW = fnb.FN_SCALE_SWIZZLE_32_4_4
    wl = synth.RowWorkload("ar_sw", M=M, H=H, P=world, mode=MX, eps=1e-6, seed=77,
                           residual=False)
    inp = wl.inputs(device="cuda")
    bufs = _rank_buffers(fnb, MX, M, H, world, flags=SW, emit_y=True)
    ptr = lambda key: [b[key].data_ptr() for b in bufs]  # noqa: E731
    for r in range(world):
        st = fnb.fn_ar_rmsnorm_quant([p.data_ptr() for p in inp["parts"]], world, r, None,
                                     inp["weight"].data_ptr(), wl.eps, MX | SW, M, H, ptr("q"),
                                     ptr("scale"), None, ptr("y"), None)
        assert st == fnb.FN_OK
    torch.cuda.synchronize()
    for b in bufs[1:]:
        assert torch.equal(b["q"], bufs[0]["q"]) and torch.equal(b["scale"], bufs[0]["scale"])
    y = gpu_util.bits(bufs[0]["y"])
    rq, rs = oracle.quant_rows(y, MX)
    assert np.array_equal(gpu_util.u8(bufs[0]["q"]).reshape(rq.shape), rq)
    want = oracle.place_scales(rs.reshape(M, -1), oracle.SCALE_SWIZZLE_32_4_4, fill=0)
    assert np.array_equal(gpu_util.u8(bufs[0]["scale"]).reshape(-1), want)
    orc = oracle.rmsnorm_quant([gpu_util.bits(p) for p in inp["parts"]], None,
                               gpu_util.bits(inp["weight"]), wl.eps, MX)
    assert parity.ulp_diff(y, orc["y"]).max() <= 1


# ---- two processes, one GPU, CUDA IPC ---------------------------------------------


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, H, M_list, out):
    import torch.distributed as dist

    from mxfp4_quantization_b200 import tp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=90))
    try:
        torch.cuda.set_device(0)
        M_max = max(M_list)
        wl = synth.RowWorkload("tp", M=M_max, H=H, P=world, mode=mode, eps=1e-6, seed=91,
                               channel_decades=1.0)
        inp = wl.inputs(device="cuda")
        ar = tp.FusedAllReduceRMSNormQuant(M_max, H, mode, sync="host", emit_y=True)
        ar.partial.copy_(inp["parts"][rank])
        results = []
        for M in M_list:
            ar.residual.copy_(inp["residual"])
            o = ar(inp["weight"], wl.eps, M)
            torch.cuda.synchronize()
            gpu = {"q": gpu_util.u8(o[0]), "scale": gpu_util.scale_np(o[1], mode),
                   "residual_out": gpu_util.bits(o[2]), "y": gpu_util.bits(o[3])}
            parity.check_rmsnorm(mode, wl.eps, [gpu_util.bits(p[:M]) for p in inp["parts"]],
                                 gpu_util.bits(inp["residual"][:M]), gpu_util.bits(inp["weight"]),
                                 gpu)
            digest = [hashlib.sha256(gpu[k].tobytes()).hexdigest()
                      for k in ("q", "scale", "residual_out", "y")]
            results.append((M, tp.one_stage(M, H), digest))
        assert ar(inp["weight"], wl.eps, M_max + 1) is None  # preflight: no collective
        ar.close()
        dist.barrier()
        out[rank] = results
    except Exception as e:  # reported to the parent
        out[rank] = f"error: {type(e).__name__}: {e}"
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [MX, TOKEN], ids=["mxfp4", "token"])
def test_two_processes_share_one_gpu(mode):
    world, H, M_list = 2, 7168, [40, 150]  # one-stage, then two-stage
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, H, M_list, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], (codes, res)
    assert res[0] == res[1], "ranks disagree"
    assert [(m, s) for m, s, _ in res[0]] == [(40, True), (150, False)]


def _leg_main(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=90))
    try:
        torch.cuda.set_device(0)
        fnb = gpu_util.lib()
        out[rank] = bench.tp_leg(fnb, torch.device("cuda", 0), rank, world, sync="host",
                                 Ms=(40, 150), steps=3, H=2048)
    except Exception as e:  # reported to the parent
        out[rank] = f"error: {type(e).__name__}: {e}"
        raise
    finally:
        dist.destroy_process_group()


def test_bench_tensor_parallel_leg_runs_on_two_processes():
    """The bench's fused all-reduce leg (both forms, timing, the check against
    the one-GPU kernel, ranks holding the same bits), run by two processes
    sharing one GPU through CUDA IPC with host barriers."""
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_leg_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], (codes, res)
    rec = res[0]
    for M in ("40", "150"):
        for form in ("one_stage", "two_stage"):
            r = rec["rows"][M][form]
            assert r["ranks_identical"], (M, form)
            c = r["vs_one_gpu_kernel"]
            assert c["residual_equal"] and c["code_bytes_equal_frac"] > 0.99, (M, form, c)
            assert r["us_kernel"] > 0 and r["us_per_call"] >= r["us_kernel"]
