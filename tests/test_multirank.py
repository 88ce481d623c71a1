"""The multi-GPU host logic of bench.py on CPU: two gloo ranks, no GPU.

Rows are independent problems, so N GPUs run N replicas on their own rows
(weak scaling) with no collective on the data path.  What needs checking is
the host side: every rank draws different rows, the step time is the max over
ranks, and the reported value counts all ranks' rows.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    from mxfp4_quantization_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        # each rank its own rows
        wl = synth.PREFILL_MXFP4
        seed = bench.rank_seed(wl.seed, rank)
        wl_r = synth.RowWorkload(**{**wl.__dict__, "seed": seed})
        x = wl_r.inputs(device="cpu", M=4)["parts"][0]
        # a fake per-rank step time: the slowest rank decides
        ms = 1.0 + rank
        ms_max = bench.dist_max(ms, dev)
        bench.barrier(dev)
        value = bench.aggregate(wl.M, world, ms_max)
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out[rank] = (ms_max, value, all(not torch.equal(gathered[0], g) for g in gathered[1:]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0, f"rank exited with {p.exitcode}"
        res = dict(out)
    assert set(res) == {0, 1}
    for rank, (ms_max, value, distinct) in res.items():
        assert ms_max == 2.0, "step time is the max over ranks"
        assert value == pytest.approx(8192 * 2 / 2e-3), "value counts every rank's rows"
        assert distinct, "ranks draw different rows"


def test_single_rank_helpers_without_process_group():
    import bench
    assert bench.dist_max(3.5, torch.device("cpu")) == 3.5
    assert bench.aggregate(100, 1, 2.0) == pytest.approx(50_000.0)
    assert bench.rank_seed(3, 0) != bench.rank_seed(3, 1)
