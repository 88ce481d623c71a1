"""Host logic of the tensor-parallel fused collective on CPU: the two-stage
row shards of all ranks cover every row exactly once, the one-stage rule
(the pages' token limits, with the 80/81 and 56/57 boundaries), and two gloo
ranks reaching the same decisions for the same calls."""
import datetime
import os
import socket

import torch.multiprocessing as mp

from mxfp4_quantization_b200 import tp


def test_shards_cover_every_row_once():
    for world in range(2, 9):
        for M in (0, 1, 2, 7, 8, 37, 150, 8192):
            rows = []
            for r in range(world):
                a, b = tp.shard_rows(M, world, r)
                assert 0 <= a <= b <= M
                rows += list(range(a, b))
            assert rows == list(range(M)), (world, M)


def test_one_stage_boundaries():
    assert tp.one_stage(80, 4096) and not tp.one_stage(81, 4096)
    assert tp.one_stage(56, 7168) and not tp.one_stage(57, 7168)
    assert not tp.one_stage(81, 7168)
    assert tp.one_stage(1, 7168) and tp.one_stage(80, 8192)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        plan = [(M, tp.one_stage(M, 7168), tp.shard_rows(M, world, rank)) for M in (1, 56, 57, 300)]
        every = [None] * world
        dist.all_gather_object(every, plan)
        out[rank] = every
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_plan():
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert [p.exitcode for p in procs] == [0, 0]
        res = dict(out)
    every = res[0]
    assert res[1] == every
    for i, M in enumerate((1, 56, 57, 300)):
        stages = {every[r][i][1] for r in range(world)}
        assert len(stages) == 1  # every rank takes the same form
        rows = sorted(x for r in range(world) for x in range(*every[r][i][2]))
        assert rows == list(range(M))


def test_object_rejects_what_it_does_not_offer():
    """Checks that run before any device buffer or collective: M-major scales
    (their stride depends on M), float16 rows, an unknown sync mode, and a
    group of one rank."""
    import pytest
    import torch.distributed as dist
    from mxfp4_quantization_b200 import fusednorm as fn
    for mode in (fn.FN_FP8_PER_GROUP128 | fn.FN_SCALE_MN_MAJOR, fn.FN_MXFP4 | fn.FN_IO_FP16):
        with pytest.raises(ValueError):
            tp.FusedAllReduceRMSNormQuant(64, 2048, mode)
    with pytest.raises(ValueError):
        tp.FusedAllReduceRMSNormQuant(64, 2048, fn.FN_MXFP4, sync="spin")
    port = _free_port()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=30))
    try:
        with pytest.raises(ValueError):
            tp.FusedAllReduceRMSNormQuant(64, 2048, fn.FN_MXFP4)
    finally:
        dist.destroy_process_group()
