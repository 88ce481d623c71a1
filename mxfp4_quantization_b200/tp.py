"""Fused all-reduce + residual add + RMSNorm + quantization for a
tensor-parallel group (one process per GPU), over peer memory.

The pages fuse the all-reduce that follows a row-parallel linear with the
RMSNorm and the activation quantization that precede the next linear (sglang
PR #29723, "Motivation"): one kernel instead of AllReduce -> RMSNorm ->
quantize.  Here every rank owns a partial buffer (where its row-parallel GEMM
writes), a residual replica and the output buffers of the quantized tuple;
the buffers are mapped into every other rank's address space once (CUDA IPC:
each rank opens its peers' memory handles, exchanged over torch.distributed,
with its own device current and peer access enabled, so its kernels reach
the peers' memory over NVLink with plain loads and stores), and each step
runs one of two forms of the fused kernel between two group barriers:

  one-stage  every rank computes every row from all ranks' partials and
             writes only its own outputs (fn_rmsnorm_quant with the peer
             partial pointers): more NVLink reads, no gather; for few tokens.
  two-stage  rank r computes its row shard from all ranks' partials and writes
             the results into every rank's outputs (fn_ar_rmsnorm_quant): the
             reduce-scatter and the all-gather are the kernel's own peer loads
             and stores.

Choice between them (`one_stage`): the pages' rule for the 1-stage MXFP4 path
(PR #29723, review: at most 80 tokens for any 1-stage decision, and at
H=7168 the measured crossover, 1-stage through 56 tokens).  Those figures
were measured on MI355X; they are kept as the default until B200 groups
measure their own.

Failure contract (PR #29723 review): `__call__` returns None only from its
deterministic preflight checks, before any collective; once the first
barrier is entered every error raises, on every rank alike.
"""
import datetime
from typing import Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import fusednorm as fn

ONE_STAGE_MAX_TOKENS = 80
ONE_STAGE_MAX_TOKENS_H7168 = 56


def shard_rows(M: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [row0, row1) that `rank` computes in the two-stage form (the same
    split as fn_ar_rmsnorm_quant)."""
    return M * rank // world, M * (rank + 1) // world


def one_stage(M: int, H: int, max_tokens: int = ONE_STAGE_MAX_TOKENS,
              max_tokens_h7168: int = ONE_STAGE_MAX_TOKENS_H7168) -> bool:
    """The pages' 1-stage rule: a hard limit on tokens, and the measured
    cutoff at H=7168 as a further restriction."""
    if M > max_tokens:
        return False
    return M <= max_tokens_h7168 if H == 7168 else True


def _ipc_handle(t: torch.Tensor):
    """(CUDA IPC handle of the cudaMalloc allocation holding t, byte offset of
    t in it), from torch's storage sharing.  torch's handle string is a
    version byte, a kind byte ('c': a plain cudaMalloc segment) and the 64
    bytes of the cudaIpcMemHandle_t; the offset is the storage's offset in
    that segment."""
    info = t.untyped_storage()._share_cuda_()
    raw, storage_offset = bytes(info[1]), int(info[3])
    if len(raw) == 66 and raw[1:2] == b"c":
        handle = raw[2:]
    elif len(raw) == 64:
        handle = raw
    else:
        raise RuntimeError("this CUDA allocation cannot be shared through a CUDA IPC handle "
                           "(expandable segments?)")
    return handle, storage_offset + t.storage_offset() * t.element_size()


def share(tensors: Sequence[Optional[torch.Tensor]], group=None):
    """Map every rank's `tensors` into this process: returns (addresses,
    opened), where addresses[d][i] is the device address (int) of rank d's
    i-th tensor, valid for kernels on this rank's device (this rank's own
    tensors at d == rank; peers' through their CUDA IPC handles, opened with
    this rank's device current and peer access enabled), and `opened` lists
    the mappings to close with unshare().  Collective over `group`; the
    owners must keep their tensors alive until every rank has unshared."""
    from cuda.bindings import runtime as cudart
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    mine = [None if t is None else _ipc_handle(t) for t in tensors]
    everyone = [None] * world
    dist.all_gather_object(everyone, mine, group=group)
    addresses, opened = [], []
    for d in range(world):
        if d == rank:
            addresses.append([None if t is None else t.data_ptr() for t in tensors])
            continue
        row = []
        for h in everyone[d]:
            if h is None:
                row.append(None)
                continue
            handle = cudart.cudaIpcMemHandle_t()
            handle.reserved = h[0]
            err, base = cudart.cudaIpcOpenMemHandle(handle,
                                                    cudart.cudaIpcMemLazyEnablePeerAccess)
            if err != cudart.cudaError_t.cudaSuccess:
                unshare(opened)
                raise RuntimeError(f"cudaIpcOpenMemHandle of rank {d}'s buffer: {err}")
            opened.append(int(base))
            row.append(int(base) + h[1])
        addresses.append(row)
    return addresses, opened


def unshare(opened: Sequence[int]) -> None:
    """Close the peer mappings that share() opened (this rank's device must be
    current, and no work may still use them)."""
    from cuda.bindings import runtime as cudart
    for base in opened:
        cudart.cudaIpcCloseMemHandle(base)


class FusedAllReduceRMSNormQuant:
    """Per-rank state of the fused collective for batches of up to `M_max`
    rows of H.  Write this rank's partial into `self.partial[:M]` (and the
    residual into `self.residual[:M]` before the first step), then call.

    sync: "stream" orders ranks with a one-element NCCL all-reduce on the
    current stream (no host synchronisation); "host" synchronises the device
    and takes a store barrier (for process groups without a device backend).
    """

    def __init__(self, M_max: int, H: int, mode: int, group=None, device=None,
                 residual: bool = True, emit_y: bool = False, sync: str = "stream",
                 max_tokens: int = ONE_STAGE_MAX_TOKENS,
                 max_tokens_h7168: int = ONE_STAGE_MAX_TOKENS_H7168):
        if mode & (fn.FN_SCALE_MN_MAJOR | fn.FN_IO_FP16):
            raise ValueError("M-major scales (their stride depends on M) and float16 rows are "
                             "not offered by the fused collective")
        if sync not in ("stream", "host"):
            raise ValueError("sync is 'stream' or 'host'")
        self.group = group
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        if not 2 <= self.world <= 8:
            raise ValueError("2 to 8 ranks")
        self.M_max, self.H, self.mode, self.sync = M_max, H, mode, sync
        self.max_tokens, self.max_tokens_h7168 = max_tokens, max_tokens_h7168
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        bf = torch.bfloat16
        self.partial = torch.zeros((M_max, H), dtype=bf, device=dev)
        self.residual = torch.zeros((M_max, H), dtype=bf, device=dev) if residual else None
        self.q, self.scale = fn.alloc_outputs(mode, M_max, H, dev)
        self.y = torch.empty((M_max, H), dtype=bf, device=dev) if emit_y else None
        # the residual is updated in place on every rank (its replica)
        self._flag = torch.zeros(1, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        self.peers, self._opened = share([self.partial, self.residual, self.q, self.scale, self.y],
                                         group)
        self.device = dev

    def close(self) -> None:
        """Close this rank's mappings of its peers' buffers.  Every rank calls
        it after its last step, before any rank frees its buffers."""
        torch.cuda.synchronize(self.device)
        unshare(self._opened)
        self._opened = []

    # -- ordering ---------------------------------------------------------------------
    def _barrier(self):
        if self.sync == "stream":
            dist.all_reduce(self._flag, group=self.group)
        else:
            torch.cuda.synchronize(self.device)
            dist.barrier(group=self.group)

    def preflight(self, weight: torch.Tensor, eps: float, M: int) -> bool:
        """Deterministic checks on the call's arguments (identical on every
        rank by contract); False means the caller takes the unfused path."""
        return (0 < M <= self.M_max and weight.dtype == torch.bfloat16 and weight.is_cuda and
                weight.numel() == self.H and weight.is_contiguous() and eps >= 0.0)

    def __call__(self, weight: torch.Tensor, eps: float, M: int, events=None):
        """One fused step over rows [0, M).  Returns (q, scale, residual_out, y)
        views of this rank's buffers, or None if the preflight declined (no
        collective entered).  `events`: an optional pair of CUDA events
        recorded on the current stream just before and just after the kernel
        (the time between the two barriers)."""
        if not self.preflight(weight, eps, M):
            return None
        self._barrier()  # every rank's partial and residual are complete
        if events is not None:
            events[0].record()
        stream = torch.cuda.current_stream(self.device).cuda_stream
        H, mode = self.H, self.mode
        parts = [p[0] for p in self.peers]
        res = None if self.residual is None else self.residual.data_ptr()
        if one_stage(M, H, self.max_tokens, self.max_tokens_h7168):
            st = fn.fn_rmsnorm_quant(parts, self.world, res, weight.data_ptr(), float(eps), mode,
                                     M, H, self.q.data_ptr(), self.scale.data_ptr(), res,
                                     None if self.y is None else self.y.data_ptr(), stream)
            name = "fn_rmsnorm_quant"
        else:
            col = lambda i: [p[i] for p in self.peers]  # noqa: E731
            st = fn.fn_ar_rmsnorm_quant(parts, self.world, self.rank, res, weight.data_ptr(),
                                        float(eps), mode, M, H, col(2), col(3),
                                        None if res is None else col(1),
                                        None if self.y is None else col(4), stream)
            name = "fn_ar_rmsnorm_quant"
        if st != fn.FN_OK:
            raise fn.FusedNormError(name, st)
        if events is not None:
            events[1].record()
        self._barrier()  # every rank's outputs are complete
        scale = self.scale[:M] if self.scale.dim() == 2 else self.scale  # swizzled: padded, flat
        return (self.q[:M], scale, None if self.residual is None else self.residual[:M],
                None if self.y is None else self.y[:M])


def default_timeout() -> datetime.timedelta:
    """A short process-group timeout, so that ranks waiting on a lost peer end
    with an error instead of waiting for good."""
    return datetime.timedelta(seconds=60)
