"""Benchmark of the fused residual-add + RMSNorm + quantization path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

The workload is the largest one-GPU configuration, the large prefill
per-group-128 FP8 pass: M=32768 rows of H=8192, x = 2 N(0,1), residual
N(0,1) updated in place, RMSNorm, per-group-128 E4M3 quantization.  A step is
192 back-to-back fused calls, alternating between two independently drawn
input slabs (each call reads 1.07 GB, far more than L2, so no flush is
needed); every call runs every step of the hot path on its rows.  A step
lasts about 55 ms, so even 20 steps time about a second.  `value` is rows/s
over all ranks (weak scaling: each rank owns its own rows, no collective on
the data path); `us_per_call` and the roofline figures are per launch.

Rank 0 prints one JSON line.  For N=1 it also carries the secondary workloads
(prefill MXFP4 with four partials, float16 rows, the quantization step alone,
per-token decode at M=16, the decode sweep per mode, the QK prologue), each
timed with CUDA events, and the CPU oracle timed on a bounded sample of the
same workload.

`--impl reference` times the CPU oracle instead (the method's plain
definition; there is no runnable GPU reference for this path) on the same
metric, one bounded sample of rows per step.
"""
import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "rows/s and achieved HBM GB/s (% of B200 peak); µs/call at M≤16"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (context beside the measured copy peak)


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def dist_max(value: float, device) -> float:
    """Max of a scalar over ranks (1 rank: the value itself)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own rows (independent problems)."""
    return base + 1000 * rank


def aggregate(rows_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job rows/s: all ranks' rows over the slowest rank's step time."""
    return rows_per_rank * world / (ms_per_step_max * 1e-3)


# ---------------------------------------------------------------------------
# clocks (read-only sampling of the GPU's clocks and throttle reasons)
# ---------------------------------------------------------------------------


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons (read only).
    `mark_start()` / `mark_end()` bracket the timed region; only samples taken
    inside it are summarised."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 50):
        self.proc = None
        self.out = None
        self.dev = device_index
        self.period = period_ms
        self.t0 = self.t1 = None

    def _uuid(self):
        import torch
        try:
            return "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
        except Exception:
            return None

    def start(self):
        uid = self._uuid()
        if uid is None:
            return
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_start(self):
        import datetime
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        import datetime
        self.t1 = datetime.datetime.now()

    def stop(self):
        import datetime
        if self.proc is None:
            return None
        time.sleep(2 * self.period / 1000.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        rows = [ln.strip().split(", ") for ln in self.out.read().splitlines() if ln.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons, n_all = [], [], set(), 0
        for r in rows:
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f")
                smv, mxv = float(r[1]), float(r[2])
            except (ValueError, IndexError):
                continue
            n_all += 1
            if self.t0 and self.t1 and not (self.t0 <= ts <= self.t1):
                continue
            sm.append(smv)
            mx.append(mxv)
            for n, v in zip(self.REASONS, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "samples_total": n_all}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm), "samples_total": n_all}


# ---------------------------------------------------------------------------
# GPU timing helpers
# ---------------------------------------------------------------------------


def time_steps(fn_step, steps: int, warmup: int, device, stream, clocks=None):
    """Untimed warm-up, then `steps` calls bracketed by a barrier and a
    synchronize, timed with CUDA events on the launching stream.
    Returns ms per step on this rank."""
    import torch
    for _ in range(warmup):
        fn_step()
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.mark_start()
    e0.record(stream)
    for _ in range(steps):
        fn_step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    if clocks is not None:
        clocks.mark_end()
    barrier(device)
    return e0.elapsed_time(e1) / steps


def _code_only(src: str) -> str:
    """Kernel source with comments and layout removed: the hash below changes
    with the code, not with its comments."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


# The sources of the row kernels (rmsnorm_quant): the traffic record below
# stays valid while these are unchanged and the launch shape is the recorded one.
ROW_KERNEL_SOURCES = ("fn_device.cuh", "quant.cuh", "rq_kernel.cuh", "rq_params.h", "rq_inst.cu")


def source_hash(files=ROW_KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mxfp4_quantization_b200", "csrc")
    for f in sorted(files):
        h.update(f.encode())
        h.update(_code_only(open(os.path.join(csrc, f)).read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel_key: str, launch=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current row-kernel sources and (when given) the same launch shape;
    None otherwise."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(p))
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != source_hash():
        return None
    if launch is not None and e.get("launch") is not None and list(e["launch"]) != list(launch):
        return None
    return e.get("dram_bytes_per_launch")


def hbm_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


MODE_NAMES = {0: "fp8_per_token", 1: "fp8_per_group128", 2: "mxfp4"}


# One benchmark step: this many back-to-back fused calls, alternating between
# two input slabs of the workload, so that even the driver's short runs
# (20 steps) time about a second of work and the clock sampler (one sample
# per 50 ms) sees the timed region.
CALLS_PER_STEP = 192
SLABS = 2


def workload_config(wl, world: int, calls_per_step: int = 1) -> dict:
    """The `config` object of the JSON line (both arms)."""
    in_mb = wl.M * wl.H * 2 * (wl.P + (1 if wl.residual else 0)) / 1e6
    return {"workload": wl.name, "M": wl.M, "H": wl.H, "P": wl.P, "mode": MODE_NAMES[wl.mode],
            "eps": wl.eps, "calls_per_step": calls_per_step,
            "rows_per_step_per_gpu": wl.M * calls_per_step, "in_place": wl.in_place,
            "io": "bf16 in; codes + scales + bf16 residual out",
            "l2": f"each call reads {in_mb:.0f} MB of inputs (L2 is 126 MB) and calls alternate "
                  f"between {SLABS} input slabs: no flush needed",
            "parallelism": f"dp{world} (independent rows, no collective)"}


def make_row_step(fn, wl, device, seed, calls: int = 1, slabs: int = 1):
    """A step of `calls` fused calls through the C ABI, alternating between
    `slabs` independently drawn input sets of the workload (each with its own
    outputs; with an in-place workload each slab's residual is updated in
    place by every call on it)."""
    import torch
    from mxfp4_quantization_b200 import synth
    mode = wl.mode | (fn.FN_IO_FP16 if wl.dtype == torch.float16 else 0)
    sets = []
    for i in range(slabs):
        wli = synth.RowWorkload(**{**wl.__dict__, "seed": seed + 7919 * i})
        inp = wli.inputs(device=device)
        parts, res, w = inp["parts"], inp["residual"], inp["weight"]
        q, s = fn.alloc_outputs(mode, wl.M, wl.H, device)
        r_out = res if wl.in_place else torch.empty_like(res)
        sets.append({"parts": parts, "ptrs": [p.data_ptr() for p in parts], "residual": res,
                     "weight": w, "q": q, "scale": s, "r_out": r_out})
    stream = torch.cuda.current_stream(device)
    sp = stream.cuda_stream
    args = [(st["ptrs"], len(st["ptrs"]), st["residual"].data_ptr(), st["weight"].data_ptr(),
             wl.eps, mode, wl.M, wl.H, st["q"].data_ptr(), st["scale"].data_ptr(),
             st["r_out"].data_ptr(), None, sp) for st in sets]

    def step():
        for i in range(calls):
            st = fn.fn_rmsnorm_quant(*args[i % slabs])
            if st != fn.FN_OK:
                raise fn.FusedNormError("fn_rmsnorm_quant", st)

    return step, stream, sets


def make_row_call(fn, wl, device, seed):
    """One fused call per step on one input set."""
    step, stream, sets = make_row_step(fn, wl, device, seed, 1, 1)
    return step, stream, sets[0]


def e2e_row(fn, wl, device, steps, warmup, seed):
    """Rows/s through the public tensor API from pinned host memory: every
    step copies its inputs host->device, runs the fused call and reads the
    quantized tuple (codes, scales, residual_out) back to pinned host memory.
    Steps are pipelined the way a serving loop would run them: two device
    buffer sets, host->device copies on one stream, the kernel on a second,
    device->host copies on a third, so that step i+1's inputs travel while
    step i computes and its results travel back (PCIe is full duplex).
    Returns (ms per step, h2d bytes per step, d2h bytes per step)."""
    import torch
    from mxfp4_quantization_b200 import synth
    wl = synth.RowWorkload(**{**wl.__dict__, "seed": seed})
    src = wl.inputs(device=device)
    h_parts = [p.to("cpu").pin_memory() for p in src["parts"]]
    h_res = src["residual"].to("cpu").pin_memory()
    w = src["weight"]
    sets = []
    for _ in range(2):
        q, s = fn.alloc_outputs(wl.mode, wl.M, wl.H, device)
        sets.append({"parts": [torch.empty_like(p) for p in src["parts"]],
                     "res": torch.empty_like(src["residual"]),
                     "rout": torch.empty_like(src["residual"]), "q": q, "s": s})
    q0, s0 = sets[0]["q"], sets[0]["s"]
    h_q = torch.empty(q0.shape, dtype=q0.dtype, pin_memory=True)
    h_s = torch.empty(s0.shape, dtype=s0.dtype, pin_memory=True)
    h_rout = torch.empty(sets[0]["rout"].shape, dtype=torch.bfloat16, pin_memory=True)
    del src
    h2d = sum(p.numel() * p.element_size() for p in h_parts) + h_res.numel() * 2
    d2h = q0.numel() * q0.element_size() + s0.numel() * s0.element_size() + h_rout.numel() * 2
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    in_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    for e in cmp_done + out_done:
        e.record(torch.cuda.current_stream(device))

    def step(i):
        b = i & 1
        st = sets[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[b])  # this set's inputs were consumed two steps ago
            for hp, dp in zip(h_parts, st["parts"]):
                dp.copy_(hp, non_blocking=True)
            st["res"].copy_(h_res, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[b])
            s_cmp.wait_event(out_done[b])  # and its outputs were read back
            fn.rmsnorm_quant(st["parts"], w, wl.eps, wl.mode, residual=st["res"],
                             out_residual=st["rout"], out_q=st["q"], out_scale=st["s"])
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            h_q.copy_(st["q"], non_blocking=True)
            h_s.copy_(st["s"], non_blocking=True)
            h_rout.copy_(st["rout"], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_cmp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    barrier(device)
    return e0.elapsed_time(e1) / steps, h2d, d2h


def time_graph_calls(make_calls, n_sets, replays, device):
    """µs per call of `n_sets` calls captured in one CUDA graph (median of
    replays), plus one eager call's device time."""
    import torch
    calls = make_calls(n_sets)
    s = torch.cuda.Stream(device)
    s.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(s):
        for c in calls[:3]:
            c()
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for c in calls:
                c()
    torch.cuda.synchronize(device)
    g.replay()
    torch.cuda.synchronize(device)
    times = []
    with torch.cuda.stream(s):
        for _ in range(replays):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            g.replay()
            e1.record(s)
            torch.cuda.synchronize(device)
            times.append(e0.elapsed_time(e1) * 1e3 / len(calls))
        eager = []
        for _ in range(20):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            calls[0]()
            e1.record(s)
            torch.cuda.synchronize(device)
            eager.append(e0.elapsed_time(e1) * 1e3)
    del g
    return statistics.median(times), statistics.median(eager)


def decode_calls(fn, wl, device):
    """Factory of rotating-buffer calls for a small-M workload: enough input
    sets that their total exceeds L2, so every call reads cold inputs."""
    import torch

    def make(n):
        inp = wl.inputs(device=device)
        parts0, res0, w = inp["parts"], inp["residual"], inp["weight"]
        calls = []
        for i in range(n):
            parts = [p.roll(i, 0).clone() for p in parts0]
            res = res0.roll(i, 0).clone()
            q, s = fn.alloc_outputs(wl.mode, wl.M, wl.H, device)
            r_out = torch.empty_like(res)
            ptrs = [p.data_ptr() for p in parts]
            keep = (parts, res, q, s, r_out)

            def call(ptrs=ptrs, res=res, q=q, s=s, r_out=r_out, keep=keep):
                sp = torch.cuda.current_stream(device).cuda_stream
                st = fn.fn_rmsnorm_quant(ptrs, len(ptrs), res.data_ptr(), w.data_ptr(), wl.eps,
                                         wl.mode, wl.M, wl.H, q.data_ptr(), s.data_ptr(),
                                         r_out.data_ptr(), None, sp)
                assert st == fn.FN_OK
            calls.append(call)
        return calls
    return make


def qk_calls(fn, wl, device, fp8=False):
    import torch

    def make(n):
        inp = wl.inputs(device=device)
        calls = []
        bf, f8, f32 = torch.bfloat16, torch.uint8, torch.float32
        for i in range(n):
            qkv = inp["qkv"].roll(i, 0).clone()
            if fp8:
                bufs = [torch.empty((wl.M, wl.Hq, wl.D), dtype=f8, device=device),
                        torch.empty((wl.M, wl.Hq), dtype=f32, device=device),
                        torch.empty((wl.M, wl.Hk, wl.D), dtype=f8, device=device),
                        torch.empty((wl.M, wl.Hk), dtype=f32, device=device),
                        torch.empty((wl.M, wl.Hq, wl.D), dtype=bf, device=device)]

                def call(qkv=qkv, bufs=bufs):
                    st = fn.fn_qk_norm_gate_fp8(
                        qkv.data_ptr(), wl.M, qkv.stride(0), wl.Hq, wl.Hk, wl.D,
                        inp["q_weight"].data_ptr(), inp["k_weight"].data_ptr(), wl.eps,
                        *[b.data_ptr() for b in bufs], None, None,
                        torch.cuda.current_stream(device).cuda_stream)
                    assert st == fn.FN_OK
            else:
                out = fn.QKOutput(torch.empty((wl.M, wl.Hq, wl.D), dtype=bf, device=device),
                                  torch.empty((wl.M, wl.Hk, wl.D), dtype=bf, device=device),
                                  torch.empty((wl.M, wl.Hq, wl.D), dtype=bf, device=device))

                def call(qkv=qkv, out=out):
                    fn.qk_norm_gate(qkv, wl.Hq, wl.Hk, wl.D, inp["q_weight"], inp["k_weight"],
                                    wl.eps, out=out)
            calls.append(call)
        return calls
    return make


def hc_calls(fn, wl, device):
    """Factory of rotating-weight hc_mix calls: every call of a graph reads its
    own copy of both weight factors (and of x), enough copies that they exceed
    L2, so every call reads its weights cold from HBM (the hc_mix page's
    method: CUDA-graph replay with rotating weights)."""
    import torch

    def make(n):
        inp = wl.inputs(device=device)
        calls = []
        for i in range(n):
            x = inp["x"].roll(i, 1).clone()
            wd = inp["w_down"].roll(i, 1).clone()
            wu = inp["w_up"].roll(i, 0).clone()
            out = torch.empty((wl.M, wl.C), dtype=torch.bfloat16, device=device)
            ws = torch.empty((wl.M * wl.r,), dtype=torch.float32, device=device)

            def call(x=x, wd=wd, wu=wu, out=out, ws=ws):
                st = fn.fn_hc_mix(x.data_ptr(), wd.data_ptr(), wu.data_ptr(), wl.M, wl.hc, wl.C,
                                  wl.r, out.data_ptr(), ws.data_ptr(),
                                  torch.cuda.current_stream(device).cuda_stream)
                assert st == fn.FN_OK
            calls.append(call)
        return calls
    return make


def small_graph_leg(fn, device, wl, per_call_bytes, make):
    """µs per call of a small-M workload: a CUDA graph of calls over rotating
    buffers whose total exceeds L2 (cold inputs), plain and as a chain of
    programmatic launches."""
    n_sets = max(64, int(2 * L2_BYTES / per_call_bytes) + 1)
    n_sets = min(n_sets, 8192)
    us, eager = time_graph_calls(make, n_sets, 7, device)
    launch = list(fn.fn_last_launch())
    # the same graph with every call a programmatic dependent of the one before
    with fn.programmatic_launch(True):
        us_pdl, _ = time_graph_calls(make, n_sets, 7, device)
    return {"us_per_call_graph": us, "us_per_call_graph_programmatic": us_pdl,
            "us_single_call_host_to_device": eager, "calls_per_graph": n_sets,
            "GB_s": per_call_bytes / (us * 1e-6) / 1e9, "launch": launch}


def secondary_workloads(fn, device, peak):
    """Every other workload, each on its own timed region (N=1 only)."""
    import torch
    from mxfp4_quantization_b200 import synth
    res = {}
    # prefill MXFP4 with four partials summed in the kernel (inputs 587 MB > L2)
    wl = synth.PREFILL_MXFP4
    step, stream, keep = make_row_step(fn, wl, device, wl.seed, 64, SLABS)
    ms = time_steps(step, 10, 3, device, stream) / 64
    b = wl.bytes_per_call()
    res["prefill_mxfp4"] = {"M": wl.M, "H": wl.H, "P": wl.P, "us_per_call": ms * 1e3,
                            "rows_per_s": wl.M / (ms * 1e-3), "GB_s": b / (ms * 1e-3) / 1e9,
                            "frac_of_peak": b / (ms * 1e-3) / 1e9 / peak,
                            "bytes_per_call": b, "variant": fn.fn_last_variant(),
                            "launch": list(fn.fn_last_launch()),
                            "traffic": measured_traffic(wl.name, fn.fn_last_launch())}
    del keep
    torch.cuda.empty_cache()

    # the two large-M shapes with float16 rows (FN_IO_FP16: the producer's dtype
    # carried through the tuple; same bytes per call)
    f16 = {}
    for base in (synth.PREFILL_MXFP4, synth.PREFILL_GROUP128):
        wl = dataclasses.replace(base, name=base.name + "_fp16", dtype=torch.float16)
        step, stream, keep = make_row_call(fn, wl, device, wl.seed)
        ms = time_steps(step, 100, 5, device, stream)
        b = wl.bytes_per_call()
        f16[wl.name] = {"M": wl.M, "H": wl.H, "P": wl.P, "us_per_call": ms * 1e3,
                        "GB_s": b / (ms * 1e-3) / 1e9, "frac_of_peak": b / (ms * 1e-3) / 1e9 / peak,
                        "variant": fn.fn_last_variant(), "launch": list(fn.fn_last_launch())}
        del keep
        torch.cuda.empty_cache()
    res["fp16_rows"] = f16

    # the quantization step alone (fn_quant) on the two large shapes' rows
    qo = {}
    for base in (synth.PREFILL_MXFP4, synth.PREFILL_GROUP128):
        wl = dataclasses.replace(base, P=1, residual=False)
        y = synth.normal_bf16((wl.M, wl.H), wl.seed, "y", device=device)
        q, s = fn.alloc_outputs(wl.mode, wl.M, wl.H, device)
        stream = torch.cuda.current_stream(device)

        def qstep(y=y, q=q, s=s, wl=wl, sp=stream.cuda_stream):
            st = fn.fn_quant(y.data_ptr(), wl.mode, wl.M, wl.H, q.data_ptr(), s.data_ptr(), sp)
            if st != fn.FN_OK:
                raise fn.FusedNormError("fn_quant", st)

        ms = time_steps(qstep, 100, 5, device, stream)
        b = wl.M * (2 * wl.H + (wl.H // 2 + wl.H // 32 if wl.mode == synth.MXFP4
                                else wl.H + 4 * (wl.H // 128)))
        qo[base.name] = {"M": wl.M, "H": wl.H, "us_per_call": ms * 1e3,
                         "GB_s": b / (ms * 1e-3) / 1e9, "frac_of_peak": b / (ms * 1e-3) / 1e9 / peak,
                         "bytes_per_call": b, "variant": fn.fn_last_variant(),
                         "launch": list(fn.fn_last_launch())}
        del y, q, s
        torch.cuda.empty_cache()
    res["quant_only"] = qo

    def small(wl, per_call_bytes, make):
        return small_graph_leg(fn, device, wl, per_call_bytes, make)

    wl = synth.PER_TOKEN_SMALL
    r = small(wl, wl.bytes_per_call(), decode_calls(fn, wl, device))
    r["variant"] = fn.fn_last_variant()
    res["per_token_small"] = r
    names = {synth.FP8_PER_TOKEN: "fp8_per_token", synth.FP8_PER_GROUP128: "fp8_per_group128",
             synth.MXFP4: "mxfp4"}
    dec = {}
    for mode in (synth.FP8_PER_TOKEN, synth.FP8_PER_GROUP128, synth.MXFP4):
        for M in synth.DECODE_M:
            wl = synth.decode(M, mode)
            r = small(wl, wl.bytes_per_call(), decode_calls(fn, wl, device))
            r["variant"] = fn.fn_last_variant()
            dec[f"{names[mode]}_m{M}"] = r
        torch.cuda.empty_cache()
    res["decode"] = dec
    qk = {}
    for M in synth.QK_M:
        wl = synth.qk_prologue(M)
        qk[f"m{M}"] = small(wl, wl.bytes_per_call(), qk_calls(fn, wl, device))
        # FP8 epilogue: codes (1 byte) and a scale per head replace the bf16 q, k
        b8 = wl.bytes_per_call() - M * (wl.Hq + wl.Hk) * (wl.D - 4)
        qk[f"m{M}_fp8"] = small(wl, b8, qk_calls(fn, wl, device, fp8=True))
    res["qk_prologue"] = qk
    res["hc_mix"] = hc_mix_leg(fn, device, peak, small)
    return res


def hc_mix_leg(fn, device, peak, small, Ms=None):
    """hc_mix at each M: graph replays over rotating cold weight sets."""
    import torch
    from mxfp4_quantization_b200 import synth
    hc = {}
    for M in (Ms or synth.HC_M):
        wl = synth.hc_mix(M)
        r = small(wl, wl.bytes_per_call(), hc_calls(fn, wl, device))
        wb = wl.weight_bytes()
        r.update({"hc": wl.hc, "C": wl.C, "r": wl.r, "bytes_per_call": wl.bytes_per_call(),
                  "weight_bytes_per_call": wb,
                  "weight_GB_s": wb / (r["us_per_call_graph"] * 1e-6) / 1e9,
                  "weight_GB_s_programmatic": wb / (r["us_per_call_graph_programmatic"] * 1e-6) / 1e9,
                  "frac_of_peak_programmatic": wl.bytes_per_call()
                  / (r["us_per_call_graph_programmatic"] * 1e-6) / 1e9 / peak,
                  "variant": fn.fn_last_variant()})
        hc[f"m{M}"] = r
        torch.cuda.empty_cache()
    return hc


# ---------------------------------------------------------------------------
# fused all-reduce across the ranks (opt-in: --tp-leg, N > 1)
# ---------------------------------------------------------------------------

TP_M = (56, 57, 80, 81, 4096)


def tp_leg(fn, device, rank: int, world: int, sync: str = "stream", Ms=TP_M, steps: int = 20,
           H: int = 7168, sample_rows: int = 8):
    """The fused all-reduce + RMSNorm + MXFP4 step across the ranks of the job
    (tp.FusedAllReduceRMSNormQuant: peer loads and stores over NVLink, no
    multicast), both forms at each M: per-call time (two group barriers and
    the kernel) and kernel-only time, both the max over ranks, the NVLink
    bytes each rank moves, a check of sampled rows against the one-GPU kernel
    on the same partials (rank 0) and of all ranks holding the same bits.  Every
    rank takes the same collective steps.  Returns the record (rank 0's is
    complete)."""
    import hashlib
    import torch
    import torch.distributed as dist
    from mxfp4_quantization_b200 import synth, tp
    mode = synth.MXFP4
    M_max = max(Ms)
    wl = synth.RowWorkload("tp_leg", M=M_max, H=H, P=world, mode=mode, eps=1e-6, seed=23,
                           channel_decades=1.0)
    inp = wl.inputs(device=device)  # every rank draws every partial; each keeps its own
    ar = tp.FusedAllReduceRMSNormQuant(M_max, H, mode, device=device, sync=sync)
    ar.partial.copy_(inp["parts"][rank])
    w = inp["weight"]
    codes_scales = H // 2 + H // 32
    out = {"H": H, "mode": "mxfp4", "world": world, "sync": sync, "steps": steps, "rows": {}}
    try:
        for M in Ms:
            row = {}
            for form, limits in (("one_stage", (M_max, M_max)), ("two_stage", (0, 0))):
                ar.max_tokens, ar.max_tokens_h7168 = limits
                # parity: one call from the drawn residual
                ar.residual.copy_(inp["residual"])
                o = ar(w, wl.eps, M)
                torch.cuda.synchronize(device)
                h = hashlib.sha256()
                for t in o[:3]:
                    h.update(t.contiguous().view(torch.uint8).cpu().numpy().tobytes())
                digests = [None] * world
                dist.all_gather_object(digests, h.hexdigest())
                check = None
                if rank == 0:
                    # against the one-GPU kernel on local copies of every
                    # rank's partial rows (the tests check that kernel against
                    # the oracle): residual bit-exact, codes equal except where
                    # the one-ulp freedom of y moves one
                    g = torch.Generator().manual_seed(M)
                    rows = sorted(set([0, M - 1] + torch.randint(0, M, (sample_rows,),
                                                                 generator=g).tolist()))
                    sel = torch.tensor(rows, device=device)
                    pick = lambda t: t.index_select(0, sel).contiguous()  # noqa: E731
                    ref = fn.rmsnorm_quant([pick(p) for p in inp["parts"]], w, wl.eps, mode,
                                           residual=pick(inp["residual"]))
                    torch.cuda.synchronize(device)
                    q, qr = pick(o[0]), ref.q
                    check = {"rows": len(rows),
                             "residual_equal": bool(torch.equal(pick(o[2]), ref.residual_out)),
                             "code_bytes_equal_frac": float((q == qr).float().mean()),
                             "scales_equal_frac": float((pick(o[1]) == ref.scale).float().mean())}
                # timing
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                ek = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(steps)]
                for _ in range(3):
                    ar(w, wl.eps, M)
                torch.cuda.synchronize(device)
                e[0].record()
                for i in range(steps):
                    ar(w, wl.eps, M, events=ek[i])
                e[1].record()
                torch.cuda.synchronize(device)
                us_call = dist_max(e[0].elapsed_time(e[1]) * 1e3 / steps, device)
                us_kernel = dist_max(statistics.median(a.elapsed_time(b) * 1e3 for a, b in ek),
                                     device)
                if form == "one_stage":
                    nvl_read, nvl_write = (world - 1) * M * 2 * H, 0
                else:
                    shard = M // world + (1 if M % world else 0)
                    nvl_read = (world - 1) * shard * 2 * H
                    nvl_write = (world - 1) * shard * (2 * H + codes_scales)
                row[form] = {"us_per_call": us_call, "us_kernel": us_kernel,
                             "nvlink_bytes_read_per_rank": nvl_read,
                             "nvlink_bytes_written_per_rank": nvl_write,
                             "nvlink_GB_s_per_rank": (nvl_read + nvl_write) / (us_kernel * 1e-6)
                             / 1e9 if us_kernel > 0 else None,
                             "ranks_identical": len(set(digests)) == 1,
                             "vs_one_gpu_kernel": check}
            row["faster_kernel"] = min(("one_stage", "two_stage"),
                                       key=lambda f: row[f]["us_kernel"])
            out["rows"][str(M)] = row
    finally:
        ar.close()
        dist.barrier()
        del ar
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; the reference arm)
# ---------------------------------------------------------------------------


def pick_workload(name: str):
    from mxfp4_quantization_b200 import synth
    return synth.PREFILL_MXFP4 if name == "prefill_mxfp4" else synth.PREFILL_GROUP128


def oracle_rows_per_s(rows: int, min_seconds: float, max_seconds: float, workload: str):
    """The oracle, as it stands, single-threaded, on `rows` rows of the
    workload's recipe, repeated until `min_seconds` have passed."""
    import oracle
    from mxfp4_quantization_b200 import synth
    wl = pick_workload(workload)
    inp = wl.inputs(device="cpu", M=rows)
    parts = [synth.to_bits(p) for p in inp["parts"]]
    res, w = synth.to_bits(inp["residual"]), synth.to_bits(inp["weight"])
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)
        done += rows
        el = time.perf_counter() - t0
        if el >= min_seconds or el >= max_seconds:
            break
    return done / el, done, el


def _time_calls(fn, min_seconds: float, max_calls: int):
    """Calls of `fn` until `min_seconds` have passed (at least one, at most
    max_calls); returns (seconds per call, calls)."""
    done, t0 = 0, time.perf_counter()
    while True:
        fn()
        done += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or done >= max_calls:
            return el / done, done


def oracle_per_config(seconds: float = 1.0):
    """The oracle, as it stands, single-threaded, on every other configuration
    of the run: each call of a decode-sized configuration whole (µs per call,
    the GPU figures' unit), the MXFP4 prefill on a 64-row sample (rows/s);
    about `seconds` of repeated calls each."""
    import oracle
    from mxfp4_quantization_b200 import synth
    out = {}

    def rows_cfg(wl, M=None):
        inp = wl.inputs(device="cpu", M=M)
        parts = [synth.to_bits(p) for p in inp["parts"]]
        res = synth.to_bits(inp["residual"]) if inp.get("residual") is not None else None
        w = synth.to_bits(inp["weight"])
        return lambda: oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)

    wl = synth.PREFILL_MXFP4
    sec, n = _time_calls(rows_cfg(wl, 64), seconds, 1000)
    out["prefill_mxfp4"] = {"value": 64 / sec, "unit": "rows/s", "cores": 1,
                            "sample": f"64 rows of the recipe (H={wl.H}, P={wl.P}), {n} calls"}
    wl = synth.PER_TOKEN_SMALL
    sec, n = _time_calls(rows_cfg(wl), seconds, 10000)
    out["per_token_small"] = {"value": sec * 1e6, "unit": "us/call", "cores": 1,
                              "sample": f"whole call (M={wl.M}, H={wl.H}), {n} calls"}
    for mode, mname in ((synth.FP8_PER_TOKEN, "fp8_per_token"),
                        (synth.FP8_PER_GROUP128, "fp8_per_group128"), (synth.MXFP4, "mxfp4")):
        wl = synth.decode(16, mode)
        sec, n = _time_calls(rows_cfg(wl), seconds / 3, 10000)
        out[f"decode_{mname}_m16"] = {"value": sec * 1e6, "unit": "us/call", "cores": 1,
                                      "sample": f"whole call (M=16, H={wl.H}), {n} calls"}
    for M in synth.QK_M:
        wl = synth.qk_prologue(M)
        inp = wl.inputs(device="cpu")
        qkv, qw, kw = (synth.to_bits(inp[k]) for k in ("qkv", "q_weight", "k_weight"))
        sec, n = _time_calls(lambda: oracle.qk_norm_gate(qkv, wl.row_stride, wl.Hq, wl.Hk, wl.D,
                                                         qw, kw, wl.eps),
                             seconds / 2, 10000)
        out[f"qk_prologue_m{M}"] = {"value": sec * 1e6, "unit": "us/call", "cores": 1,
                                    "sample": f"whole call (M={M}), {n} calls"}
    for M in (1, 16):
        wl = synth.hc_mix(M)
        inp = wl.inputs(device="cpu")
        x, wd, wu = (synth.to_bits(inp[k]) for k in ("x", "w_down", "w_up"))
        sec, n = _time_calls(lambda: oracle.hc_mix(x, wd, wu, wl.hc, wl.C, wl.r), seconds / 2,
                             10000)
        out[f"hc_mix_m{M}"] = {"value": sec * 1e6, "unit": "us/call", "cores": 1,
                               "sample": f"whole call (M={M}, C={wl.C}, r={wl.r}), {n} calls"}
    return out


def _oracle_worker(job):
    rows, seconds, workload = job
    rate, done, el = oracle_rows_per_s(rows, seconds, 3 * seconds, workload)
    return done, el


def oracle_rows_per_s_all_cores(rows: int, seconds: float, workload: str):
    """The same oracle run row-parallel: one process per host core (spawned,
    so no process inherits a CUDA context), each on its own `rows` rows for
    about `seconds`.  Returns (rows/s over all processes, processes)."""
    import multiprocessing as mp
    n = os.cpu_count() or 1
    with mp.get_context("spawn").Pool(n) as pool:
        res = pool.map(_oracle_worker, [(rows, seconds, workload)] * n)
    return sum(d for d, _ in res) / max(el for _, el in res), n


def reference_arm(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from mxfp4_quantization_b200 import synth
    oracle.load()
    wl = pick_workload(args.workload)
    rate, _, _ = oracle_rows_per_s(8, 0.5, 5.0, args.workload)
    budget_s = 90.0
    rows_per_step = int(max(1, min(wl.M, rate * budget_s / max(1, args.steps + args.warmup))))
    inp = synth.RowWorkload(**{**wl.__dict__}).inputs(device="cpu", M=rows_per_step)
    parts = [synth.to_bits(p) for p in inp["parts"]]
    res, w = synth.to_bits(inp["residual"]), synth.to_bits(inp["weight"])
    for _ in range(args.warmup):
        oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.rmsnorm_quant(parts, res, w, wl.eps, wl.mode)
    el = time.perf_counter() - t0
    value = rows_per_step * args.steps / el
    sample = (f"{rows_per_step} rows of the {wl.name} workload (H={wl.H}, P={wl.P}) per step, "
              f"single-threaded oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world, args.calls_per_step),
            "rows_per_step": rows_per_step,
            "cpu_baseline": {"value": value, "unit": "rows/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# main arm
# ---------------------------------------------------------------------------


def main_arm(args):
    import torch
    rank, world, local = dist_env()
    if world != args.gpus:
        world = max(world, 1)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    if rank == 0:
        from mxfp4_quantization_b200.build import build_library
        build_library()
    barrier(device)
    from mxfp4_quantization_b200 import fusednorm as fn
    from mxfp4_quantization_b200 import synth

    wl = pick_workload(args.workload)
    seed = rank_seed(wl.seed, rank)
    calls = args.calls_per_step
    step, stream, keep = make_row_step(fn, wl, device, seed, calls, SLABS)
    clocks = ClockSampler(local)
    # the sampler needs a moment to start; it runs over the warm-up and the
    # timed steps, and only samples taken while steps run are kept
    clocks.start()
    time.sleep(0.5)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    ms = time_steps(step, args.steps, 0, device, stream, clocks)
    clk = clocks.stop()
    variant, launch = fn.fn_last_variant(), fn.fn_last_launch()
    ms_max = dist_max(ms, device)
    value = aggregate(wl.M * calls, world, ms_max)
    bytes_call = wl.bytes_per_call()
    peak, peak_kind = hbm_peak()
    us_call = ms * 1e3 / calls  # every launch of the step is the same kernel
    achieved = bytes_call / (us_call * 1e-6) / 1e9
    traffic = measured_traffic(wl.name, launch)
    # the same step with every call a programmatic dependent of the one before
    # (reported beside the line's value, which keeps plain launches)
    with fn.programmatic_launch(True):
        step()
        ms_pdl = time_steps(step, max(3, min(args.steps, 5)), 0, device, stream)
    us_call_pdl = dist_max(ms_pdl, device) * 1e3 / calls
    del keep
    torch.cuda.empty_cache()

    e2e_steps = max(4, min(args.steps, 20))
    e2e_ms, h2d, d2h = e2e_row(fn, wl, device, e2e_steps, 2, seed)
    e2e_ms_max = dist_max(e2e_ms, device)

    tp_record = None
    if world > 1 and args.tp_leg:
        tp_record = tp_leg(fn, device, rank, world)

    extra = None
    cpu = cpu_all = cpu_configs = None
    if world == 1 and not args.no_extras and args.workload == "prefill_group128":
        extra = secondary_workloads(fn, device, peak)
    if world == 1 and not args.no_cpu_baseline:
        rate, rows, el = oracle_rows_per_s(256, args.cpu_seconds, 3 * args.cpu_seconds,
                                           args.workload)
        cpu = {"value": rate, "unit": "rows/s", "cores": 1, "kind": "oracle",
               "sample": f"{rows} rows (256 rows of the {wl.name} recipe, H={wl.H}, P={wl.P}, "
                         f"repeated) in {el:.1f} s, single-threaded; "
                         f"host has {os.cpu_count()} cores"}
        rate_all, procs = oracle_rows_per_s_all_cores(64, max(1.0, args.cpu_seconds / 2),
                                                      args.workload)
        cpu_all = {"value": rate_all, "unit": "rows/s", "cores": procs,
                   "kind": "oracle, row-parallel processes (context beside cpu_baseline)",
                   "sample": f"64 rows of the {wl.name} recipe per process, repeated for "
                             f"about {max(1.0, args.cpu_seconds / 2):.0f} s, {procs} processes"}
        if extra is not None:
            cpu_configs = oracle_per_config()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, world, calls),
            "us_per_call": us_call,
            "us_per_call_programmatic": us_call_pdl,
            "hbm_GB_s": achieved, "frac_of_peak": achieved / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "achieved_is": "algorithmic bytes per launch / CUDA-event time per "
                                        "launch (timed region / launches)",
                         "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                         "traffic": traffic,
                         "traffic_is": "ncu dram__bytes_read.sum + dram__bytes_write.sum per "
                                       "launch (profiles/), null if the kernel changed since",
                         "algorithmic_bytes_per_launch": bytes_call,
                         "kernel": {fn.FN_VARIANT_ROW_CTA: "rq_kernel (one block per row)",
                                    fn.FN_VARIANT_ROW_CLUSTER: "rq_kernel (cluster per row)"}.get(
                                        variant, str(variant)),
                         "launch": list(launch), "variant": variant},
            "e2e": {"value": aggregate(wl.M, world, e2e_ms_max), "unit": "rows/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "method": "public tensor API, one call per e2e step; pinned host buffers; "
                              "copies in, kernel and copies out on three streams, two buffer "
                              "sets (steps pipelined)"},
            "gpu_launches": args.steps * calls,
            "clocks": clk,
            "cpu_baseline": cpu,
            "cpu_baseline_all_cores": cpu_all,
            "cpu_baseline_per_config": cpu_configs,
            "workloads": extra,
            "tensor_parallel": tp_record,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        barrier(device)
        dist.destroy_process_group()
    return 0


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=["prefill_mxfp4", "prefill_group128"],
                    default="prefill_group128", help="the workload a step runs")
    ap.add_argument("--calls-per-step", type=int, default=CALLS_PER_STEP,
                    help="fused calls per step (alternating between input slabs)")
    ap.add_argument("--no-extras", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--leg", choices=["hc_mix"], default=None,
                    help="run only this secondary workload and print its record")
    ap.add_argument("--hc-m", type=int, nargs="*", default=None,
                    help="with --leg hc_mix: the row counts (default 1 2 4 8 16)")
    ap.add_argument("--tp-leg", action="store_true",
                    help="with N > 1: also time the fused all-reduce across the ranks")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    a = ap.parse_args(argv)
    a.warmup = max(a.warmup, 3)  # timing rule: at least 3 untimed warm-up steps
    return a


def leg_arm(args):
    """One secondary workload alone (one GPU), its record as one JSON line."""
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    from mxfp4_quantization_b200.build import build_library
    build_library()
    from mxfp4_quantization_b200 import fusednorm as fn
    peak, _ = hbm_peak()
    small = lambda wl, b, make: small_graph_leg(fn, device, wl, b, make)  # noqa: E731
    rec = hc_mix_leg(fn, device, peak, small, args.hc_m)
    print(json.dumps({"leg": args.leg, "record": rec}), flush=True)
    return 0


if __name__ == "__main__":
    args = parse()
    if args.impl == "reference":
        sys.exit(reference_arm(args))
    sys.exit(leg_arm(args) if args.leg else main_arm(args))
