"""Comparison of the CUDA path with the oracle (host side, numpy).

Criteria (the tolerances of the fused path):
  residual_out   bit-exact.
  y              within 1 ulp (bf16, or binary16 for binary16 rows) of the
                 oracle (the GPU reduces mean(h^2) in fp32 in another order
                 than the oracle's fp64 sum).
  quant stage    fed the GPU's own y, the oracle reproduces the GPU's codes and
                 scales bit for bit.
  end to end     against the oracle run from the inputs: in groups whose scale
                 agrees, codes may differ only where y differs, by one code
                 step at most, and (over at least 1000 codes) in at most 0.1 %
                 of positions; a group whose scale differs must have a 1-ulp
                 difference of its amax element, and the count is reported
                 separately.
  hc_mix         against the oracle's float64 u, per element: the page's
                 |gpu - u| <= 4e-3 + 1e-2 |u| (sglang PR #41880, "Accuracy
                 Tests") and the derived |gpu - u| <= 2^-8 |u| + 2e-5 * scale
                 (one bf16 rounding, at most half an ulp of 8 significant
                 bits, plus the fp32 path; `scale` grows the fp32 term with
                 the size of the logits).
"""
import numpy as np

import oracle

MX, G128, TOKEN = oracle.MXFP4, oracle.FP8_PER_GROUP128, oracle.FP8_PER_TOKEN


def bf16_ord(bits):
    """Order-preserving integers of 16-bit sign-magnitude patterns (bf16 and
    binary16 alike): neighbours differ by one."""
    b = np.asarray(bits).astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def ulp_diff(a, b):
    return np.abs(bf16_ord(a) - bf16_ord(b))


def unpack_e2m1(packed):
    p = np.asarray(packed)
    return np.stack([p & 0xF, p >> 4], axis=-1).reshape(p.shape[0], -1)


def code_ord(codes, mode):
    c = np.asarray(codes).astype(np.int64)
    if mode == MX:
        return np.where(c & 0x8, -(c & 0x7), c & 0x7)
    return np.where(c & 0x80, -(c & 0x7F), c & 0x7F)


def group_size(mode, H):
    return 32 if mode == MX else 128 if mode == G128 else H


def compare_quant_stage(y_bits, q, s, mode, io=oracle.IO_BF16):
    """GPU codes/scales vs the oracle fed the GPU's y: bit-exact."""
    rq, rs = oracle.quant_rows(y_bits, mode, io=io)
    q = np.asarray(q).reshape(rq.shape)
    s = np.asarray(s).reshape(rs.shape)
    bad_q = np.argwhere(q != rq)
    assert bad_q.size == 0, f"quant stage codes differ at {bad_q[:5].tolist()}"
    if mode == MX:
        assert np.array_equal(s, rs), f"E8M0 scales differ at {np.argwhere(s != rs)[:5].tolist()}"
    else:
        assert np.array_equal(s.view(np.uint32), rs.view(np.uint32)), \
            f"fp32 scales differ at {np.argwhere(s.view(np.uint32) != rs.view(np.uint32))[:5].tolist()}"


def compare_end_to_end(mode, H, y_gpu, q_gpu, s_gpu, y_orc, q_orc, s_orc):
    """Returns stats; asserts the end-to-end criterion."""
    M = y_gpu.shape[0]
    G = group_size(mode, H)
    ng = H // G
    if mode == MX:
        cg, co = unpack_e2m1(q_gpu), unpack_e2m1(q_orc)
        sg, so = np.asarray(s_gpu).reshape(M, ng), np.asarray(s_orc).reshape(M, ng)
        s_eq = sg == so
    else:
        cg, co = np.asarray(q_gpu).reshape(M, H), np.asarray(q_orc).reshape(M, H)
        sg = np.asarray(s_gpu, dtype=np.float32).reshape(M, ng)
        so = np.asarray(s_orc, dtype=np.float32).reshape(M, ng)
        s_eq = sg.view(np.uint32) == so.view(np.uint32)
    y_flip = ulp_diff(y_gpu, y_orc) != 0
    elem_s_eq = np.repeat(s_eq, G, axis=1)
    dcode = np.abs(code_ord(cg, mode) - code_ord(co, mode))
    in_eq = elem_s_eq
    diff = (dcode != 0) & in_eq
    n = int(in_eq.sum())
    stats = {"codes": int(cg.size), "codes_diff": int(diff.sum()),
             "max_step": int(dcode[in_eq].max()) if n else 0,
             "groups": int(s_eq.size), "scale_diff": int((~s_eq).sum()),
             "y_flips": int(y_flip.sum())}
    assert stats["max_step"] <= 1, f"code differs by {stats['max_step']} steps"
    assert not np.any(diff & ~y_flip), "a code differs where y agrees"
    if n >= 1000:
        assert stats["codes_diff"] <= 1e-3 * n, f"{stats['codes_diff']} of {n} codes differ"
    # |y| as 15-bit magnitude patterns: their integer order is the value order
    yg = (np.asarray(y_gpu).astype(np.int64) & 0x7FFF).reshape(M, ng, G)
    yo = (np.asarray(y_orc).astype(np.int64) & 0x7FFF).reshape(M, ng, G)
    for m, g in np.argwhere(~s_eq):
        assert abs(int(yg[m, g].max()) - int(yo[m, g].max())) == 1, \
            f"scale of group ({m},{g}) differs without a 1-ulp amax difference"
    return stats


def check_rmsnorm(mode, eps, parts_bits, res_bits, w_bits, gpu, io=oracle.IO_BF16):
    """gpu: dict of numpy arrays q, scale, residual_out (or None), y for the same rows."""
    orc = oracle.rmsnorm_quant(parts_bits, res_bits, w_bits, eps, mode, io=io)
    M, H = parts_bits[0].shape
    if gpu.get("residual_out") is not None:
        bad = np.argwhere(gpu["residual_out"] != orc["residual_out"])
        assert bad.size == 0, f"residual_out differs at {bad[:5].tolist()}"
    d = ulp_diff(gpu["y"], orc["y"])
    assert d.max(initial=0) <= 1, f"y differs by {d.max()} ulp at {np.argwhere(d > 1)[:5].tolist()}"
    compare_quant_stage(gpu["y"], gpu["q"], gpu["scale"], mode, io)
    return compare_end_to_end(mode, H, gpu["y"], gpu["q"], gpu["scale"], orc["y"], orc["q"],
                              orc["scale"])


# ---- every row of a full-size workload, row-parallel ---------------------------------

def _check_rows_job(job):
    """Worker (spawned process): the oracle and the criteria above on rows
    [r0, r1) of arrays saved by check_rmsnorm_all_rows."""
    d, names, n_parts, mode, eps, io, r0, r1 = job
    a = {n: np.load(f"{d}/{n}.npy", mmap_mode="r") for n in names}
    parts = [np.ascontiguousarray(a[f"part{p}"][r0:r1]) for p in range(n_parts)]
    res = np.ascontiguousarray(a["residual"][r0:r1]) if "residual" in a else None
    gpu = {"q": np.ascontiguousarray(a["q"][r0:r1]),
           "scale": np.ascontiguousarray(a["scale"][r0:r1]),
           "residual_out": (np.ascontiguousarray(a["residual_out"][r0:r1])
                            if "residual_out" in a else None),
           "y": np.ascontiguousarray(a["y"][r0:r1])}
    return check_rmsnorm(mode, eps, parts, res, np.asarray(a["weight"]), gpu, io)


def check_rmsnorm_all_rows(mode, eps, parts_bits, res_bits, w_bits, gpu, io=oracle.IO_BF16,
                           chunk=512, procs=None):
    """check_rmsnorm over every row, the oracle run row-parallel: one spawned
    process per host core (spawned, so none inherits the caller's CUDA
    context), each on chunks of `chunk` rows read from memory-mapped copies.
    Returns the summed statistics plus the number of rows compared."""
    import multiprocessing as mp
    import os
    import tempfile
    M = parts_bits[0].shape[0]
    base = "/dev/shm" if os.path.isdir("/dev/shm") else None
    with tempfile.TemporaryDirectory(dir=base) as d:
        arrays = {f"part{p}": x for p, x in enumerate(parts_bits)}
        arrays["weight"] = w_bits
        if res_bits is not None:
            arrays["residual"] = res_bits
        for k in ("q", "scale", "residual_out", "y"):
            if gpu.get(k) is not None:
                arrays[k] = gpu[k]
        for n, x in arrays.items():
            np.save(f"{d}/{n}.npy", np.asarray(x))
        jobs = [(d, tuple(arrays), len(parts_bits), mode, eps, io, r0, min(M, r0 + chunk))
                for r0 in range(0, M, chunk)]
        n = procs or os.cpu_count() or 1
        with mp.get_context("spawn").Pool(min(n, len(jobs))) as pool:
            results = pool.map(_check_rows_job, jobs)
    out = {"rows": M}
    for r in results:
        for k, v in r.items():
            out[k] = max(out.get(k, 0), v) if k == "max_step" else out.get(k, 0) + v
    return out


HC_ATOL, HC_RTOL = 4e-3, 1e-2


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def check_hc_mix(u, ub, got_bits, logit_scale=1.0):
    """hc_mix output bits (bf16 [M, C]) against the oracle's float64 u and its
    bf16 rounding ub; raises AssertionError on a failed criterion, returns
    the statistics."""
    g = bf16_bits_to_f64(got_bits)
    err = np.abs(g - u)
    assert np.all(err <= HC_ATOL + HC_RTOL * np.abs(u)), f"page tolerance: max err {err.max()}"
    bad = err > 2.0 ** -8 * np.abs(u) + 2e-5 * logit_scale
    assert not bad.any(), f"derived bound at {np.argwhere(bad)[:5].tolist()}, err {err[bad][:5]}"
    return {"max_abs_err": float(err.max()),
            "bf16_equal_frac": float(np.mean(np.asarray(got_bits) == np.asarray(ub)))}
