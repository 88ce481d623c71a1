"""Python binding of libfusednorm.so (argument marshalling only).

Two layers:
  * `fn_rmsnorm_quant`, `fn_quant`, `fn_qk_norm_gate`, `fn_status_string`,
    `fn_last_variant`, `fn_last_launch`, `fn_version`: the C ABI of
    include/fusednorm.h one to one, taking raw device addresses (ints) and
    returning the status code.
  * `rmsnorm_quant`, `quant`, `qk_norm_gate`: take torch CUDA tensors, allocate
    the outputs with torch (device memory is torch's plumbing), call the C
    ABI on the current stream, and raise `FusedNormError` on a non-zero status.
    Every step of the computation runs in the library's kernels.

There is no fallback: if the library is missing, importing this module fails.
"""
import ctypes
import os
from collections import namedtuple
from typing import Optional, Sequence, Union

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfusednorm.so")

FN_FP8_PER_TOKEN = 0
FN_FP8_PER_GROUP128 = 1
FN_MXFP4 = 2

FN_OK = 0
FN_ERR_INVALID = -1
FN_ERR_ALIGN = -2
FN_ERR_UNSUPPORTED = -3
FN_ERR_CUDA = -4

FN_VARIANT_NONE = 0
FN_VARIANT_ROW_CTA = 1
FN_VARIANT_ROW_CLUSTER = 2
FN_VARIANT_QUANT_ONLY = 3
FN_VARIANT_QK_WARP = 4
FN_VARIANT_QK_WARP_FP8 = 6
FN_VARIANT_ROW_ALLREDUCE = 7
FN_VARIANT_HC_MIX = 8

FN_MODE_MASK = 0xFF
FN_SCALE_SWIZZLE_32_4_4 = 0x100
FN_SCALE_MN_MAJOR = 0x200
FN_IO_FP16 = 0x1000

HC_STREAMS = 4
HC_MAX_ROWS = 16

FN_MAX_PARTS = 8
FN_MAX_H = 32768
FN_MAX_HEAD_DIM = 1024

MODES = {"fp8_per_token": FN_FP8_PER_TOKEN, "fp8_per_group128": FN_FP8_PER_GROUP128,
         "mxfp4": FN_MXFP4}

# The exported symbols of include/fusednorm.h.
ABI_SYMBOLS = ("fn_rmsnorm_quant", "fn_ar_rmsnorm_quant", "fn_quant", "fn_qk_norm_gate",
               "fn_qk_norm_gate_fp8", "fn_hc_mix", "fn_hc_mix_workspace_bytes",
               "fn_hc_mix_noalloc",
               "fn_status_string",
               "fn_last_variant", "fn_last_launch", "fn_prefer_variant",
               "fn_programmatic_launch", "fn_version")


class FusedNormError(RuntimeError):
    def __init__(self, func: str, status: int):
        super().__init__(f"{func}: {fn_status_string(status)} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m mxfp4_quantization_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.fn_rmsnorm_quant.argtypes = [ctypes.POINTER(vp), i32, vp, vp, ctypes.c_float, i32, i64,
                                     i64, vp, vp, vp, vp, vp]
    lib.fn_rmsnorm_quant.restype = i32
    pvp = ctypes.POINTER(vp)
    lib.fn_ar_rmsnorm_quant.argtypes = [pvp, i32, i32, vp, vp, ctypes.c_float, i32, i64, i64,
                                        pvp, pvp, pvp, pvp, vp]
    lib.fn_ar_rmsnorm_quant.restype = i32
    lib.fn_quant.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    lib.fn_quant.restype = i32
    lib.fn_qk_norm_gate.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, ctypes.c_float, vp, vp,
                                    vp, vp]
    lib.fn_qk_norm_gate.restype = i32
    lib.fn_qk_norm_gate_fp8.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp, ctypes.c_float, vp,
                                        vp, vp, vp, vp, vp, vp, vp]
    lib.fn_qk_norm_gate_fp8.restype = i32
    lib.fn_hc_mix.argtypes = [vp, vp, vp, i64, i32, i64, i32, vp, vp, vp]
    lib.fn_hc_mix.restype = i32
    lib.fn_hc_mix_workspace_bytes.argtypes = [i64, i32]
    lib.fn_hc_mix_workspace_bytes.restype = i64
    lib.fn_hc_mix_noalloc.argtypes = [vp, vp, vp, i64, i32, i64, i32, vp, vp]
    lib.fn_hc_mix_noalloc.restype = i32
    lib.fn_status_string.argtypes = [i32]
    lib.fn_status_string.restype = ctypes.c_char_p
    lib.fn_last_variant.argtypes = []
    lib.fn_last_variant.restype = i32
    lib.fn_last_launch.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    lib.fn_last_launch.restype = None
    lib.fn_prefer_variant.argtypes = [i32]
    lib.fn_prefer_variant.restype = i32
    lib.fn_programmatic_launch.argtypes = [i32]
    lib.fn_programmatic_launch.restype = i32
    lib.fn_version.argtypes = []
    lib.fn_version.restype = i32
    return lib


_lib = _load()


# ---- the C ABI, one to one --------------------------------------------------------


def fn_rmsnorm_quant(x_parts: Sequence[int], num_parts: int, residual: Optional[int],
                     weight: int, eps: float, mode: int, M: int, H: int, out_q: int,
                     out_scale: int, out_residual: Optional[int], out_y: Optional[int],
                     stream: Optional[int]) -> int:
    arr = (ctypes.c_void_p * max(1, len(x_parts)))(*x_parts)
    return _lib.fn_rmsnorm_quant(arr, num_parts, residual, weight, eps, mode, M, H, out_q,
                                 out_scale, out_residual, out_y, stream)


def _ptr_array(ptrs: Optional[Sequence[int]]):
    return None if ptrs is None else (ctypes.c_void_p * max(1, len(ptrs)))(*ptrs)


def fn_ar_rmsnorm_quant(x_parts: Sequence[int], num_ranks: int, rank: int,
                        residual: Optional[int], weight: int, eps: float, mode: int, M: int,
                        H: int, out_q: Sequence[int], out_scale: Sequence[int],
                        out_residual: Optional[Sequence[int]], out_y: Optional[Sequence[int]],
                        stream: Optional[int]) -> int:
    return _lib.fn_ar_rmsnorm_quant(_ptr_array(x_parts), num_ranks, rank, residual, weight, eps,
                                    mode, M, H, _ptr_array(out_q), _ptr_array(out_scale),
                                    _ptr_array(out_residual), _ptr_array(out_y), stream)


def fn_quant(y: int, mode: int, M: int, H: int, out_q: int, out_scale: int,
             stream: Optional[int]) -> int:
    return _lib.fn_quant(y, mode, M, H, out_q, out_scale, stream)


def fn_qk_norm_gate(qkv: int, M: int, row_stride: int, Hq: int, Hk: int, D: int,
                    q_weight: Optional[int], k_weight: Optional[int], eps: float,
                    out_q: Optional[int], out_k: Optional[int], out_gate: Optional[int],
                    stream: Optional[int]) -> int:
    return _lib.fn_qk_norm_gate(qkv, M, row_stride, Hq, Hk, D, q_weight, k_weight, eps, out_q,
                                out_k, out_gate, stream)


def fn_qk_norm_gate_fp8(qkv: int, M: int, row_stride: int, Hq: int, Hk: int, D: int,
                        q_weight: Optional[int], k_weight: Optional[int], eps: float,
                        out_q8: Optional[int], out_q_scale: Optional[int], out_k8: Optional[int],
                        out_k_scale: Optional[int], out_gate: Optional[int],
                        out_q: Optional[int], out_k: Optional[int],
                        stream: Optional[int]) -> int:
    return _lib.fn_qk_norm_gate_fp8(qkv, M, row_stride, Hq, Hk, D, q_weight, k_weight, eps,
                                    out_q8, out_q_scale, out_k8, out_k_scale, out_gate, out_q,
                                    out_k, stream)


def fn_hc_mix(x: int, w_down: int, w_up: int, M: int, hc: int, C: int, r: int,
              out: int, workspace: int, stream: Optional[int]) -> int:
    return _lib.fn_hc_mix(x, w_down, w_up, M, hc, C, r, out, workspace, stream)


def fn_hc_mix_workspace_bytes(M: int, r: int) -> int:
    return _lib.fn_hc_mix_workspace_bytes(M, r)


def fn_hc_mix_noalloc(x: int, w_down: int, w_up: int, M: int, hc: int, C: int, r: int,
                      out: int, stream: Optional[int]) -> int:
    return _lib.fn_hc_mix_noalloc(x, w_down, w_up, M, hc, C, r, out, stream)


def fn_status_string(status: int) -> str:
    return _lib.fn_status_string(status).decode()


def fn_last_variant() -> int:
    return _lib.fn_last_variant()


def fn_last_launch():
    out = (ctypes.c_int32 * 4)()
    _lib.fn_last_launch(out)
    return tuple(out)


def fn_prefer_variant(variant: int) -> int:
    return _lib.fn_prefer_variant(variant)


def fn_programmatic_launch(on: int) -> int:
    return _lib.fn_programmatic_launch(on)


def fn_version() -> int:
    return _lib.fn_version()


class programmatic_launch:
    """Context manager: this thread's calls launch their kernels as
    programmatic dependents of the stream's previous work (see
    fn_programmatic_launch)."""

    def __init__(self, on: bool = True):
        self.on = on

    def __enter__(self):
        self.old = fn_programmatic_launch(1 if self.on else 0)
        return self

    def __exit__(self, *exc):
        fn_programmatic_launch(self.old)


class prefer_variant:
    """Context manager: ask fn_rmsnorm_quant for one kernel on this thread."""

    def __init__(self, variant: int):
        self.variant = variant

    def __enter__(self):
        self.old = fn_prefer_variant(self.variant)
        return self

    def __exit__(self, *exc):
        fn_prefer_variant(self.old)
        return False


# ---- tensor API ----------------------------------------------------------------------

RMSNormQuantOutput = namedtuple("RMSNormQuantOutput", "q scale residual_out y")
QKOutput = namedtuple("QKOutput", "q k gate")
QKFp8Output = namedtuple("QKFp8Output", "q8 q_scale k8 k_scale gate q k")


def _mode(mode: Union[int, str]) -> int:
    return MODES[mode] if isinstance(mode, str) else int(mode)


def _rows(t: torch.Tensor, name: str, H: Optional[int] = None,
          dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if H is not None and t.shape[-1] != H:
        raise ValueError(f"{name} has last dim {t.shape[-1]}, expected {H}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.reshape(-1, t.shape[-1])


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def _row_format(t: torch.Tensor, mode: int):
    """The 16-bit format of a call (bf16, or float16 -> FN_IO_FP16), taken from
    its first input; every other 16-bit tensor must match it."""
    if t.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError(f"rows must be bfloat16 or float16, got {t.dtype}")
    if t.dtype == torch.float16:
        return t.dtype, mode | FN_IO_FP16
    if mode & FN_IO_FP16:
        raise TypeError("FN_IO_FP16 was asked for but the rows are bfloat16")
    return t.dtype, mode


def alloc_outputs(mode: int, M: int, H: int, device) -> tuple:
    """Codes and scales for `mode` (with its layout flag, if any): FP8 codes as
    float8_e4m3fn [M, H]; MXFP4 codes as uint8 [M, H/2]; scales fp32 [M, 1] /
    fp32 [M, H/128] / uint8 E8M0 [M, H/32] row-major, or, with a layout flag,
    the padded buffer that layout needs (zero-filled: padding is not written):
    uint8 [roundup(M,128) * roundup(H/32,4)] for FN_SCALE_SWIZZLE_32_4_4,
    fp32 [H/128, roundup(M,4)] for FN_SCALE_MN_MAJOR."""
    q_mode, flags = mode & FN_MODE_MASK, mode & (FN_SCALE_SWIZZLE_32_4_4 | FN_SCALE_MN_MAJOR)
    if q_mode == FN_MXFP4:
        q = torch.empty((M, H // 2), dtype=torch.uint8, device=device)
        if flags == FN_SCALE_SWIZZLE_32_4_4:
            n = _round_up(M, 128) * _round_up(H // 32, 4)
            return q, torch.zeros((n,), dtype=torch.uint8, device=device)
        return q, torch.empty((M, H // 32), dtype=torch.uint8, device=device)
    q = torch.empty((M, H), dtype=torch.float8_e4m3fn, device=device)
    if q_mode == FN_FP8_PER_TOKEN:
        return q, torch.empty((M, 1), dtype=torch.float32, device=device)
    if flags == FN_SCALE_MN_MAJOR:
        return q, torch.zeros((H // 128, _round_up(M, 4)), dtype=torch.float32, device=device)
    return q, torch.empty((M, H // 128), dtype=torch.float32, device=device)


def rmsnorm_quant(x: Union[torch.Tensor, Sequence[torch.Tensor]], weight: torch.Tensor,
                  eps: float, mode: Union[int, str], residual: Optional[torch.Tensor] = None,
                  *, in_place: bool = False, out_residual: Optional[torch.Tensor] = None,
                  emit_y: bool = False, out_q: Optional[torch.Tensor] = None,
                  out_scale: Optional[torch.Tensor] = None,
                  out_y: Optional[torch.Tensor] = None) -> RMSNormQuantOutput:
    """Fused (sum of partials) + residual add + RMSNorm + quantization.

    x: a bf16 (or float16) CUDA tensor [..., H] or a list of up to 8 such
    partial tensors (summed in the kernel).  With `in_place`, residual_out is
    written into `residual`.  Returns (q, scale, residual_out, y); y is None
    unless `emit_y` (or `out_y`) asks for the normed row.  float16 rows select
    FN_IO_FP16: residual, weight, residual_out and y are then float16 too, so
    the producer's dtype is carried through the tuple.
    """
    parts = list(x) if isinstance(x, (list, tuple)) else [x]
    if not 1 <= len(parts) <= FN_MAX_PARTS:
        raise ValueError("between 1 and 8 partial tensors")
    H = parts[0].shape[-1]
    lead = parts[0].shape[:-1]
    dt, m = _row_format(parts[0], _mode(mode))
    rows = [_rows(p, f"x[{i}]", H, dt) for i, p in enumerate(parts)]
    for r in rows:
        if r.shape != rows[0].shape:
            raise ValueError("all partials must have the same shape")
    M = rows[0].shape[0]
    w = _rows(weight, "weight", H, dt)
    dev = rows[0].device
    res = None if residual is None else _rows(residual, "residual", H, dt)
    if res is not None and res.shape[0] != M:
        raise ValueError("residual rows differ from x rows")
    if in_place:
        if res is None:
            raise ValueError("in_place needs a residual")
        r_out = res
    elif out_residual is not None:
        r_out = _rows(out_residual, "out_residual", H, dt)
    elif res is not None:
        r_out = torch.empty_like(res)
    else:
        r_out = None
    if out_q is None or out_scale is None:
        q, s = alloc_outputs(m, M, H, dev)
        out_q = q if out_q is None else out_q
        out_scale = s if out_scale is None else out_scale
    if out_y is None and emit_y:
        out_y = torch.empty((M, H), dtype=dt, device=dev)
    elif out_y is not None:
        out_y = _rows(out_y, "out_y", H, dt)
    st = fn_rmsnorm_quant([r.data_ptr() for r in rows], len(rows), _ptr(res), w.data_ptr(),
                          float(eps), m, M, H, out_q.data_ptr(), out_scale.data_ptr(),
                          _ptr(r_out), _ptr(out_y), _stream(dev))
    if st != FN_OK:
        raise FusedNormError("fn_rmsnorm_quant", st)
    ro = None if r_out is None else r_out.view(*lead, H)
    yo = None if out_y is None else out_y.view(*lead, H)
    return RMSNormQuantOutput(out_q, out_scale, ro, yo)


def quant(y: torch.Tensor, mode: Union[int, str], *, out_q: Optional[torch.Tensor] = None,
          out_scale: Optional[torch.Tensor] = None):
    """Quantization step alone on bf16 (or float16) rows [..., H]; returns
    (q, scale)."""
    dt, m = _row_format(y, _mode(mode))
    rows = _rows(y, "y", None, dt)
    M, H = rows.shape
    if out_q is None or out_scale is None:
        q, s = alloc_outputs(m, M, H, rows.device)
        out_q = q if out_q is None else out_q
        out_scale = s if out_scale is None else out_scale
    st = fn_quant(rows.data_ptr(), m, M, H, out_q.data_ptr(), out_scale.data_ptr(),
                  _stream(rows.device))
    if st != FN_OK:
        raise FusedNormError("fn_quant", st)
    return out_q, out_scale


def qk_norm_gate(qkv: torch.Tensor, Hq: int, Hk: int, D: int, q_weight: torch.Tensor,
                 k_weight: torch.Tensor, eps: float, *,
                 out: Optional[QKOutput] = None) -> QKOutput:
    """Gemma (1 + w) RMSNorm of q and k heads read from the interleaved
    [q_h0, gate_h0, q_h1, gate_h1, ..., k..., v...] rows of `qkv` [M, row_stride]
    (any row stride, last dim contiguous); returns contiguous q [M,Hq,D],
    k [M,Hk,D] and gate [M,Hq,D]."""
    if not qkv.is_cuda or qkv.dtype != torch.bfloat16:
        raise TypeError("qkv must be a bf16 CUDA tensor")
    if qkv.dim() != 2 or qkv.stride(1) != 1:
        raise ValueError("qkv must be [M, row] with a contiguous last dim")
    M, row_stride = qkv.shape[0], qkv.stride(0)
    if qkv.shape[1] < (2 * Hq + Hk) * D:
        raise ValueError("qkv rows are too short for the heads")
    qw = _rows(q_weight, "q_weight", D)
    kw = _rows(k_weight, "k_weight", D)
    dev = qkv.device
    if out is None:
        out = QKOutput(torch.empty((M, Hq, D), dtype=torch.bfloat16, device=dev),
                       torch.empty((M, Hk, D), dtype=torch.bfloat16, device=dev),
                       torch.empty((M, Hq, D), dtype=torch.bfloat16, device=dev))
    st = fn_qk_norm_gate(qkv.data_ptr(), M, row_stride, Hq, Hk, D, qw.data_ptr(),
                         kw.data_ptr(), float(eps), out.q.data_ptr(), out.k.data_ptr(),
                         out.gate.data_ptr(), _stream(dev))
    if st != FN_OK:
        raise FusedNormError("fn_qk_norm_gate", st)
    return out


def qk_norm_gate_fp8(qkv: torch.Tensor, Hq: int, Hk: int, D: int, q_weight: torch.Tensor,
                     k_weight: torch.Tensor, eps: float, *, emit_bf16: bool = False) -> QKFp8Output:
    """qk_norm_gate with E4M3 q and k (one fp32 scale per token and head);
    returns (q8 [M,Hq,D] float8_e4m3fn, q_scale [M,Hq], k8, k_scale, gate [M,Hq,D]
    bf16, q, k) where q and k are the bf16 normed heads if `emit_bf16`."""
    if not qkv.is_cuda or qkv.dtype != torch.bfloat16:
        raise TypeError("qkv must be a bf16 CUDA tensor")
    if qkv.dim() != 2 or qkv.stride(1) != 1:
        raise ValueError("qkv must be [M, row] with a contiguous last dim")
    M, row_stride = qkv.shape[0], qkv.stride(0)
    if qkv.shape[1] < (2 * Hq + Hk) * D:
        raise ValueError("qkv rows are too short for the heads")
    qw = _rows(q_weight, "q_weight", D)
    kw = _rows(k_weight, "k_weight", D)
    dev = qkv.device
    f8, f32, bf = torch.float8_e4m3fn, torch.float32, torch.bfloat16
    out = QKFp8Output(torch.empty((M, Hq, D), dtype=f8, device=dev),
                      torch.empty((M, Hq), dtype=f32, device=dev),
                      torch.empty((M, Hk, D), dtype=f8, device=dev),
                      torch.empty((M, Hk), dtype=f32, device=dev),
                      torch.empty((M, Hq, D), dtype=bf, device=dev),
                      torch.empty((M, Hq, D), dtype=bf, device=dev) if emit_bf16 else None,
                      torch.empty((M, Hk, D), dtype=bf, device=dev) if emit_bf16 else None)
    st = fn_qk_norm_gate_fp8(qkv.data_ptr(), M, row_stride, Hq, Hk, D, qw.data_ptr(),
                             kw.data_ptr(), float(eps), out.q8.data_ptr(), out.q_scale.data_ptr(),
                             out.k8.data_ptr(), out.k_scale.data_ptr(), out.gate.data_ptr(),
                             _ptr(out.q), _ptr(out.k), _stream(dev))
    if st != FN_OK:
        raise FusedNormError("fn_qk_norm_gate_fp8", st)
    return out


def hc_mix(x: torch.Tensor, w_down: torch.Tensor, w_up: torch.Tensor, *, hc: int = HC_STREAMS,
           out: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Low-rank gate over the hyper-state: x bf16 [M, hc*C] (M <= 16),
    w_down bf16 [r, hc*C], w_up bf16 [hc*C, r]; returns the gated mix of the
    hc streams, bf16 [M, C] (see fn_hc_mix).  The workspace (t, fp32 [M, r]:
    fn_hc_mix_workspace_bytes(M, r) bytes) is allocated with torch unless
    given."""
    for t, n in ((x, "x"), (w_down, "w_down"), (w_up, "w_up")):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous 2-D bf16 CUDA tensor")
    M, K = x.shape
    r = w_down.shape[0]
    if K % hc or w_down.shape[1] != K or tuple(w_up.shape) != (K, r):
        raise ValueError("shapes must be x [M, hc*C], w_down [r, hc*C], w_up [hc*C, r]")
    C = K // hc
    if out is None:
        out = torch.empty((M, C), dtype=torch.bfloat16, device=x.device)
    need = fn_hc_mix_workspace_bytes(M, r)
    if workspace is None:
        workspace = torch.empty((max(1, need // 4),), dtype=torch.float32, device=x.device)
    elif workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace holds fewer than the {need} bytes fn_hc_mix needs")
    st = fn_hc_mix(x.data_ptr(), w_down.data_ptr(), w_up.data_ptr(), M, hc, C, r,
                   out.data_ptr(), workspace.data_ptr(), _stream(x.device))
    if st != FN_OK:
        raise FusedNormError("fn_hc_mix", st)
    return out
