"""ctypes wrapper of the C oracle (orc.c).  Test infrastructure only."""
import ctypes
import os

import numpy as np

from .build import LIB, build_oracle

FP8_PER_TOKEN = 0
FP8_PER_GROUP128 = 1
MXFP4 = 2

# storage format of the 16-bit tensors
IO_BF16 = 0
IO_FP16 = 1

_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)


class OracleError(RuntimeError):
    pass


def load(path: str = LIB):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is not None and path == LIB:
        return _lib
    build_oracle() if path == LIB else None
    lib = ctypes.CDLL(os.path.abspath(path))
    lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_double.restype = ctypes.c_double
    lib.orc_bf16_from_double.argtypes = [ctypes.c_double]
    lib.orc_bf16_from_double.restype = ctypes.c_uint16
    lib.orc_fp16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_fp16_to_double.restype = ctypes.c_double
    lib.orc_fp16_from_double.argtypes = [ctypes.c_double]
    lib.orc_fp16_from_double.restype = ctypes.c_uint16
    lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_decode.restype = ctypes.c_double
    lib.orc_e4m3_encode.argtypes = [ctypes.c_double]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
    lib.orc_e2m1_decode.restype = ctypes.c_double
    lib.orc_e2m1_encode.argtypes = [ctypes.c_double]
    lib.orc_e2m1_encode.restype = ctypes.c_uint8
    lib.orc_mx_scale_code.argtypes = [ctypes.c_double]
    lib.orc_mx_scale_code.restype = ctypes.c_uint8
    lib.orc_rstd.argtypes = [_u16p, ctypes.c_int64, ctypes.c_float, ctypes.c_int]
    lib.orc_rstd.restype = ctypes.c_double
    lib.orc_quant_rows.argtypes = [_u16p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                   _u8p, ctypes.c_void_p, ctypes.c_int]
    lib.orc_quant_rows.restype = ctypes.c_int
    lib.orc_rmsnorm_quant.argtypes = [ctypes.POINTER(_u16p), ctypes.c_int, _u16p, _u16p,
                                      ctypes.c_float, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_int64, _u8p, ctypes.c_void_p, _u16p, _u16p,
                                      ctypes.c_int]
    lib.orc_rmsnorm_quant.restype = ctypes.c_int
    lib.orc_qk_norm_gate.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, _u16p, _u16p,
                                     ctypes.c_float, _u16p, _u16p, _u16p]
    lib.orc_qk_norm_gate.restype = ctypes.c_int
    _f32p = ctypes.POINTER(ctypes.c_float)
    lib.orc_qk_norm_gate_fp8.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _u16p, _u16p,
                                         ctypes.c_float, _u8p, _f32p, _u8p, _f32p, _u16p,
                                         _u16p, _u16p]
    lib.orc_qk_norm_gate_fp8.restype = ctypes.c_int
    lib.orc_hc_mix.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int,
                               ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                               _u16p]
    lib.orc_hc_mix.restype = ctypes.c_int
    if path == LIB:
        _lib = lib
    return lib


def _p16(a):
    return None if a is None else a.ctypes.data_as(_u16p)


def _p8(a):
    return a.ctypes.data_as(_u8p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 arrays travel as uint16 bit patterns")
    return a


def scale_shape(mode: int, M: int, H: int):
    return {FP8_PER_TOKEN: (M,), FP8_PER_GROUP128: (M, H // 128), MXFP4: (M, H // 32)}[mode]


def code_shape(mode: int, M: int, H: int):
    return (M, H // 2) if mode == MXFP4 else (M, H)


def _scale_dtype(mode):
    return np.uint8 if mode == MXFP4 else np.float32


# ---- scalar format helpers (vectorised over numpy inputs) -------------------

def bf16_to_double(bits, lib=None):
    lib = lib or load()
    return np.array([lib.orc_bf16_to_double(int(b)) for b in np.ravel(bits)]).reshape(np.shape(bits))


def bf16_from_double(v, lib=None):
    lib = lib or load()
    return np.array([lib.orc_bf16_from_double(float(x)) for x in np.ravel(v)],
                    dtype=np.uint16).reshape(np.shape(v))


def fp16_to_double(bits, lib=None):
    lib = lib or load()
    return np.array([lib.orc_fp16_to_double(int(b)) for b in np.ravel(bits)]).reshape(np.shape(bits))


def fp16_from_double(v, lib=None):
    lib = lib or load()
    return np.array([lib.orc_fp16_from_double(float(x)) for x in np.ravel(v)],
                    dtype=np.uint16).reshape(np.shape(v))


def e4m3_encode(v, lib=None):
    lib = lib or load()
    return np.array([lib.orc_e4m3_encode(float(x)) for x in np.ravel(v)],
                    dtype=np.uint8).reshape(np.shape(v))


def e4m3_decode(c, lib=None):
    lib = lib or load()
    return np.array([lib.orc_e4m3_decode(int(x)) for x in np.ravel(c)]).reshape(np.shape(c))


def e2m1_encode(v, lib=None):
    lib = lib or load()
    return np.array([lib.orc_e2m1_encode(float(x)) for x in np.ravel(v)],
                    dtype=np.uint8).reshape(np.shape(v))


def e2m1_decode(c, lib=None):
    lib = lib or load()
    return np.array([lib.orc_e2m1_decode(int(x)) for x in np.ravel(c)]).reshape(np.shape(c))


def mx_scale_code(amax, lib=None):
    lib = lib or load()
    return np.array([lib.orc_mx_scale_code(float(x)) for x in np.ravel(amax)],
                    dtype=np.uint8).reshape(np.shape(amax))


# ---- row operations ---------------------------------------------------------

def rstd(h_bits, eps: float, lib=None, io: int = IO_BF16) -> float:
    lib = lib or load()
    h = _u16(h_bits)
    return lib.orc_rstd(_p16(h), h.size, eps, io)


def quant_rows(y_bits, mode: int, lib=None, io: int = IO_BF16):
    """Quantize 16-bit rows [M, H] (bf16, or binary16 with io=IO_FP16);
    returns (codes, scales)."""
    lib = lib or load()
    y = _u16(y_bits)
    M, H = y.shape
    q = np.zeros(code_shape(mode, M, H), dtype=np.uint8)
    s = np.zeros(scale_shape(mode, M, H), dtype=_scale_dtype(mode))
    rc = lib.orc_quant_rows(_p16(y), mode, M, H, _p8(q), s.ctypes.data_as(ctypes.c_void_p), io)
    if rc != 0:
        raise OracleError(f"orc_quant_rows rejected mode={mode} H={H}")
    return q, s


def rmsnorm_quant(parts, residual, weight, eps: float, mode: int, lib=None,
                  io: int = IO_BF16):
    """Unfused reference sequence over [M, H] rows.

    parts: list of P uint16 [M, H] arrays; residual: uint16 [M, H] or None;
    weight: uint16 [H]; all bf16 bit patterns, or binary16 with io=IO_FP16.
    Returns dict(q, scale, residual_out, y).
    """
    lib = lib or load()
    parts = [_u16(p) for p in parts]
    M, H = parts[0].shape
    arr = (_u16p * len(parts))(*[_p16(p) for p in parts])
    res = None if residual is None else _u16(residual)
    w = _u16(weight)
    q = np.zeros(code_shape(mode, M, H), dtype=np.uint8)
    s = np.zeros(scale_shape(mode, M, H), dtype=_scale_dtype(mode))
    r_out = np.zeros((M, H), dtype=np.uint16)
    y = np.zeros((M, H), dtype=np.uint16)
    rc = lib.orc_rmsnorm_quant(arr, len(parts), _p16(res), _p16(w), eps, mode, M, H, _p8(q),
                               s.ctypes.data_as(ctypes.c_void_p), _p16(r_out), _p16(y), io)
    if rc != 0:
        raise OracleError(f"orc_rmsnorm_quant rejected P={len(parts)} mode={mode} H={H}")
    return {"q": q, "scale": s, "residual_out": r_out, "y": y}


def qk_norm_gate(qkv, row_stride: int, Hq: int, Hk: int, D: int, q_weight, k_weight,
                 eps: float, lib=None):
    """qkv: uint16 [M, row_stride]; returns dict(q [M,Hq,D], k [M,Hk,D], gate [M,Hq,D])."""
    lib = lib or load()
    x = _u16(qkv)
    M = x.shape[0]
    q = np.zeros((M, Hq, D), dtype=np.uint16)
    k = np.zeros((M, Hk, D), dtype=np.uint16)
    g = np.zeros((M, Hq, D), dtype=np.uint16)
    rc = lib.orc_qk_norm_gate(_p16(x), M, row_stride, Hq, Hk, D, _p16(_u16(q_weight)),
                              _p16(_u16(k_weight)), eps, _p16(q), _p16(k), _p16(g))
    if rc != 0:
        raise OracleError("orc_qk_norm_gate rejected the shape")
    return {"q": q, "k": k, "gate": g}


def qk_norm_gate_fp8(qkv, row_stride: int, Hq: int, Hk: int, D: int, q_weight, k_weight,
                     eps: float, lib=None):
    """Returns dict(q8, qs, k8, ks, gate, q, k) (see orc_qk_norm_gate_fp8)."""
    lib = lib or load()
    x = _u16(qkv)
    M = x.shape[0]
    f32p = ctypes.POINTER(ctypes.c_float)
    out = {"q8": np.zeros((M, Hq, D), np.uint8), "qs": np.zeros((M, Hq), np.float32),
           "k8": np.zeros((M, Hk, D), np.uint8), "ks": np.zeros((M, Hk), np.float32),
           "gate": np.zeros((M, Hq, D), np.uint16), "q": np.zeros((M, Hq, D), np.uint16),
           "k": np.zeros((M, Hk, D), np.uint16)}
    rc = lib.orc_qk_norm_gate_fp8(_p16(x), M, row_stride, Hq, Hk, D, _p16(_u16(q_weight)),
                                  _p16(_u16(k_weight)), eps, _p8(out["q8"]),
                                  out["qs"].ctypes.data_as(f32p), _p8(out["k8"]),
                                  out["ks"].ctypes.data_as(f32p), _p16(out["gate"]),
                                  _p16(out["q"]), _p16(out["k"]))
    if rc != 0:
        raise OracleError("orc_qk_norm_gate_fp8 rejected the shape")
    return out


def hc_mix(x, w_down, w_up, hc: int, C: int, r: int, lib=None):
    """Low-rank gate over the hyper-state (reading A19 of orc.c).

    x: uint16 bf16 [M, hc*C]; w_down: uint16 bf16 [r, hc*C]; w_up: uint16 bf16
    [hc*C, r].  Returns (u fp64 [M, C], u_bf16 uint16 [M, C])."""
    lib = lib or load()
    xx, wd, wu = _u16(x), _u16(w_down), _u16(w_up)
    M = xx.shape[0]
    if xx.shape[1] != hc * C or wd.shape != (r, hc * C) or wu.shape != (hc * C, r):
        raise OracleError("hc_mix: shapes do not match hc, C, r")
    u = np.zeros((M, C), dtype=np.float64)
    ub = np.zeros((M, C), dtype=np.uint16)
    rc = lib.orc_hc_mix(_p16(xx), _p16(wd), _p16(wu), M, hc, C, r,
                        u.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), _p16(ub))
    if rc != 0:
        raise OracleError("orc_hc_mix rejected the shape")
    return u, ub


# ---- scale layouts ------------------------------------------------------------

SCALE_SWIZZLE_32_4_4 = 0x100
SCALE_MN_MAJOR = 0x200


def _round_up(x, m):
    return (x + m - 1) // m * m


def place_scales(scales, layout: int, fill=0):
    """Row-major scales [M, G] -> the flat buffer of `layout`.

    SCALE_SWIZZLE_32_4_4: [M, G] padded to [roundup(M,128), roundup(G,4)] and
    cut into 128 x 4 tiles of 512 entries, tiles in row-tile-major order;
    inside a tile, row r and group c sit at (r % 32) * 16 + (r // 32) * 4 + c.
    SCALE_MN_MAJOR: [G, roundup(M,4)], entry (g, m) = scale of row m, group g.
    Padding entries hold `fill`.
    """
    scales = np.asarray(scales)
    M, G = scales.shape
    if layout == SCALE_SWIZZLE_32_4_4:
        Mp, Gp = _round_up(M, 128), _round_up(G, 4)
        out = np.full(Mp * Gp, fill, dtype=scales.dtype)
        ct = Gp // 4
        for m in range(M):
            for g in range(G):
                off = ((m // 128) * ct + g // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + g % 4
                out[off] = scales[m, g]
        return out
    if layout == SCALE_MN_MAJOR:
        Mp = _round_up(M, 4)
        out = np.full((G, Mp), fill, dtype=scales.dtype)
        out[:, :M] = scales.T
        return out.reshape(-1)
    raise OracleError(f"unknown scale layout {layout:#x}")
