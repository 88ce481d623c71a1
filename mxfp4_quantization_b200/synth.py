"""Seeded synthetic inputs for the fused RMSNorm + quantization path.

This module only draws random numbers and casts them to bf16 (or float16)
with torch; it
holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can be fed from it.  Every tensor gets its own seed, derived from the
workload seed and the tensor's name, so a sub-range of rows can be regenerated
on its own and a tensor never depends on the order in which others were drawn.

Recipes (shapes follow the pages' models: hidden size 7168 from the fused
AllReduce + RMSNorm + quant PR's 1-stage MXFP4 heuristic, head_dim 256 with
interleaved gate heads from the fused QK-norm + gate PR):

  per_token_small   M=16, H=2048, P=1; x, residual ~ N(0,1); w = 1 + 0.1 N(0,1)
  decode            M in {1,2,4,8,16}, H=7168; x ~ N(0,1) with 1 % of entries
                    (Bernoulli(0.01)) multiplied by 20; residual ~ N(0,1);
                    w = 1 + 0.1 N(0,1)
  qk_prologue       M in {4, 64}; 32 q heads interleaved with 32 gate heads,
                    4 k heads (then 4 v heads, never read), head_dim 256;
                    qkv ~ N(0,1); w ~ 0.1 N(0,1)
  prefill_mxfp4     M=8192, H=7168, P=4 partial buffers, each N(0,1) * c_j
                    with one per-channel scale c_j = 10^U(-1,1) shared by all
                    partials; residual ~ N(0,1); w = 1 + 0.1 N(0,1)
  prefill_group128  M=32768, H=8192, P=1; x = 2 N(0,1); residual ~ N(0,1);
                    w = 1 + 0.1 N(0,1); residual updated in place
  hc_mix            M in {1,2,4,8,16} rows of the hyper-state, hc = 4 streams of
                    C = 2560 (the hc_mix PR's [M, 4*2560]), rank r = 64;
                    x ~ N(0,1); W_down [r, hc*C] ~ N(0,1) / sqrt(hc*C);
                    W_up [hc*C, r] ~ N(0,1) / sqrt(r) (unit-variance gate
                    logits, so the gates spread over (0, 1))
"""
import zlib
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

FP8_PER_TOKEN = 0
FP8_PER_GROUP128 = 1
MXFP4 = 2


def tensor_seed(seed: int, name: str) -> int:
    """Stable per-tensor seed (independent of draw order)."""
    return (int(seed) * 1_000_003 + zlib.crc32(name.encode())) % (2 ** 63)


def _gen(device, seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, name))
    return g


def normal_bf16(shape, seed: int, name: str, std: float = 1.0, mean: float = 0.0,
                device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(device, seed, name)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (t * std + mean).to(dtype)


def normal_with_outliers_bf16(shape, seed: int, name: str, frac: float, mult: float,
                              device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(device, seed, name)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(shape, generator=g, device=device) < frac
    return torch.where(mask, t * mult, t).to(dtype)


def channel_scale(H: int, seed: int, name: str, decades: float, device="cpu") -> torch.Tensor:
    """c_j = 10^U(-decades, decades), fp32 [H]."""
    g = _gen(device, seed, name)
    u = torch.rand((H,), generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
    return torch.pow(10.0, u * decades)


@dataclass
class RowWorkload:
    name: str
    M: int
    H: int
    P: int
    mode: int
    eps: float
    seed: int = 0
    outlier_frac: float = 0.0
    outlier_mult: float = 20.0
    x_std: float = 1.0
    channel_decades: float = 0.0
    residual: bool = True
    in_place: bool = False
    dtype: torch.dtype = torch.bfloat16  # of every 16-bit tensor (float16: binary16 rows)

    def inputs(self, device="cpu", rows: Optional[slice] = None, M: Optional[int] = None):
        """Draw the inputs. `M` overrides the row count (same recipe)."""
        M = self.M if M is None else M
        H, s, dt = self.H, self.seed, self.dtype
        shape = (M, H)
        if self.channel_decades > 0:
            c = channel_scale(H, s, "channel", self.channel_decades, device)
            parts = []
            for p in range(self.P):
                g = _gen(device, s, f"part{p}")
                t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
                parts.append((t * c[None, :]).to(dt))
        elif self.outlier_frac > 0:
            parts = [normal_with_outliers_bf16(shape, s, f"part{p}", self.outlier_frac,
                                               self.outlier_mult, device, dt)
                     for p in range(self.P)]
        else:
            parts = [normal_bf16(shape, s, f"part{p}", std=self.x_std, device=device, dtype=dt)
                     for p in range(self.P)]
        residual = (normal_bf16(shape, s, "residual", device=device, dtype=dt)
                    if self.residual else None)
        weight = normal_bf16((H,), s, "weight", std=0.1, mean=1.0, device=device, dtype=dt)
        return {"parts": parts, "residual": residual, "weight": weight}

    def bytes_per_row(self) -> int:
        """Algorithmic HBM bytes per row: P*2H + 2H (residual) read,
        2H residual_out + codes + scales written (no bf16 y sidecar)."""
        H = self.H
        rd = self.P * 2 * H + (2 * H if self.residual else 0)
        wr = (2 * H if self.residual else 0)
        if self.mode == MXFP4:
            wr += H // 2 + H // 32
        elif self.mode == FP8_PER_GROUP128:
            wr += H + 4 * (H // 128)
        else:
            wr += H + 4
        return rd + wr

    def bytes_per_call(self, M: Optional[int] = None) -> int:
        M = self.M if M is None else M
        return M * self.bytes_per_row() + 2 * self.H


@dataclass
class QKWorkload:
    name: str
    M: int
    Hq: int = 32
    Hk: int = 4
    Hv: int = 4
    D: int = 256
    eps: float = 1e-6
    seed: int = 0

    @property
    def row_stride(self) -> int:
        return (2 * self.Hq + self.Hk + self.Hv) * self.D

    def inputs(self, device="cpu", M: Optional[int] = None):
        M = self.M if M is None else M
        s = self.seed
        qkv = normal_bf16((M, self.row_stride), s, "qkv", device=device)
        qw = normal_bf16((self.D,), s, "q_weight", std=0.1, device=device)
        kw = normal_bf16((self.D,), s, "k_weight", std=0.1, device=device)
        return {"qkv": qkv, "q_weight": qw, "k_weight": kw}

    def bytes_per_call(self, M: Optional[int] = None) -> int:
        """Read q, gate and k heads; write q, k, gate; plus both weights."""
        M = self.M if M is None else M
        per_tok = 2 * self.D * (2 * self.Hq + self.Hk) * 2
        return M * per_tok + 2 * 2 * self.D


@dataclass
class HCWorkload:
    """Inputs of the low-rank gate over the hyper-state (hc_mix)."""
    name: str
    M: int
    hc: int = 4
    C: int = 2560
    r: int = 64
    seed: int = 0

    @property
    def K(self) -> int:
        return self.hc * self.C

    def inputs(self, device="cpu", M: Optional[int] = None):
        M = self.M if M is None else M
        s, K, r = self.seed, self.K, self.r
        x = normal_bf16((M, K), s, "x", device=device)
        w_down = normal_bf16((r, K), s, "w_down", std=K ** -0.5, device=device)
        w_up = normal_bf16((K, r), s, "w_up", std=r ** -0.5, device=device)
        return {"x": x, "w_down": w_down, "w_up": w_up}

    def weight_bytes(self) -> int:
        return 2 * (2 * self.K * self.r)

    def bytes_per_call(self, M: Optional[int] = None) -> int:
        """Algorithmic HBM bytes: both weight factors, the hyper-state rows
        and the mixed output (bf16 each)."""
        M = self.M if M is None else M
        return self.weight_bytes() + M * self.K * 2 + M * self.C * 2


HC_M = (1, 2, 4, 8, 16)


def hc_mix(M: int) -> HCWorkload:
    return HCWorkload(f"hc_mix_m{M}", M=M, seed=5)


PER_TOKEN_SMALL = RowWorkload("per_token_small", M=16, H=2048, P=1, mode=FP8_PER_TOKEN,
                              eps=1e-6, seed=0)
DECODE_M = (1, 2, 4, 8, 16)


def decode(M: int, mode: int) -> RowWorkload:
    return RowWorkload(f"decode_m{M}_mode{mode}", M=M, H=7168, P=1, mode=mode, eps=1e-6,
                       seed=1, outlier_frac=0.01, outlier_mult=20.0)


QK_M = (4, 64)


def qk_prologue(M: int) -> QKWorkload:
    return QKWorkload(f"qk_prologue_m{M}", M=M, seed=2)


PREFILL_MXFP4 = RowWorkload("prefill_mxfp4", M=8192, H=7168, P=4, mode=MXFP4, eps=1e-6,
                            seed=3, channel_decades=1.0)
PREFILL_GROUP128 = RowWorkload("prefill_group128", M=32768, H=8192, P=1,
                               mode=FP8_PER_GROUP128, eps=1e-5, seed=4, x_std=2.0,
                               in_place=True)


def to_bits(t: torch.Tensor):
    """bf16 / float16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    import numpy as np
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
