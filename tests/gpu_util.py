"""Helpers for the GPU tests: the library handle, host copies, guarded outputs."""
import numpy as np
import torch

from mxfp4_quantization_b200 import synth

GUARD = 4096  # bytes of canary on each side of a guarded output
CANARY = 0xA5


def lib():
    from mxfp4_quantization_b200.build import build_library
    build_library()
    from mxfp4_quantization_b200 import fusednorm
    return fusednorm


def bits(t):
    return None if t is None else synth.to_bits(t)


def u8(t):
    return t.detach().to("cpu").contiguous().view(torch.uint8).numpy()


def scale_np(t, mode):
    t = t.detach().to("cpu").contiguous()
    return t.view(torch.uint8).numpy() if mode == synth.MXFP4 else t.numpy().astype(np.float32)


class Guarded:
    """A device buffer with canary bytes before and after the usable region,
    to catch writes outside an output (compute-sanitizer stand-in)."""

    def __init__(self, shape, dtype, device="cuda"):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.uint8, device=device)
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self) -> bool:
        r = self.raw.to("cpu").numpy()
        return bool(np.all(r[:GUARD] == CANARY) and np.all(r[GUARD + self.n:] == CANARY))

    def untouched(self) -> bool:
        return bool(np.all(self.raw.to("cpu").numpy() == CANARY))
