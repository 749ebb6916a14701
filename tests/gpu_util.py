"""Shared helpers for the GPU parity tests (host-side only)."""

import numpy as np
import torch

from stream_sequence_attention_b200 import synth

# Parity bounds.  float32 inputs: max-abs 1e-4; bf16 inputs with fp32
# accumulation: max-abs 2e-2 (both against the float64 oracle).
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def lib():
    from stream_sequence_attention_b200 import build as hd_build
    hd_build.build()
    from stream_sequence_attention_b200 import hd
    hd.lib()
    return hd


def host_qkv(B, P, Hq, Hkv, D, seed, dtype):
    q = synth.normal((B, P, Hq, D), seed, dtype=dtype)
    k = synth.normal((B, P, Hkv, D), seed + 1, dtype=dtype)
    v = synth.normal((B, P, Hkv, D), seed + 2, dtype=dtype)
    return q, k, v


def dev(x, dtype):
    return synth.to_torch(x, dtype, "cuda")


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))


class Guarded:
    """A device tensor of ``shape``/``dtype`` inside a larger byte buffer with
    ``guard`` bytes before and after it, the whole buffer filled with the
    canary byte ``fill``.  After a call writes the tensor, ``guards_intact``
    says whether any byte outside it changed (an out-of-bounds write), and
    ``fully_written`` whether every element was overwritten (no element still
    holds the canary pattern in all of its bytes)."""

    def __init__(self, shape, dtype, guard=1 << 16, fill=0xA5, init=None):
        esz = torch.empty((), dtype=dtype).element_size()
        numel = 1
        for s in shape:
            numel *= s
        self.esz, self.guard, self.fill, self.nbytes = esz, guard, fill, numel * esz
        self.raw = torch.full((2 * guard + self.nbytes,), fill, dtype=torch.uint8, device="cuda")
        self.t = self.raw[guard:guard + self.nbytes].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init)
        assert self.t.data_ptr() % 256 == 0

    def guards_intact(self) -> bool:
        torch.cuda.synchronize()
        g = self.guard
        return bool((self.raw[:g] == self.fill).all()) and bool((self.raw[g + self.nbytes:] == self.fill).all())

    def fully_written(self) -> bool:
        torch.cuda.synchronize()
        body = self.raw[self.guard:self.guard + self.nbytes].view(-1, self.esz)
        return not bool((body == self.fill).all(dim=1).any())
