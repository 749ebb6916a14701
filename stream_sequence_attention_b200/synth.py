"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module draws random numbers and casts them; it holds none of the
method's arithmetic.  Two sources:

* host draws with ``numpy.random.Generator(PCG64(seed))`` in float32, cast
  to bfloat16 with round-to-nearest-even when asked (small and medium cases,
  where the oracle needs every value);
* device draws with a seeded ``torch.Generator`` on the GPU (full-size cases,
  where only sampled rows are copied back to the host for checking).
"""

from __future__ import annotations

import numpy as np


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 value (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    nan = np.isnan(x)
    out = (rounded.astype(np.uint32) << 16).view(np.float32)
    out = np.where(nan, np.float32(np.nan), out)
    return out.astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def normal(shape, seed: int, std: float = 1.0, dtype: str = "f32") -> np.ndarray:
    """N(0, std^2) samples in float32; ``dtype='bf16'`` rounds them to bf16."""
    x = rng(seed).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x = (x * np.float32(std)).astype(np.float32)
    if dtype == "bf16":
        x = bf16_round(x)
    return x


def ids_uniform(B: int, L: int, V: int, seed: int) -> np.ndarray:
    return rng(seed).integers(0, V, size=(B, L), dtype=np.int32)


def ids_zipf(B: int, L: int, V: int, alpha: float, seed: int) -> np.ndarray:
    """Token ids with P(rank r) proportional to r^-alpha, r = 1..V, drawn by
    inverse CDF; rank r is mapped to an id through a seeded permutation."""
    g = rng(seed)
    r = np.arange(1, V + 1, dtype=np.float64)
    cdf = np.cumsum(r ** (-alpha))
    cdf /= cdf[-1]
    u = g.random(size=(B, L))
    rank = np.searchsorted(cdf, u, side="right")
    rank = np.minimum(rank, V - 1)
    perm = g.permutation(V).astype(np.int32)
    return perm[rank].astype(np.int32)


def to_torch(x: np.ndarray, dtype: str, device="cpu"):
    """Host array -> torch tensor of the requested element type (exact)."""
    import torch

    if dtype == "bf16":
        t = torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16)
    elif dtype == "f32":
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    elif dtype == "i32":
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32))
    else:
        raise ValueError(dtype)
    return t.to(device)


def normal_device(shape, seed: int, std: float = 1.0, dtype: str = "bf16",
                  device="cuda", chunk: int = 1 << 28):
    """N(0, std^2) drawn on the device by a seeded torch generator, cast to
    ``dtype`` (round to nearest even).  Generated in chunks so no float32
    copy of the whole tensor is needed."""
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty(shape, dtype=tdt, device=device)
    flat = out.view(-1)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        x = torch.randn(e - s, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[s:e].copy_(x)
    return out
