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
