"""Algorithmic work of each hot-path call (closed forms), used by the bench.

Useful FLOP convention: visible (query, key) pairs x 4 x head_dim (QK^T and
PV, forward only, self pairs included).  Algorithmic bytes: what the call
must move at least once (inputs read once, outputs written once).
"""

from __future__ import annotations


def pairs_per_head(L: int, n: int, mode: str, window: int = 0) -> int:
    """Visible (query, key) pairs per (batch, query head).

    intra ("Stream-Factorized Attention", O(nL^2)): n causal streams of L
    tokens, optionally banded to W tokens; cross: one causal sequence of nL
    positions, optionally banded to W positions."""
    if mode == "intra":
        streams, length = n, L
    elif mode == "cross":
        streams, length = 1, n * L
    else:
        raise ValueError(mode)
    W = length if window <= 0 else min(window, length)
    return streams * (W * (W + 1) // 2 + (length - W) * W)


def attn_flops(B: int, L: int, n: int, Hq: int, D: int, mode: str, window: int = 0) -> int:
    return B * Hq * pairs_per_head(L, n, mode, window) * 4 * D


def attn_min_bytes(B: int, L: int, n: int, Hq: int, Hkv: int, D: int, esize: int = 2, out_esize: int = 2) -> int:
    P = n * L
    return B * P * D * (Hq * esize + 2 * Hkv * esize + Hq * out_esize)


def expand_bytes(B: int, L: int, n: int, d: int, esize: int = 2) -> int:
    """Read the gathered table rows once, write the expanded rows, read ids."""
    return 2 * B * L * n * d * esize + 4 * B * L


def gather_bytes(B: int, L: int, d: int, esize: int = 2) -> int:
    return 2 * B * L * d * esize


def decode_bytes(B: int, n: int, T: int, Hq: int, Hkv: int, D: int, esize: int = 2, out_esize: int = 2) -> int:
    """K and V of every visible cache entry once, plus q and O."""
    return 2 * B * n * T * Hkv * D * esize + B * n * Hq * D * (esize + out_esize)


def decode_flops(B: int, n: int, T: int, Hq: int, D: int, mode: str) -> int:
    """Visible pairs per (b, query head, stream) x 4D, summed over the n
    stream queries of the new token."""
    if mode == "intra":
        pairs = n * T
    else:
        # stream s sees n*(T-1) older entries plus s+1 entries of the new token
        pairs = n * n * (T - 1) + n * (n + 1) // 2
    return B * Hq * pairs * 4 * D


def pairs_final_stream(L: int, n: int, mode: str, window: int = 0) -> int:
    """Visible pairs per (batch, query head) when only the final-stream
    queries run (KV-mirror layers): query i sits at position i*n + n-1.
    intra: causal over the final stream's L tokens (window in tokens);
    cross: all positions <= i*n + n-1 (window in positions)."""
    if mode == "intra":
        return pairs_per_head(L, 1, "intra", window)
    if mode != "cross":
        raise ValueError(mode)
    total = 0
    for i in range(L):
        vis = (i + 1) * n
        total += vis if window <= 0 else min(vis, window)
    return total


def attn_flops_final_stream(B: int, L: int, n: int, Hq: int, D: int, mode: str, window: int = 0) -> int:
    return B * Hq * pairs_final_stream(L, n, mode, window) * 4 * D


def attn_bwd_flops(B: int, L: int, n: int, Hq: int, D: int, mode: str, window: int = 0) -> int:
    """Useful backward FLOPs: visible pairs x 10 x head_dim -- five products
    per pair (recomputed scores, dP, dV, dK, dQ), 2 x head_dim each; 2.5x
    the forward's useful FLOPs."""
    return B * Hq * pairs_per_head(L, n, mode, window) * 10 * D


def attn_bwd_exec_flops(B: int, L: int, n: int, Hq: int, D: int, mode: str, window: int = 0) -> int:
    """Tensor-core FLOPs the bf16 backward executes on visible pairs: the
    dK/dV pass forms S, dP, dV, dK and the dQ pass forms S, dP, dQ again, so
    seven products per pair (full 128 x 128 tiles on the diagonal add more)."""
    return B * Hq * pairs_per_head(L, n, mode, window) * 14 * D


def attn_bwd_min_bytes(B: int, L: int, n: int, Hq: int, Hkv: int, D: int, esize: int = 2) -> int:
    """Read q, k, v, o, dO and lse once, write dq, dk, dv once."""
    P = n * L
    return B * P * (D * esize * (3 * Hq + 2 * Hkv + 2 * Hkv + Hq) + 4 * Hq)


def pairs_cross_shard(L: int, n: int, R: int, r: int, window: int = 0) -> int:
    """Visible pairs per (batch, query head) of rank r's queries in a
    cross-stream layer under stream parallelism: positions p = i*n + r + R*l
    see every p' <= p (within the window)."""
    nl = n // R
    total = 0
    for i in range(L):
        for l in range(nl):
            vis = i * n + r + R * l + 1
            total += vis if window <= 0 else min(vis, window)
    return total
