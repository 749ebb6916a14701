"""Pure-Python brute force of Stream-Factorized Attention for tiny shapes.

TEST INFRASTRUCTURE ONLY.  Written independently of ``hd_oracle``: it uses
the pages' own 1-based index maps ("Hidden Decoding at Scale",
"Stream-Factorized Attention": i(t) = ceil(t/n), s(t) = (t-1) mod n + 1) and
explicit loops with ``math.exp``/``math.log``, so an index, sign or operand
mistake in either implementation shows up as a disagreement.
"""

from __future__ import annotations

import math


def _i(t, n):
    return -(-t // n)  # ceil(t / n)


def _s(t, n):
    return (t - 1) % n + 1


def _allowed(t, u, n, mode, window):
    """Figure 2: (c) intra-stream, (a) full cross-stream, (b) local window."""
    if mode == "intra":
        if _s(u, n) != _s(t, n) or _i(u, n) > _i(t, n):
            return False
        return window == 0 or _i(t, n) - _i(u, n) < window
    if u > t:
        return False
    return window == 0 or t - u < window


def attn(q, k, v, n, mode, window=0, scale=None):
    """q[b][p][h][d], k/v[b][p][kvh][d] nested lists (or arrays).
    Returns (out[b][p][h][d], lse[b][h][p]) as nested lists of floats."""
    B = len(q)
    P = len(q[0])
    Hq = len(q[0][0])
    D = len(q[0][0][0])
    Hkv = len(k[0][0])
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = [[[[0.0] * D for _ in range(Hq)] for _ in range(P)] for _ in range(B)]
    lse = [[[0.0] * P for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for t in range(1, P + 1):
                keys = [u for u in range(1, P + 1) if _allowed(t, u, n, mode, window)]
                sc = []
                for u in keys:
                    acc = 0.0
                    for d in range(D):
                        acc += float(q[b][t - 1][h][d]) * float(k[b][u - 1][g][d])
                    sc.append(scale * acc)
                mx = max(sc)
                e = [math.exp(x - mx) for x in sc]
                z = sum(e)
                for d in range(D):
                    acc = 0.0
                    for w, u in zip(e, keys):
                        acc += (w / z) * float(v[b][u - 1][g][d])
                    out[b][t - 1][h][d] = acc
                lse[b][h][t - 1] = mx + math.log(z)
    return out, lse
