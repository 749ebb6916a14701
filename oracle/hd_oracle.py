"""Plain, slow, float64 definition of the Hidden Decoding hot path.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every routine follows
its definition literally: build the visible set from the index maps, take
scores, softmax over the visible set, weight the values.  No blocking, no
online softmax, no reordering beyond what a numpy matmul does internally.

Indexing is 0-based throughout: token i in [0, L), stream s in [0, n), physical
position p = i*n + s.  This is the pages' t = (i-1)n + k with i -> i+1 and
k -> s+1 ("Hidden Decoding at Scale", "Multi-Stream Expansion and Training
Objective").  The final stream is s = n-1.

Readings where the pages are silent (each listed in the design notes):
  * window W: intra-stream layers count W in tokens of the stream
    (key (j,s) visible to query (i,s) iff i-W < j <= i); cross-stream layers
    count W in physical positions (p-W < p' <= p).  W = 0 means no window.
  * GQA: query head h reads KV head h // (Hq // Hkv).
  * decode: ctx_len counts tokens per stream including the new one; the new
    token's stream s sees the new token's streams s' <= s in cross mode
    (causal in p), i.e. exactly the prefill row of that position.
  * lse is the natural-log log-sum-exp of the scaled visible scores.
  * RoPE: the pages fix only the positions (contiguous over the expanded
    sequence); the rotation is the standard rotary embedding with
    theta_j = base^(-2j/rot_dim), in either pairing convention.
"""

from __future__ import annotations

import numpy as np

INTRA = "intra"
CROSS = "cross"


def _mode(mode) -> str:
    if mode in (INTRA, 0):
        return INTRA
    if mode in (CROSS, 1):
        return CROSS
    raise ValueError(f"unknown mode {mode!r}")


def token_index(p, n):
    """i(t) = ceil(t/n) of "Stream-Factorized Attention", 0-based: p // n."""
    return np.asarray(p) // n


def stream_index(p, n):
    """s(t) = (t-1) mod n + 1 of "Stream-Factorized Attention", 0-based: p % n."""
    return np.asarray(p) % n


def visible(p, pk, n, mode, window=0):
    """True where key position ``pk`` is visible to query position ``p``.

    Figure 2 of "Stream-Factorized Attention":
      (c) intra-stream: same stream and earlier-or-equal token
          (optionally within ``window`` tokens of that stream);
      (a) full cross-stream: standard causal over the interleaved order;
      (b) local cross-stream: causal with a sliding window of ``window``
          physical positions.
    Broadcasts over array arguments.
    """
    mode = _mode(mode)
    p = np.asarray(p)
    pk = np.asarray(pk)
    if mode == INTRA:
        i, s = token_index(p, n), stream_index(p, n)
        j, sk = token_index(pk, n), stream_index(pk, n)
        ok = (sk == s) & (j <= i)
        if window:
            ok = ok & (i - j < window)
    else:
        ok = pk <= p
        if window:
            ok = ok & (p - pk < window)
    return ok


def visible_matrix(L, n, mode, window=0):
    """[nL, nL] boolean mask, row = query position, column = key position."""
    P = n * L
    p = np.arange(P)[:, None]
    pk = np.arange(P)[None, :]
    return visible(p, pk, n, mode, window)


def pair_count(L, n, mode, window=0):
    """Number of visible (query, key) pairs per (batch, query head), counted by
    enumerating the mask.  Useful FLOP = pairs * 4 * head_dim (QK^T and PV,
    forward only, self pairs included)."""
    total = 0
    P = n * L
    pk = np.arange(P)
    for p in range(P):
        total += int(np.count_nonzero(visible(p, pk, n, mode, window)))
    return total


def expand(tables, ids):
    """S_t = E_k(x_i) ("Multi-Stream Expansion and Training Objective").

    tables: [n, V, d]; ids: [B, L] integers in [0, V).
    Returns out [B, n*L, d] with out[b, i*n + s] = tables[s, ids[b, i]].
    Raises on an out-of-range id.
    """
    tables = np.asarray(tables)
    ids = np.asarray(ids)
    n, V, d = tables.shape
    B, L = ids.shape
    if ids.size and (ids.min() < 0 or ids.max() >= V):
        raise ValueError("token id out of range")
    out = np.empty((B, n * L, d), dtype=tables.dtype)
    for b in range(B):
        for i in range(L):
            for s in range(n):
                out[b, i * n + s] = tables[s, ids[b, i]]
    return out


def final_stream_gather(h, n):
    """Rows of the final stream, the only ones fed to the shared LM head
    ("Multi-Stream Expansion and Training Objective"; Figure 1).

    h: [B, n*L, d] -> out [B, L, d], out[b, i] = h[b, i*n + n - 1].
    """
    h = np.asarray(h)
    B, P, d = h.shape
    if P % n:
        raise ValueError("sequence length is not a multiple of n")
    L = P // n
    out = np.empty((B, L, d), dtype=h.dtype)
    for b in range(B):
        for i in range(L):
            out[b, i] = h[b, i * n + n - 1]
    return out


def rope_angles(positions, rot_dim, base):
    """theta_j = base^(-2j/rot_dim), j < rot_dim/2; returns positions[:, None] * theta
    in float64 (the rotary embedding of Su et al., "RoFormer")."""
    j = np.arange(rot_dim // 2, dtype=np.float64)
    theta = float(base) ** (-2.0 * j / rot_dim)
    return np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]


def rope(x, rot_dim, base=10000.0, layout="half", pos_base=0, pos_mult=0, pos0=None):
    """Rotary position embedding over the expanded sequence, float64.

    "Multi-Stream Expansion and Training Objective": the expanded sequence
    runs with contiguous RoPE positions, so row r of sequence b sits at
    position p = pos_base + pos_mult * pos0[b] + r (pos0 = None: 0); for a
    prefill [B, nL, H, D] with pos_base = 0 that is p = i*n + s.  The first
    rot_dim features are rotated pairwise by the angle p * theta_j:
      layout "half":        pairs (j, j + rot_dim/2)
      layout "interleaved": pairs (2j, 2j + 1)
    (x_a, x_b) -> (x_a cos - x_b sin, x_a sin + x_b cos); features past
    rot_dim are unchanged.  x: [B, P, H, D]; returns a new array.
    """
    x = np.asarray(x, dtype=np.float64)
    B, P, H, D = x.shape
    if rot_dim % 2 or not 2 <= rot_dim <= D:
        raise ValueError("rot_dim must be even and in [2, D]")
    out = x.copy()
    half = rot_dim // 2
    for b in range(B):
        start = pos_base + (pos_mult * int(pos0[b]) if pos0 is not None else 0)
        ang = rope_angles(start + np.arange(P), rot_dim, base)  # [P, half]
        c = np.cos(ang)[:, None, :]
        s = np.sin(ang)[:, None, :]
        if layout == "half":
            xa, xb = x[b, :, :, :half], x[b, :, :, half:rot_dim]
            out[b, :, :, :half] = xa * c - xb * s
            out[b, :, :, half:rot_dim] = xa * s + xb * c
        elif layout == "interleaved":
            xa, xb = x[b, :, :, 0:rot_dim:2], x[b, :, :, 1:rot_dim:2]
            out[b, :, :, 0:rot_dim:2] = xa * c - xb * s
            out[b, :, :, 1:rot_dim:2] = xa * s + xb * c
        else:
            raise ValueError(layout)
    return out


def _softmax_weighted(scores, vals):
    """Softmax over the last axis of ``scores`` (-inf = masked) applied to
    ``vals``; returns (out, lse)."""
    m = scores.max(axis=-1, keepdims=True)
    w = np.exp(scores - m)
    l = w.sum(axis=-1, keepdims=True)
    out = (w / l) @ vals
    lse = (m + np.log(l))[..., 0]
    return out, lse


def attn(q, k, v, n, mode, window=0, scale=None):
    """Stream-Factorized Attention forward, float64.

    q: [B, nL, Hq, D]; k, v: [B, nL, Hkv, D].  Returns (O [B, nL, Hq, D],
    lse [B, Hq, nL]).  For each (b, h, p): scores over visible keys
    scale * <q, k>, softmax, weighted sum of v.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv or P % n:
        raise ValueError("bad shapes")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    mask = visible_matrix(P // n, n, mode, window)
    O = np.empty((B, P, Hq, D))
    lse = np.empty((B, Hq, P))
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = scale * (q[b, :, h, :] @ k[b, :, kv, :].T)
            s = np.where(mask, s, -np.inf)
            O[b, :, h, :], lse[b, h, :] = _softmax_weighted(s, v[b, :, kv, :])
    return O, lse


def attn_bwd(q, k, v, dO, n, mode, window=0, scale=None):
    """Gradient of the Stream-Factorized Attention forward, float64.

    The pages train through these layers ("Computational Cost", "Near-Linear
    Training Cost") but print no backward; its plain definition is the
    derivative of  sum(dO * O)  with O = attn(q, k, v) for the Figure 2 mask.
    Per (b, h), with S = scale * q k^T over the visible set, P = softmax(S):
        dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
        dQ = scale * dS K,  dK = scale * dS^T Q,
    and dK, dV of a KV head summed over the query heads that read it.
    Returns (dQ [B, nL, Hq, D], dK [B, nL, Hkv, D], dV [B, nL, Hkv, D]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv or P % n or dO.shape != q.shape:
        raise ValueError("bad shapes")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    mask = visible_matrix(P // n, n, mode, window)
    dQ = np.zeros((B, P, Hq, D))
    dK = np.zeros((B, P, Hkv, D))
    dV = np.zeros((B, P, Hkv, D))
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = np.where(mask, scale * (q[b, :, h, :] @ k[b, :, kv, :].T), -np.inf)
            e = np.exp(s - s.max(axis=-1, keepdims=True))
            p = e / e.sum(axis=-1, keepdims=True)
            g = dO[b, :, h, :]
            dp = g @ v[b, :, kv, :].T
            ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
            dV[b, :, kv, :] += p.T @ g
            dQ[b, :, h, :] = scale * (ds @ k[b, :, kv, :])
            dK[b, :, kv, :] += scale * (ds.T @ q[b, :, h, :])
    return dQ, dK, dV


def _bwd_row(q, k, v, dO, n, mode, b, h, p, G, window, scale):
    """Row p of head h: (visible keys, P over them, dS over them)."""
    P = k.shape[1]
    kv = h // G
    keys = np.arange(P)[visible(p, np.arange(P), n, mode, window)]
    kk = np.asarray(k[b, keys, kv, :], dtype=np.float64)
    vv = np.asarray(v[b, keys, kv, :], dtype=np.float64)
    qv = np.asarray(q[b, p, h, :], dtype=np.float64)
    g = np.asarray(dO[b, p, h, :], dtype=np.float64)
    s = scale * (kk @ qv)
    e = np.exp(s - s.max())
    pr = e / e.sum()
    dp = vv @ g
    ds = pr * (dp - pr @ dp)
    return keys, kk, pr, ds


def attn_bwd_final_stream(q_final, k, v, dO_final, n, mode, window=0, scale=None):
    """Gradient of :func:`attn_final_stream` (the KV-mirror layers are trained
    through too): the derivative of sum(dO_final * O_final), O_final the
    final-stream queries' attention over every stream's keys.  Per (b, h),
    with S = scale q_final k^T over the keys visible to position i*n + n-1:
        dV = P^T dO,  dS = P * (dO V^T - rowsum(P * dO V^T)),
        dQ = scale dS K,  dK = scale dS^T Q  (dK, dV summed over a GQA group).
    Returns (dQ [B, L, Hq, D], dK [B, nL, Hkv, D], dV [B, nL, Hkv, D]); keys no
    final-stream query sees get zero."""
    q_final = np.asarray(q_final, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dO_final = np.asarray(dO_final, dtype=np.float64)
    B, L, Hq, D = q_final.shape
    P, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    mask = visible((np.arange(L) * n + n - 1)[:, None], np.arange(P)[None, :], n, mode, window)
    dQ = np.zeros((B, L, Hq, D))
    dK = np.zeros((B, P, Hkv, D))
    dV = np.zeros((B, P, Hkv, D))
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = np.where(mask, scale * (q_final[b, :, h, :] @ k[b, :, kv, :].T), -np.inf)
            e = np.exp(s - s.max(axis=-1, keepdims=True))
            pr = e / e.sum(axis=-1, keepdims=True)
            g = dO_final[b, :, h, :]
            dp = g @ v[b, :, kv, :].T
            ds = pr * (dp - (pr * dp).sum(axis=-1, keepdims=True))
            dV[b, :, kv, :] += pr.T @ g
            dQ[b, :, h, :] = scale * (ds @ k[b, :, kv, :])
            dK[b, :, kv, :] += scale * (ds.T @ q_final[b, :, h, :])
    return dQ, dK, dV


def attn_bwd_blocked(q, k, v, dO, n, mode, b, kvh, window=0, scale=None, block=1024):
    """:func:`attn_bwd` for one (b, KV head), its query heads' rows taken in
    blocks so the float64 score blocks fit in memory at full sizes: for each
    query head of the group and each block of query rows, form the rows' S,
    P, dP and dS over their visible keys (all keys before the block's end),
    write the rows' dQ and add their terms to dK and dV.  Inputs may be any
    array-likes indexable as q[b, p, h, :].  Returns (dQ [P, G, D] for the
    group's query heads, dK [P, D], dV [P, D])."""
    P, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    kk_all = np.asarray(k[b, :, kvh, :], dtype=np.float64)
    vv_all = np.asarray(v[b, :, kvh, :], dtype=np.float64)
    dQ = np.zeros((P, G, D))
    dK = np.zeros((P, D))
    dV = np.zeros((P, D))
    for g in range(G):
        h = kvh * G + g
        for p0 in range(0, P, block):
            p1 = min(P, p0 + block)
            mask = visible(np.arange(p0, p1)[:, None], np.arange(p1)[None, :], n, mode, window)
            qq = np.asarray(q[b, p0:p1, h, :], dtype=np.float64)
            gg = np.asarray(dO[b, p0:p1, h, :], dtype=np.float64)
            kk, vv = kk_all[:p1], vv_all[:p1]
            s = np.where(mask, scale * (qq @ kk.T), -np.inf)
            e = np.exp(s - s.max(axis=-1, keepdims=True))
            pr = e / e.sum(axis=-1, keepdims=True)
            dp = gg @ vv.T
            ds = pr * (dp - (pr * dp).sum(axis=-1, keepdims=True))
            dQ[p0:p1, g] = scale * (ds @ kk)
            dK[:p1] += scale * (ds.T @ qq)
            dV[:p1] += pr.T @ gg
    return dQ, dK, dV


def attn_bwd_dq_rows(q, k, v, dO, n, mode, rows, window=0, scale=None):
    """dQ of :func:`attn_bwd` for selected (b, h, p), one row at a time:
    dQ[p] = scale * sum over p's visible keys of dS[p, p'] k[p'].
    Inputs may be any array-likes indexable as q[b, p, h, :].  Returns [R, D]."""
    Hq, D = q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = []
    for (b, h, p) in rows:
        _, kk, _, ds = _bwd_row(q, k, v, dO, n, mode, b, h, p, G, window, scale)
        out.append(scale * (ds @ kk))
    return np.array(out)


def attn_bwd_dkv_rows(q, k, v, dO, n, mode, rows, window=0, scale=None):
    """dK and dV of :func:`attn_bwd` for selected (b, kv head g, key p'),
    summing over the query heads of the group and every query position p
    that sees p': each such row's softmax and dS are formed over the row's
    own visible keys.  Returns (dK [R, D], dV [R, D])."""
    P, Hq, D = q.shape[1], q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dks, dvs = [], []
    pos = np.arange(P)
    for (b, kvh, pk) in rows:
        queries = pos[visible(pos, pk, n, mode, window)]
        dk = np.zeros(D)
        dv = np.zeros(D)
        for h in range(kvh * G, (kvh + 1) * G):
            for p in queries:
                keys, _, pr, ds = _bwd_row(q, k, v, dO, n, mode, b, h, p, G, window, scale)
                c = int(np.searchsorted(keys, pk))
                dv += pr[c] * np.asarray(dO[b, p, h, :], dtype=np.float64)
                dk += scale * ds[c] * np.asarray(q[b, p, h, :], dtype=np.float64)
        dks.append(dk)
        dvs.append(dv)
    return np.array(dks), np.array(dvs)


def attn_bwd_query_rows(q, k, v, dO, n, mode, rows, window=0, scale=None):
    """The terms of :func:`attn_bwd` that query row (b, h, p) contributes:
    its dQ row, and over its visible keys p' the summands P[p,p'] dO[p] of dV
    and scale dS[p,p'] q[p] of dK.  Summing the latter over every query row
    (and the heads of a group) gives dK and dV.  Returns a list of
    (keys, dq [D], dk_terms [len(keys), D], dv_terms [len(keys), D])."""
    Hq, D = q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = []
    for (b, h, p) in rows:
        keys, kk, pr, ds = _bwd_row(q, k, v, dO, n, mode, b, h, p, G, window, scale)
        qv = np.asarray(q[b, p, h, :], dtype=np.float64)
        g = np.asarray(dO[b, p, h, :], dtype=np.float64)
        out.append((keys, scale * (ds @ kk), scale * np.outer(ds, qv), np.outer(pr, g)))
    return out


def attn_rows(q, k, v, n, mode, rows, window=0, scale=None):
    """The same definition evaluated for selected output rows only.

    rows: iterable of (b, h, p).  Returns (O [R, D], lse [R]).  Inputs may be
    any array-likes indexable as q[b, p, h, :] (e.g. large float32 arrays);
    each row's arithmetic is float64.
    """
    P = k.shape[1]
    Hq = q.shape[2]
    Hkv = k.shape[2]
    G = Hq // Hkv
    D = q.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    pk_all = np.arange(P)
    outs, lses = [], []
    for (b, h, p) in rows:
        kv = h // G
        keys = pk_all[visible(p, pk_all, n, mode, window)]
        qv = np.asarray(q[b, p, h, :], dtype=np.float64)
        kk = np.asarray(k[b, keys, kv, :], dtype=np.float64)
        vv = np.asarray(v[b, keys, kv, :], dtype=np.float64)
        o, l = _softmax_weighted(scale * (kk @ qv)[None, :], vv)
        outs.append(o[0])
        lses.append(l[0])
    return np.array(outs), np.array(lses)


def attn_rows_block(q, k, v, n, mode, b, h, p0, p1, window=0, scale=None):
    """Rows p0 <= p < p1 of :func:`attn` for one (b, h), in float64: the same
    per-row definition evaluated for a block of query rows at once (so the
    score block fits in memory at full sizes).  Keys past p1 - 1 are never
    visible to these rows and are not formed.  Inputs may be any array-likes
    indexable as q[b, p, h, :].  Returns (O [p1-p0, D], lse [p1-p0])."""
    Hq, D = q.shape[2], q.shape[3]
    G = Hq // k.shape[2]
    kv = h // G
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    pq = np.arange(p0, p1)
    pk = np.arange(p1)
    mask = visible(pq[:, None], pk[None, :], n, mode, window)
    qq = np.asarray(q[b, p0:p1, h, :], dtype=np.float64)
    kk = np.asarray(k[b, :p1, kv, :], dtype=np.float64)
    vv = np.asarray(v[b, :p1, kv, :], dtype=np.float64)
    s = np.where(mask, scale * (qq @ kk.T), -np.inf)
    return _softmax_weighted(s, vv)


def attn_final_stream(q_final, k, v, n, mode, window=0, scale=None):
    """Attention of the final-stream queries only ("Persistent KV and the
    KV-mirror Saving": in a mirrored layer only the final stream is run,
    against the keys and values every stream contributed earlier).

    q_final: [B, L, Hq, D] -- the query of token i sits at physical position
    p = i*n + n-1; k, v: [B, nL, Hkv, D].  Returns (O [B, L, Hq, D],
    lse [B, Hq, L]) by the same definition as :func:`attn`, one row at a time.
    """
    q_final = np.asarray(q_final, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, L, Hq, D = q_final.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    pk = np.arange(n * L)
    O = np.empty((B, L, Hq, D))
    lse = np.empty((B, Hq, L))
    for i in range(L):
        p = i * n + n - 1
        keys = pk[visible(p, pk, n, mode, window)]
        for b in range(B):
            for h in range(Hq):
                kv = h // G
                o, l = _softmax_weighted(scale * (k[b, keys, kv, :] @ q_final[b, i, h, :])[None, :], v[b, keys, kv, :])
                O[b, i, h], lse[b, h, i] = o[0], l[0]
    return O, lse


def _decode_keys(T, n, s, mode, window):
    """Visible cache entries (j, s') for the stream-s query of the new token
    T-1, as physical positions of the expanded sequence."""
    p = (T - 1) * n + s
    pk = np.arange(T * n)
    return pk[visible(p, pk, n, mode, window)]


def decode_rows(q, k_cache, v_cache, ctx_len, n, mode, rows, window=0, scale=None):
    """Decode for selected (b, s, h): the stream-s query of the newest token
    of sequence b against the per-stream cache.

    q: [B, n, Hq, D]; k_cache, v_cache: [B, n, Lmax, Hkv, D] (stream-major);
    ctx_len: [B] tokens per stream, new token included.  Returns (O [R, D],
    lse [R]).
    """
    Hq, D = q.shape[2], q.shape[3]
    Hkv = k_cache.shape[3]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    outs, lses = [], []
    for (b, s, h) in rows:
        T = int(ctx_len[b])
        kv = h // G
        pk = _decode_keys(T, n, s, mode, window)
        j, sk = pk // n, pk % n
        kk = np.asarray(k_cache[b, sk, j, kv, :], dtype=np.float64)
        vv = np.asarray(v_cache[b, sk, j, kv, :], dtype=np.float64)
        qv = np.asarray(q[b, s, h, :], dtype=np.float64)
        o, l = _softmax_weighted(scale * (kk @ qv)[None, :], vv)
        outs.append(o[0])
        lses.append(l[0])
    return np.array(outs), np.array(lses)


def shard_streams(n, R, r):
    """Streams held by rank r of R under stream parallelism ("Persistent KV
    and the KV-mirror Saving": the intra-stream KV is sharded across ranks by
    stream): s = r, r + R, r + 2R, ...  (R must divide n)."""
    if n % R:
        raise ValueError("R must divide n")
    return list(range(r, n, R))


def stream_interleave(parts, n):
    """Re-interleave per-rank stream shards into the expanded order.

    parts: [R, B, (n/R)*L, ...] where rank r's local row i*(n/R) + l holds
    token i of global stream s = r + R*l.  Returns [B, n*L, ...] with row
    i*n + s.  A pure permutation."""
    parts = np.asarray(parts)
    R, B, PL = parts.shape[:3]
    nl = n // R
    L = PL // nl
    out = np.empty((B, n * L) + parts.shape[3:], dtype=parts.dtype)
    for r in range(R):
        for l in range(nl):
            s = r + R * l
            for i in range(L):
                out[:, i * n + s] = parts[r, :, i * nl + l]
    return out


def decode_rows_streams(q, k_cache, v_cache, ctx_len, n, streams, rows, window=0, scale=None):
    """Cross-mode decode restricted to the cache streams in ``streams``.

    q: [B, n, Hq, D] (all streams' queries of the new token); k_cache,
    v_cache: [B, len(streams), Lmax, Hkv, D] holding global streams
    ``streams`` in order.  For each (b, s, h): softmax over the keys of
    :func:`decode_rows` (cross) that lie in those streams.  Returns
    (O [R, D], lse [R]); a row with no such key gets O = 0 and lse = -inf.
    """
    Hq, D = q.shape[2], q.shape[3]
    Hkv = k_cache.shape[3]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    local = {s: l for l, s in enumerate(streams)}
    outs, lses = [], []
    for (b, s, h) in rows:
        T = int(ctx_len[b])
        kv = h // G
        pk = _decode_keys(T, n, s, CROSS, window)
        pk = pk[np.isin(pk % n, list(streams))]
        if pk.size == 0:
            outs.append(np.zeros(D))
            lses.append(-np.inf)
            continue
        j, sl = pk // n, np.array([local[x] for x in pk % n])
        kk = np.asarray(k_cache[b, sl, j, kv, :], dtype=np.float64)
        vv = np.asarray(v_cache[b, sl, j, kv, :], dtype=np.float64)
        qv = np.asarray(q[b, s, h, :], dtype=np.float64)
        o, l = _softmax_weighted(scale * (kk @ qv)[None, :], vv)
        outs.append(o[0])
        lses.append(l[0])
    return np.array(outs), np.array(lses)


def combine_partials(o_parts, lse_parts):
    """Merge softmax-weighted partial results over disjoint key sets:
    O = sum_r exp(lse_r - LSE) O_r with LSE = log sum_r exp(lse_r).
    o_parts [R, ..., D], lse_parts [R, ...] (-inf: empty part).
    Returns (O, LSE); O = 0, LSE = -inf where every part is empty."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    safe = np.where(np.isfinite(m), m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - safe), 0.0)
    tot = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / np.where(tot > 0, tot, 1.0)[..., None]
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return o, lse


def decode(q, k_cache, v_cache, ctx_len, n, mode, window=0, scale=None):
    """All rows of :func:`decode_rows`: returns (O [B, n, Hq, D], lse [B, n, Hq])."""
    B, _, Hq, D = q.shape
    rows = [(b, s, h) for b in range(B) for s in range(n) for h in range(Hq)]
    O, lse = decode_rows(q, k_cache, v_cache, ctx_len, n, mode, rows, window, scale)
    return O.reshape(B, n, Hq, D), lse.reshape(B, n, Hq)
