"""Pins for the oracle's attention backward (``oracle.attn_bwd``).

The backward is pinned to things other than its own formulas: central finite
differences of the (separately pinned) forward oracle, torch autograd through
float64 SDPA with the Figure 2 mask, and two identities that hold for any
softmax attention (rows of dS sum to zero, rows of P sum to one).  The
``planted`` test edits a copy of the oracle's source (a dropped term, a
missing scale, a transposed operand, a wrong GQA grouping) and checks that
the finite-difference pin notices each edit.
"""

import inspect

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import hd_oracle
from stream_sequence_attention_b200 import synth

CASES = [("intra", 0), ("cross", 0), ("intra", 2), ("cross", 3)]


def _inputs(B, L, n, Hq, Hkv, D, seed):
    P = n * L
    q = synth.normal((B, P, Hq, D), seed).astype(np.float64)
    k = synth.normal((B, P, Hkv, D), seed + 1).astype(np.float64)
    v = synth.normal((B, P, Hkv, D), seed + 2).astype(np.float64)
    dO = synth.normal((B, P, Hq, D), seed + 3).astype(np.float64)
    return q, k, v, dO


def _finite_difference(q, k, v, dO, n, mode, W, scale, h=1e-6):
    """Central differences of f = sum(dO * attn(q, k, v)) for every input
    element, through the forward oracle only."""
    def f(qq, kk, vv):
        return float(np.sum(dO * oracle.attn(qq, kk, vv, n, mode, W, scale)[0]))

    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        x = args[which]
        g = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            fp = f(*args)
            x[idx] = x0 - h
            fm = f(*args)
            x[idx] = x0
            g[idx] = (fp - fm) / (2 * h)
        grads.append(g)
    return grads


def _check_fd(bwd, mode, W, n=2, L=3, Hq=4, Hkv=2, D=3, seed=11, scale=0.7):
    q, k, v, dO = _inputs(1, L, n, Hq, Hkv, D, seed)
    fd = _finite_difference(q, k, v, dO, n, mode, W, scale)
    got = bwd(q, k, v, dO, n, mode, W, scale)
    for name, a, b in zip("QKV", got, fd):
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-7, err_msg=f"d{name} {mode} W={W}")


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_matches_finite_differences_of_forward(mode, W):
    _check_fd(oracle.attn_bwd, mode, W)


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_matches_torch_autograd_sdpa(mode, W):
    n, L, Hq, Hkv, D, scale = 3, 5, 4, 2, 8, 0.3
    q, k, v, dO = _inputs(2, L, n, Hq, Hkv, D, 21)
    mask = torch.from_numpy(oracle.visible_matrix(L, n, mode, W))
    G = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).requires_grad_()
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).requires_grad_()
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_()
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1),
                                       attn_mask=mask, scale=scale)
    o.backward(torch.from_numpy(dO).permute(0, 2, 1, 3))
    dQ, dK, dV = oracle.attn_bwd(q, k, v, dO, n, mode, W, scale)
    for name, a, t in (("Q", dQ, tq), ("K", dK, tk), ("V", dV, tv)):
        np.testing.assert_allclose(a, t.grad.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=f"d{name} {mode} W={W}")


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_softmax_identities(mode, W):
    # Every row of dS sums to zero, so the keys' gradients sum to zero per KV
    # head; every row of P sums to one, so the values' gradients sum to the
    # output gradients of the query heads that read them.
    n, L, Hq, Hkv, D = 2, 6, 6, 3, 5
    q, k, v, dO = _inputs(2, L, n, Hq, Hkv, D, 31)
    _, dK, dV = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    G = Hq // Hkv
    np.testing.assert_allclose(dK.sum(axis=1), 0.0, atol=1e-12)
    want = dO.reshape(2, n * L, Hkv, G, D).sum(axis=(1, 3))
    np.testing.assert_allclose(dV.sum(axis=1), want, rtol=1e-12, atol=1e-12)


def test_bwd_intra_streams_are_independent():
    # Intra-stream attention never mixes streams: the output gradient of one
    # stream moves only that stream's dQ/dK/dV.
    n, L = 3, 4
    q, k, v, dO = _inputs(1, L, n, 2, 1, 4, 41)
    base = oracle.attn_bwd(q, k, v, dO, n, "intra")
    dO2 = dO.copy()
    dO2[:, 1::n] += 1.0  # stream 1 only
    moved = oracle.attn_bwd(q, k, v, dO2, n, "intra")
    others = np.arange(n * L) % n != 1
    for a, b in zip(base, moved):
        np.testing.assert_array_equal(a[:, others], b[:, others])
        assert not np.allclose(a[:, ~others], b[:, ~others])


_PLANTS = {
    "dropped_delta": ("ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))", "ds = p * dp"),
    "missing_scale_dk": ("dK[b, :, kv, :] += scale * (ds.T @ q[b, :, h, :])", "dK[b, :, kv, :] += ds.T @ q[b, :, h, :]"),
    "transposed_dq": ("dQ[b, :, h, :] = scale * (ds @ k[b, :, kv, :])", "dQ[b, :, h, :] = scale * (ds.T @ k[b, :, kv, :])"),
    "wrong_gqa": ("kv = h // G", "kv = h % Hkv"),
    "dv_without_p": ("dV[b, :, kv, :] += p.T @ g", "dV[b, :, kv, :] += ds.T @ g"),
}


@pytest.mark.parametrize("kind", sorted(_PLANTS))
def test_planted_bwd_mistakes_are_caught(kind):
    src = inspect.getsource(hd_oracle.attn_bwd)
    a, b = _PLANTS[kind]
    assert a in src
    ns = dict(vars(hd_oracle))
    exec(src.replace(a, b), ns)
    with pytest.raises(AssertionError):
        for mode, W in CASES:
            _check_fd(ns["attn_bwd"], mode, W)


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_row_functions_match_full_backward(mode, W):
    n, L, Hq, Hkv, D = 3, 7, 4, 2, 6
    q, k, v, dO = _inputs(2, L, n, Hq, Hkv, D, 51)
    dQ, dK, dV = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    P = n * L
    qrows = [(b, h, p) for b in range(2) for h in range(Hq) for p in (0, 1, P // 2, P - 1)]
    got = oracle.attn_bwd_dq_rows(q, k, v, dO, n, mode, qrows, W)
    np.testing.assert_allclose(got, np.array([dQ[b, p, h] for b, h, p in qrows]), rtol=1e-12, atol=1e-12)
    krows = [(b, g, p) for b in range(2) for g in range(Hkv) for p in (0, 2, P // 2, P - 2, P - 1)]
    gk, gv = oracle.attn_bwd_dkv_rows(q, k, v, dO, n, mode, krows, W)
    np.testing.assert_allclose(gk, np.array([dK[b, p, g] for b, g, p in krows]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gv, np.array([dV[b, p, g] for b, g, p in krows]), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_query_row_terms_sum_to_full_backward(mode, W):
    n, L, Hq, Hkv, D = 2, 6, 4, 2, 5
    q, k, v, dO = _inputs(1, L, n, Hq, Hkv, D, 61)
    dQ, dK, dV = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    P, G = n * L, Hq // Hkv
    rows = [(0, h, p) for h in range(Hq) for p in range(P)]
    sk = np.zeros_like(dK)
    sv = np.zeros_like(dV)
    for (b, h, p), (keys, dq, tk, tv) in zip(rows, oracle.attn_bwd_query_rows(q, k, v, dO, n, mode, rows, W)):
        np.testing.assert_allclose(dq, dQ[b, p, h], rtol=1e-12, atol=1e-12)
        sk[b, keys, h // G] += tk
        sv[b, keys, h // G] += tv
    np.testing.assert_allclose(sk, dK, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sv, dV, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode,W", CASES)
def test_bwd_blocked_matches_full_backward(mode, W):
    n, L, Hq, Hkv, D = 3, 9, 4, 2, 6
    q, k, v, dO = _inputs(2, L, n, Hq, Hkv, D, 71)
    dQ, dK, dV = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    G = Hq // Hkv
    for b in range(2):
        for kvh in range(Hkv):
            for block in (1, 5, 64):
                bq, bk, bv = oracle.attn_bwd_blocked(q, k, v, dO, n, mode, b, kvh, W, block=block)
                np.testing.assert_allclose(bq, dQ[b, :, kvh * G:(kvh + 1) * G], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(bk, dK[b, :, kvh], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(bv, dV[b, :, kvh], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode,W", CASES)
def test_final_stream_bwd_is_the_full_bwd_with_only_final_rows(mode, W):
    # The final-stream queries are the rows i*n + n-1 of the full layer: with
    # those rows of q and dO and zero output gradient elsewhere, the full
    # backward gives the same dK, dV and the same dQ on those rows.
    n, L, Hq, Hkv, D = 3, 5, 4, 2, 6
    q, k, v, dO = _inputs(2, L, n, Hq, Hkv, D, 81)
    qf, gf = q[:, n - 1::n], dO[:, n - 1::n]
    dO0 = np.zeros_like(dO)
    dO0[:, n - 1::n] = gf
    fq, fk, fv = oracle.attn_bwd(q, k, v, dO0, n, mode, W)
    gq, gk, gv = oracle.attn_bwd_final_stream(qf, k, v, gf, n, mode, W)
    np.testing.assert_allclose(gq, fq[:, n - 1::n], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gk, fk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gv, fv, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode,W", CASES)
def test_final_stream_bwd_matches_finite_differences(mode, W):
    n, L, Hq, Hkv, D, h = 2, 3, 2, 1, 3, 1e-6
    q, k, v, dO = _inputs(1, L, n, Hq, Hkv, D, 91)
    qf, gf = q[:, n - 1::n].copy(), dO[:, n - 1::n]

    def f(a, b_, c):
        return float(np.sum(gf * oracle.attn_final_stream(a, b_, c, n, mode, W, 0.7)[0]))

    got = oracle.attn_bwd_final_stream(qf, k, v, gf, n, mode, W, 0.7)
    for which, x in enumerate((qf, k, v)):
        args = [qf.copy(), k.copy(), v.copy()]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            args[which][i] = x[i] + h
            fp = f(*args)
            args[which][i] = x[i] - h
            fm = f(*args)
            args[which][i] = x[i]
            fd[i] = (fp - fm) / (2 * h)
        np.testing.assert_allclose(got[which], fd, rtol=1e-6, atol=1e-7)
