"""Pins for the float64 oracle: library routines, closed forms, invariants,
the Figure 2 masks written out by hand, and a pure-Python brute force.

Each pin is chosen so that a plausible slip in the oracle (a wrong stream or
token index, a dropped self pair, a transposed operand, a wrong GQA grouping,
a wrong window edge, a wrong cache index) fails at least one of them; the
``planted`` tests at the end plant such slips in a copy of the oracle and
check that the pins notice.
"""

import itertools
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import brute
from oracle import hd_oracle
from stream_sequence_attention_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qkv(B, P, Hq, Hkv, D, seed):
    q = synth.normal((B, P, Hq, D), seed)
    k = synth.normal((B, P, Hkv, D), seed + 1)
    v = synth.normal((B, P, Hkv, D), seed + 2)
    return q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)


def _sdpa(q, k, v, scale, causal=False, mask=None):
    """torch SDPA in float64 on CPU.  q [B,P,Hq,D], k/v [B,P',Hkv,D]; GQA by
    repeating each KV head for its G consecutive query heads."""
    G = q.shape[2] // k.shape[2]
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    am = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- index maps

def test_index_maps_match_one_based_definition():
    # "Stream-Factorized Attention": i(t) = ceil(t/n), s(t) = (t-1) mod n + 1
    for n in range(1, 6):
        for t in range(1, 40):
            p = t - 1
            assert oracle.token_index(p, n) + 1 == -(-t // n)
            assert oracle.stream_index(p, n) + 1 == (t - 1) % n + 1


def _read_golden_masks():
    masks, cur = {}, None
    with open(os.path.join(GOLDEN, "fig2_masks_n2_L3.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                mode, w = line[1:-1].split()
                cur = (mode, int(w.split("=")[1]))
                masks[cur] = []
            else:
                masks[cur].append([c == "1" for c in line])
    return {k: np.array(v) for k, v in masks.items()}


def test_figure2_masks_by_hand():
    golden = _read_golden_masks()
    assert len(golden) == 4
    for (mode, w), m in golden.items():
        got = oracle.visible_matrix(3, 2, mode, w)
        np.testing.assert_array_equal(got, m, err_msg=f"{mode} W={w}")


# ------------------------------------------------------- expand and gather

@pytest.mark.parametrize("n,B,L,V,d", [(2, 1, 64, 512, 128), (4, 2, 7, 33, 8), (1, 3, 5, 9, 4), (3, 1, 1, 2, 16)])
def test_expand_equals_index_select(n, B, L, V, d):
    tables = synth.normal((n, V, d), 11, std=0.02)
    ids = synth.ids_uniform(B, L, V, 12)
    out = oracle.expand(tables, ids)
    t = torch.from_numpy(tables)
    ref = torch.stack([t[s].index_select(0, torch.from_numpy(ids.reshape(-1)).long()) for s in range(n)], dim=1)
    ref = ref.reshape(B, L * n, d).numpy()  # [B*L, n, d] -> token-major interleave
    assert out.shape == (B, n * L, d)
    np.testing.assert_array_equal(out.view(np.uint32), ref.view(np.uint32))


def test_expand_rejects_bad_ids():
    tables = np.zeros((2, 4, 8), dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.expand(tables, np.array([[0, 4]], dtype=np.int32))
    with pytest.raises(ValueError):
        oracle.expand(tables, np.array([[-1]], dtype=np.int32))


@pytest.mark.parametrize("n,B,L,d", [(2, 1, 64, 128), (4, 2, 9, 8), (1, 1, 3, 4)])
def test_gather_equals_strided_slice(n, B, L, d):
    h = synth.normal((B, n * L, d), 21)
    out = oracle.final_stream_gather(h, n)
    ref = torch.from_numpy(h)[:, n - 1::n, :].numpy()
    np.testing.assert_array_equal(out.view(np.uint32), ref.view(np.uint32))


# ------------------------------------------ attention against library SDPA

@pytest.mark.parametrize("mode", ["intra", "cross"])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (6, 3)])
def test_n1_is_standard_causal_attention(mode, Hq, Hkv):
    q, k, v = _qkv(2, 23, Hq, Hkv, 8, 100)
    O, _ = oracle.attn(q, k, v, 1, mode, 0, 0.3)
    ref = _sdpa(q, k, v, 0.3, causal=True)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [2, 3, 4])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1), (4, 2)])
def test_intra_equals_independent_causal_streams(n, Hq, Hkv):
    B, L, D = 2, 11, 8
    q, k, v = _qkv(B, n * L, Hq, Hkv, D, 200 + n)
    O, _ = oracle.attn(q, k, v, n, "intra", 0, 0.25)
    for s in range(n):
        # de-interleave: [B, L, n, H, D][:, :, s]
        qs = q.reshape(B, L, n, Hq, D)[:, :, s]
        ks = k.reshape(B, L, n, Hkv, D)[:, :, s]
        vs = v.reshape(B, L, n, Hkv, D)[:, :, s]
        ref = _sdpa(np.ascontiguousarray(qs), np.ascontiguousarray(ks), np.ascontiguousarray(vs), 0.25, causal=True)
        got = O.reshape(B, L, n, Hq, D)[:, :, s]
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [2, 4])
def test_cross_equals_dense_causal_over_nL(n):
    B, L, D = 2, 9, 8
    q, k, v = _qkv(B, n * L, 4, 2, D, 300 + n)
    O, _ = oracle.attn(q, k, v, n, "cross", 0, 0.5)
    ref = _sdpa(q, k, v, 0.5, causal=True)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,W", [(2, 1), (2, 3), (3, 4), (4, 100)])
def test_intra_window_equals_banded_streams(n, W):
    B, L, D = 1, 10, 8
    q, k, v = _qkv(B, n * L, 2, 1, D, 400 + W)
    O, _ = oracle.attn(q, k, v, n, "intra", W, 0.4)
    j = np.arange(L)
    band = (j[None, :] <= j[:, None]) & (j[:, None] - j[None, :] < W)
    for s in range(n):
        qs = np.ascontiguousarray(q.reshape(B, L, n, 2, D)[:, :, s])
        ks = np.ascontiguousarray(k.reshape(B, L, n, 1, D)[:, :, s])
        vs = np.ascontiguousarray(v.reshape(B, L, n, 1, D)[:, :, s])
        ref = _sdpa(qs, ks, vs, 0.4, mask=band)
        np.testing.assert_allclose(O.reshape(B, L, n, 2, D)[:, :, s], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n,W", [(2, 1), (2, 5), (4, 7), (3, 1000)])
def test_cross_window_equals_banded_causal(n, W):
    B, L, D = 1, 8, 8
    P = n * L
    q, k, v = _qkv(B, P, 2, 2, D, 500 + W)
    O, _ = oracle.attn(q, k, v, n, "cross", W, 0.4)
    p = np.arange(P)
    band = (p[None, :] <= p[:, None]) & (p[:, None] - p[None, :] < W)
    ref = _sdpa(q, k, v, 0.4, mask=band)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------- invariants

@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 3), ("cross", 5)])
def test_masked_keys_get_exactly_zero_weight(mode, W):
    n, L, D = 3, 8, 8
    P = n * L
    q, k, v = _qkv(1, P, 2, 1, D, 600)
    O, lse = oracle.attn(q, k, v, n, mode, W, 0.3)
    g = synth.rng(601)
    pk = np.arange(P)
    for p in [0, 1, 5, 13, P - 1]:
        hidden = ~oracle.visible(p, pk, n, mode, W)
        k2, v2 = k.copy(), v.copy()
        k2[:, hidden] += g.standard_normal(k2[:, hidden].shape) * 10
        v2[:, hidden] += g.standard_normal(v2[:, hidden].shape) * 10
        O2, lse2 = oracle.attn(q, k2, v2, n, mode, W, 0.3)
        assert np.array_equal(O2[:, p], O[:, p])
        assert np.array_equal(lse2[:, :, p], lse[:, :, p])


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 2), ("cross", 3)])
def test_softmax_rows_sum_to_one_and_constant_values(mode, W):
    n, L, D = 4, 6, 8
    P = n * L
    q, k, _ = _qkv(2, P, 4, 2, D, 700)
    ones = np.ones((2, P, 2, D))
    O, _ = oracle.attn(q, k, ones, n, mode, W, 0.7)
    assert np.max(np.abs(O - 1.0)) < 1e-12
    c = np.full((2, P, 2, D), -2.375)
    O, _ = oracle.attn(q, k, c, n, mode, W, 0.7)
    assert np.max(np.abs(O + 2.375)) < 1e-12


def _closed_form_keys(p, n, mode, W):
    """Visible key positions as explicit ranges (not via the oracle's mask)."""
    if mode == "intra":
        i, s = divmod(p, n)
        lo = 0 if W == 0 else max(0, i - W + 1)
        return [j * n + s for j in range(lo, i + 1)]
    lo = 0 if W == 0 else max(0, p - W + 1)
    return list(range(lo, p + 1))


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 3), ("cross", 6)])
def test_zero_query_gives_mean_of_visible_values(mode, W):
    # q = 0 makes every visible score equal, so the softmax is uniform.
    n, L, D = 3, 7, 4
    P = n * L
    _, k, v = _qkv(1, P, 2, 2, D, 800)
    q = np.zeros((1, P, 2, D))
    O, lse = oracle.attn(q, k, v, n, mode, W, 1.0)
    for p in range(P):
        keys = _closed_form_keys(p, n, mode, W)
        for h in range(2):
            np.testing.assert_allclose(O[0, p, h], v[0, keys, h].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[0, h, p] - np.log(len(keys))) < 1e-13


# ----------------------------------------------------------- brute force

def _brute_cases():
    cases = []
    for n in (1, 2, 3, 4):
        for mode in ("intra", "cross"):
            for W in (0, 1, 2, 5):
                cases.append((n, mode, W))
    return cases


@pytest.mark.parametrize("n,mode,W", _brute_cases())
def test_oracle_matches_brute_force(n, mode, W):
    L = {1: 9, 2: 5, 3: 4, 4: 3}[n]
    Hq, Hkv, D = 4, 2, 5
    q, k, v = _qkv(2, n * L, Hq, Hkv, D, 900 + 10 * n + W)
    O, lse = oracle.attn(q, k, v, n, mode, W, 0.45)
    bo, bl = brute.attn(q.tolist(), k.tolist(), v.tolist(), n, mode, W, 0.45)
    np.testing.assert_allclose(O, np.array(bo), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 2), ("cross", 3)])
def test_attn_rows_match_full_attention(mode, W):
    n, L = 4, 6
    q, k, v = _qkv(2, n * L, 4, 2, 8, 1000)
    O, lse = oracle.attn(q, k, v, n, mode, W, None)
    rows = [(b, h, p) for b in range(2) for h in range(4) for p in range(0, n * L, 5)]
    Or, lr = oracle.attn_rows(q, k, v, n, mode, rows, W, None)
    for r, (b, h, p) in enumerate(rows):
        np.testing.assert_allclose(Or[r], O[b, p, h], rtol=0, atol=1e-13)
        assert abs(lr[r] - lse[b, h, p]) < 1e-13


# ----------------------------------------------------------------- decode

def _to_cache(x, n, Lmax):
    """[B, nL, H, D] interleaved -> stream-major cache [B, n, Lmax, H, D]."""
    B, P, H, D = x.shape
    L = P // n
    c = synth.normal((B, n, Lmax, H, D), 1234)  # garbage beyond L must be ignored
    c = c.astype(np.float64) * 50
    c[:, :, :L] = x.reshape(B, L, n, H, D).transpose(0, 2, 1, 3, 4)
    return c


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 3), ("cross", 5)])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_decode_equals_prefill_of_last_token(mode, W, n):
    B, L, Hq, Hkv, D = 3, 7, 4, 2, 8
    Lmax = L + 3
    q, k, v = _qkv(B, n * L, Hq, Hkv, D, 1100 + n)
    kc, vc = _to_cache(k, n, Lmax), _to_cache(v, n, Lmax)
    ctx = np.array([L, 1, 4], dtype=np.int32)
    for b in range(B):
        T = int(ctx[b])
        O, lse = oracle.attn(q[b:b + 1, : n * T], k[b:b + 1, : n * T], v[b:b + 1, : n * T], n, mode, W, 0.3)
        qd = np.stack([q[b, (T - 1) * n + s] for s in range(n)])[None]  # [1, n, Hq, D]
        Od, lsed = oracle.decode(qd, kc[b:b + 1], vc[b:b + 1], ctx[b:b + 1], n, mode, W, 0.3)
        for s in range(n):
            p = (T - 1) * n + s
            np.testing.assert_allclose(Od[0, s], O[0, p], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lsed[0, s], lse[0, :, p], rtol=0, atol=1e-13)


def test_decode_against_brute_force():
    n, T, Hq, Hkv, D = 3, 4, 2, 1, 4
    q, k, v = _qkv(1, n * T, Hq, Hkv, D, 1200)
    kc, vc = _to_cache(k, n, T + 2), _to_cache(v, n, T + 2)
    qd = np.stack([q[0, (T - 1) * n + s] for s in range(n)])[None]
    for mode in ("intra", "cross"):
        Od, _ = oracle.decode(qd, kc, vc, np.array([T]), n, mode, 0, 0.5)
        bo, _ = brute.attn(q.tolist(), k.tolist(), v.tolist(), n, mode, 0, 0.5)
        for s in range(n):
            np.testing.assert_allclose(Od[0, s], np.array(bo[0][(T - 1) * n + s]), rtol=0, atol=1e-12)


# ------------------------------------------------------------ pair counts

@pytest.mark.parametrize("n,L", [(1, 9), (2, 8), (4, 6), (3, 5)])
def test_pair_counts_closed_forms(n, L):
    # Intra O(nL^2) vs dense O(n^2 L^2): "Stream-Factorized Attention" and
    # "Near-Linear Training Cost".
    P = n * L
    assert oracle.pair_count(L, n, "intra") == n * L * (L + 1) // 2
    assert oracle.pair_count(L, n, "cross") == P * (P + 1) // 2
    for W in (1, 2, L - 1, L, L + 3):
        if W <= 0:
            continue
        Wt = min(W, L)
        assert oracle.pair_count(L, n, "intra", W) == n * (Wt * (Wt + 1) // 2 + (L - Wt) * Wt)
        Wp = min(W, P)
        assert oracle.pair_count(L, n, "cross", W) == Wp * (Wp + 1) // 2 + (P - Wp) * Wp


def test_cross_over_intra_ratio_tends_to_n():
    # The pages' claim: dense attention over nL costs ~n times intra.
    L, n = 4096, 4
    intra = n * L * (L + 1) // 2
    cross = (n * L) * (n * L + 1) // 2
    assert abs(cross / intra - 3.99927) < 1e-5


# ------------------------------------------- planted mistakes are caught

def _planted_visible(kind):
    orig = hd_oracle.visible

    def bad(p, pk, n, mode, window=0):
        p = np.asarray(p)
        pk = np.asarray(pk)
        if kind == "no_self":
            return orig(p, pk, n, mode, window) & (pk != p)
        if kind == "stream_swap":  # s = p // n, i = p % n
            if hd_oracle._mode(mode) == "intra":
                i, s, j, sk = p % n, p // n, pk % n, pk // n
                return (sk == s) & (j <= i)
            return orig(p, pk, n, mode, window)
        if kind == "window_off_by_one":
            if window:
                return orig(p, pk, n, mode, window + 1)
            return orig(p, pk, n, mode, window)
        raise ValueError(kind)

    return bad


@pytest.mark.parametrize("kind", ["no_self", "stream_swap", "window_off_by_one"])
def test_planted_mask_mistakes_are_caught(kind, monkeypatch):
    monkeypatch.setattr(hd_oracle, "visible", _planted_visible(kind))
    caught = False
    try:
        test_figure2_masks_by_hand()
    except AssertionError:
        caught = True
    assert caught, kind


def test_planted_gqa_and_transpose_mistakes_are_caught(monkeypatch):
    q, k, v = _qkv(1, 12, 4, 2, 8, 1300)
    ref = _sdpa(q, k, v, 0.3, causal=True)
    # wrong grouping: kv = h % Hkv instead of h // G
    O_bad = np.empty_like(ref)
    for h in range(4):
        O_bad[:, :, h] = oracle.attn(q[:, :, h:h + 1], k[:, :, h % 2:h % 2 + 1], v[:, :, h % 2:h % 2 + 1], 1, "cross", 0, 0.3)[0][:, :, 0]
    assert np.max(np.abs(O_bad - ref)) > 1e-3
    # swapped K and V
    O_swap, _ = oracle.attn(q, v, k, 1, "cross", 0, 0.3)
    assert np.max(np.abs(O_swap - ref)) > 1e-3


# ------------------------------------------- final-stream queries (KV mirror)

@pytest.mark.parametrize("n,mode,W", [(1, "cross", 0), (2, "intra", 0), (3, "cross", 0), (4, "intra", 3),
                                      (4, "cross", 7), (2, "cross", 1)])
def test_final_stream_rows_equal_full_attention_rows(n, mode, W):
    """Each output row depends only on its own query, so the final-stream
    call equals the full call's rows p = i*n + n-1 whatever the other queries
    are."""
    B, L, Hq, Hkv, D = 2, 6, 4, 2, 8
    P = n * L
    q, k, v = _qkv(B, P, Hq, Hkv, D, 1400 + n + W)
    qf = np.ascontiguousarray(q[:, n - 1::n])
    O, lse = oracle.attn(q, k, v, n, mode, W, 0.35)
    Of, lf = oracle.attn_final_stream(qf, k, v, n, mode, W, 0.35)
    np.testing.assert_allclose(Of, O[:, n - 1::n], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lf, lse[:, :, n - 1::n], rtol=0, atol=1e-13)


def test_final_stream_intra_is_causal_attention_on_last_stream():
    B, n, L, Hq, Hkv, D = 1, 3, 9, 2, 1, 8
    q, k, v = _qkv(B, n * L, Hq, Hkv, D, 1500)
    qf = np.ascontiguousarray(q[:, n - 1::n])
    Of, _ = oracle.attn_final_stream(qf, k, v, n, "intra", 0, 0.5)
    ks = np.ascontiguousarray(k[:, n - 1::n])
    vs = np.ascontiguousarray(v[:, n - 1::n])
    ref = _sdpa(qf, ks, vs, 0.5, causal=True)
    np.testing.assert_allclose(Of, ref, rtol=0, atol=1e-12)


def test_final_stream_cross_pair_count_equals_intra():
    # Final-stream queries over all streams: sum_i n*(i+1) = n L(L+1)/2 pairs,
    # the intra-layer count -- the saving of running only the final stream.
    for n, L in [(2, 5), (4, 7)]:
        pk = np.arange(n * L)
        pairs = sum(int(np.count_nonzero(oracle.visible(i * n + n - 1, pk, n, "cross"))) for i in range(L))
        assert pairs == n * L * (L + 1) // 2


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("intra", 3), ("cross", 5)])
def test_attn_rows_block_matches_full_attention(mode, W):
    n, L, Hq, Hkv, D = 3, 11, 4, 2, 8
    q, k, v = _qkv(2, n * L, Hq, Hkv, D, 77)
    O, lse = oracle.attn(q, k, v, n, mode, W)
    for b, h, p0, p1 in [(0, 0, 0, 33), (1, 3, 5, 17), (1, 2, 32, 33), (0, 1, 0, 1)]:
        o, l = oracle.attn_rows_block(q, k, v, n, mode, b, h, p0, p1, W)
        np.testing.assert_allclose(o, O[b, p0:p1, h], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(l, lse[b, h, p0:p1], rtol=1e-13, atol=1e-13)
