"""Pins for the oracle's stream-parallel pieces: the stream partition, the
re-interleave of per-rank shards, decode restricted to a rank's cache streams,
and the merge of partial softmax results.

Pinned to: a numpy reshape/transpose split (the interleave must invert it
exactly), the full decode oracle (restricting to every stream is the full
decode; merging the partials of a partition of streams is the full decode,
including ranks that see no key), and hand-written merges."""

import inspect
import math

import numpy as np
import pytest

import oracle
from oracle import hd_oracle
from stream_sequence_attention_b200 import synth


@pytest.mark.parametrize("n,R", [(4, 1), (4, 2), (4, 4), (6, 3), (8, 2)])
def test_shard_streams_partition(n, R):
    parts = [oracle.shard_streams(n, R, r) for r in range(R)]
    assert sorted(s for p in parts for s in p) == list(range(n))
    for r, p in enumerate(parts):
        assert all(s % R == r for s in p) and len(p) == n // R
    with pytest.raises(ValueError):
        oracle.shard_streams(5, 2, 0)


def _split(x, n, R):
    """[B, n*L, ...] -> [R, B, (n/R)*L, ...] by reshape: stream s = l*R + r."""
    B, P = x.shape[:2]
    L, nl = P // n, n // R
    x5 = x.reshape((B, L, nl, R) + x.shape[2:])
    return np.stack([x5[:, :, :, r].reshape((B, L * nl) + x.shape[2:]) for r in range(R)])


@pytest.mark.parametrize("n,R", [(4, 2), (4, 4), (6, 3), (2, 1)])
def test_interleave_inverts_the_split(n, R):
    x = synth.normal((2, n * 5, 3, 4), 17)
    parts = _split(x, n, R)
    for r in range(R):  # the split puts global stream r + R*l at local stream l
        for l in range(n // R):
            np.testing.assert_array_equal(parts[r][:, l::n // R], x[:, r + R * l::n])
    np.testing.assert_array_equal(oracle.stream_interleave(parts, n), x)


def _cache(B, n, T, Hkv, D, seed):
    k = synth.normal((B, n, T, Hkv, D), seed).astype(np.float64)
    v = synth.normal((B, n, T, Hkv, D), seed + 1).astype(np.float64)
    return k, v


@pytest.mark.parametrize("W", [0, 5])
def test_all_streams_is_the_full_decode(W):
    B, n, T, Hq, Hkv, D = 2, 4, 6, 4, 2, 8
    q = synth.normal((B, n, Hq, D), 21).astype(np.float64)
    k, v = _cache(B, n, T, Hkv, D, 22)
    ctx = np.array([T, 3])
    rows = [(b, s, h) for b in range(B) for s in range(n) for h in range(Hq)]
    o, l = oracle.decode_rows(q, k, v, ctx, n, "cross", rows, W)
    o2, l2 = oracle.decode_rows_streams(q, k, v, ctx, n, list(range(n)), rows, W)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l2, l, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("R,W,T", [(2, 0, 6), (4, 0, 6), (4, 0, 1), (2, 3, 5), (4, 6, 2)])
def test_merged_shard_partials_are_the_full_decode(R, W, T):
    B, n, Hq, Hkv, D = 2, 4, 4, 2, 8
    q = synth.normal((B, n, Hq, D), 31).astype(np.float64)
    k, v = _cache(B, n, T, Hkv, D, 32)
    ctx = np.array([T, max(1, T - 1)])
    rows = [(b, s, h) for b in range(B) for s in range(n) for h in range(Hq)]
    full_o, full_l = oracle.decode_rows(q, k, v, ctx, n, "cross", rows, W)
    po, pl = [], []
    for r in range(R):
        st = oracle.shard_streams(n, R, r)
        o, l = oracle.decode_rows_streams(q, k[:, st], v[:, st], ctx, n, st, rows, W)
        po.append(o)
        pl.append(l)
    if T == 1:  # stream s of a one-token context sees only streams s' <= s: some ranks see nothing
        assert np.isneginf(np.array(pl)).any()
    o, l = oracle.combine_partials(np.array(po), np.array(pl))
    np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l, full_l, rtol=1e-12, atol=1e-12)


def test_combine_by_hand():
    # two parts: lse log 1 and log 3 -> weights 1/4, 3/4; LSE = log 4
    o, l = oracle.combine_partials(np.array([[[2.0, 0.0]], [[0.0, 4.0]]]), np.array([[0.0], [math.log(3.0)]]))
    np.testing.assert_allclose(o, [[0.5, 3.0]], rtol=1e-15)
    np.testing.assert_allclose(l, [math.log(4.0)], rtol=1e-15)
    # an empty part changes nothing; all empty gives zeros and -inf
    o, l = oracle.combine_partials(np.array([[[2.0, 1.0]], [[9.0, 9.0]]]), np.array([[0.5], [-np.inf]]))
    np.testing.assert_allclose(o, [[2.0, 1.0]])
    np.testing.assert_allclose(l, [0.5])
    o, l = oracle.combine_partials(np.zeros((2, 1, 2)), np.full((2, 1), -np.inf))
    assert not o.any() and np.isneginf(l).all()


def test_planted_combine_mistake_is_caught(monkeypatch):
    src = inspect.getsource(hd_oracle.combine_partials)
    a = "w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - safe), 0.0)"
    assert a in src
    ns = dict(vars(hd_oracle))
    exec(src.replace(a, "w = np.where(np.isfinite(lse_parts), 1.0, 0.0)"), ns)
    monkeypatch.setattr(oracle, "combine_partials", ns["combine_partials"])
    with pytest.raises(AssertionError):
        test_merged_shard_partials_are_the_full_decode(2, 0, 6)
