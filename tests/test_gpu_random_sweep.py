"""Seeded random sweep of the attention calls against the float64 oracle.

Beyond the hand-picked cases of the other GPU tests: shapes drawn from a
fixed generator (stream count n, tokens per stream L including ragged tails,
query/KV heads with every GQA ratio, head dim 64 or 128, window or none, mode,
input dtype), each case run through the forward, the final-stream forward,
decode and the backward.  Sizes stay small enough for the oracle to finish in
seconds; the same seeds give the same cases on every run."""

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, TOL_F32, dev, lib, max_abs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hd():
    return lib()


def _case(seed):
    g = np.random.default_rng(seed)
    n = int(g.choice([1, 2, 3, 4, 5, 8]))
    L = int(g.integers(1, 300 // n + 40))
    Hkv = int(g.choice([1, 2, 3]))
    G = int(g.choice([1, 2, 3, 4, 8]))
    D = int(g.choice([64, 128]))
    mode = str(g.choice(["intra", "cross"]))
    W = 0 if g.random() < 0.5 else int(g.integers(1, max(2, (L if mode == "intra" else n * L))))
    dt = "bf16" if g.random() < 0.75 else "f32"
    return n, L, Hkv * G, Hkv, D, mode, W, dt


SEEDS = list(range(9000, 9096))


@pytest.mark.parametrize("seed", SEEDS)
def test_forward_and_final_stream(hd, seed):
    n, L, Hq, Hkv, D, mode, W, dt = _case(seed)
    B, P = 2, n * L
    q = synth.normal((B, P, Hq, D), seed, dtype=dt)
    k = synth.normal((B, P, Hkv, D), seed + 1, dtype=dt)
    v = synth.normal((B, P, Hkv, D), seed + 2, dtype=dt)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(dev(q, dt), dev(k, dt), dev(v, dt), n, mode, W, lse=True, out_dtype=torch.float32,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.attn(q, k, v, n, mode, W)
    assert max_abs(to_f64(o), ro) <= tol, (n, L, Hq, Hkv, D, mode, W, dt)
    assert max_abs(to_f64(lse), rl) <= (1e-3 if dt == "bf16" else 1e-4)
    qf = np.ascontiguousarray(q.reshape(B, L, n, Hq, D)[:, :, n - 1])
    of = hd.hd_attn_fwd_final_stream(dev(qf, dt), dev(k, dt), dev(v, dt), n, mode, W, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rf, _ = oracle.attn_final_stream(qf, k, v, n, mode, W)
    assert max_abs(to_f64(of), rf) <= tol


@pytest.mark.parametrize("seed", SEEDS[:48])
def test_backward(hd, seed):
    n, L, Hq, Hkv, D, mode, W, dt = _case(seed)
    B, P = 1, n * L
    q = synth.normal((B, P, Hq, D), seed + 10, dtype=dt)
    k = synth.normal((B, P, Hkv, D), seed + 11, dtype=dt)
    v = synth.normal((B, P, Hkv, D), seed + 12, dtype=dt)
    dO = synth.normal((B, P, Hq, D), seed + 13, dtype=dt)
    qd, kd, vd, gd = dev(q, dt), dev(k, dt), dev(v, dt), dev(dO, dt)
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(qd, kd, vd, n, mode, W, lse=True, dev_status=st)
    dq, dk, dv = hd.hd_attn_bwd(qd, kd, vd, o, gd, lse, n, mode, W, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rq, rk, rv = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    tol = TOL_BF16 if dt == "bf16" else TOL_F32
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert max_abs(to_f64(got), ref) <= tol * max(1.0, float(np.max(np.abs(ref)))), (n, L, Hq, Hkv, D, mode, W)


@pytest.mark.parametrize("seed", SEEDS[:48])
def test_decode(hd, seed):
    n, L, Hq, Hkv, D, mode, W, dt = _case(seed)
    D = 128  # the decode kernels take head dim 128
    B, Lmax = 3, L + 7
    q = synth.normal((B, n, Hq, D), seed + 20, dtype="bf16")
    kc = synth.normal((B, n, Lmax, Hkv, D), seed + 21, dtype="bf16")
    vc = synth.normal((B, n, Lmax, Hkv, D), seed + 22, dtype="bf16")
    g = np.random.default_rng(seed + 23)
    ctx = g.integers(1, Lmax + 1, size=B).astype(np.int32)
    st = hd.new_status()
    o, lse = hd.hd_attn_decode(dev(q, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"), mode, W,
                               out_dtype=torch.float32, lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.decode(q, kc, vc, ctx, n, mode, W)
    assert max_abs(to_f64(o), ro) <= TOL_BF16, (n, Lmax, Hq, Hkv, mode, W, ctx.tolist())
    assert max_abs(to_f64(lse), rl) <= 1e-3


def _shard(x, n, R, r):
    """Rank r's streams of x [B, n*L, ...] in local order (reshape, no oracle)."""
    B, P = x.shape[:2]
    L, nl = P // n, n // R
    return np.ascontiguousarray(x.reshape((B, L, nl, R) + x.shape[2:])[:, :, :, r].reshape((B, L * nl) + x.shape[2:]))


@pytest.mark.parametrize("seed", list(range(9100, 9132)))
def test_rank_shard_prefill(hd, seed):
    """hd_attn_fwd_parts and hd_attn_fwd_peer_gather for a random rank of a
    random stream-parallel layout (R | n, n | 128), against the oracle."""
    g = np.random.default_rng(seed)
    n = int(g.choice([1, 2, 4, 8]))
    R = int(g.choice([d for d in (1, 2, 4, 8) if n % d == 0]))
    r = int(g.integers(0, R))
    L = int(g.integers(1, 400 // n + 20))
    Hkv = int(g.choice([1, 2]))
    Hq = Hkv * int(g.choice([1, 2, 3, 4]))
    D = int(g.choice([64, 128]))
    W = 0 if g.random() < 0.6 else int(g.integers(1, n * L + 1))
    B, P = 2, n * L
    q = synth.normal((B, P, Hq, D), seed, dtype="bf16")
    k = synth.normal((B, P, Hkv, D), seed + 1, dtype="bf16")
    v = synth.normal((B, P, Hkv, D), seed + 2, dtype="bf16")
    ro, _ = oracle.attn(q, k, v, n, "cross", W)
    want = _shard(ro, n, R, r)
    # Shards either as the slots of one [R, ...] tensor (one stride: the
    # stacked view) or as separate tensors with gaps between them.
    stacked = bool(g.random() < 0.5)
    if stacked:
        kstk = dev(np.stack([_shard(k, n, R, rho) for rho in range(R)]), "bf16")
        vstk = dev(np.stack([_shard(v, n, R, rho) for rho in range(R)]), "bf16")
        ks, vs = list(kstk), list(vstk)
    else:
        ks, vs, gaps = [], [], []
        for rho in range(R):
            ks.append(dev(_shard(k, n, R, rho), "bf16"))
            gaps.append(torch.empty(4096 * (rho + 1), dtype=torch.uint8, device="cuda"))
            vs.append(dev(_shard(v, n, R, rho), "bf16"))
    ql = dev(_shard(q, n, R, r), "bf16")
    st = hd.new_status()
    o1 = hd.hd_attn_fwd_parts(ql, ks, vs, n, R, r, W, out_dtype=torch.float32, dev_status=st)
    own_slot = bool(g.random() < 0.7)
    kdt = torch.zeros((R,) + tuple(ks[0].shape), dtype=torch.bfloat16, device="cuda")
    vdt = torch.zeros_like(kdt)
    kd = [None if (rho == r and not own_slot) else kdt[rho] for rho in range(R)]
    vd = [None if (rho == r and not own_slot) else vdt[rho] for rho in range(R)]
    o2 = hd.hd_attn_fwd_peer_gather(ql, ks, vs, kd, vd, n, R, r, window=W, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    case = (n, R, r, L, Hq, Hkv, D, W, stacked, own_slot)
    assert max_abs(to_f64(o1), want) <= TOL_BF16, case
    assert max_abs(to_f64(o2), want) <= TOL_BF16, case
    for rho in range(R):
        if R > 1 and (rho != r or own_slot):
            assert torch.equal(kd[rho].view(torch.int16), ks[rho].view(torch.int16)), case
            assert torch.equal(vd[rho].view(torch.int16), vs[rho].view(torch.int16)), case
