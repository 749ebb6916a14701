"""GPU parity at full workload sizes, in the launch configuration the bench
times, on sampled outputs the oracle computes one row at a time.

Inputs are drawn on the device by a seeded torch generator; the sampled
rows' inputs are copied to the host for the float64 oracle.  Sampled rows
include the first and last positions, tile boundaries and rows of every
stream.
"""

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, lib, max_abs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hd():
    return lib()


def _sample_positions(P, n, k, seed):
    g = synth.rng(seed)
    fixed = [0, 1, n - 1, 127, 128, 129, P // 2, P - n, P - 1]
    rand = g.integers(0, P, size=k).tolist()
    return sorted(set(p for p in fixed + rand if 0 <= p < P))


class _QRows:
    """Stands in for q[b, p, h, :] with a few prefetched rows (one head)."""

    def __init__(self, rows, shape):
        self.rows = rows
        self.shape = shape

    def __getitem__(self, idx):
        return self.rows[idx[1]]


def _check_prefill_rows(q, k, v, o, n, mode, W, heads, positions, batches):
    """Oracle rows for (b, h, p) from a host copy of one GQA group's K/V."""
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    worst = 0.0
    for b in batches:
        for h in heads:
            kv = h // G
            kh = to_f64(k[b:b + 1, :, kv:kv + 1])
            vh = to_f64(v[b:b + 1, :, kv:kv + 1])
            qh = to_f64(q[b, positions, h])  # [R, D]
            qv = _QRows({p: qh[r] for r, p in enumerate(positions)}, (1, P, 1, D))
            ref, _ = oracle.attn_rows(qv, kh, vh, n, mode, [(0, 0, p) for p in positions], W, D ** -0.5)
            got = to_f64(o[b, positions, h])
            worst = max(worst, max_abs(got, ref))
    return worst


@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_prefill_full_size_sampled(hd, mode):
    """n=4, L=4096 (nL=16384), batch 2, 32/8 heads, head_dim 128, bf16."""
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 101)
    k = synth.normal_device((B, P, Hkv, D), 102)
    v = synth.normal_device((B, P, Hkv, D), 103)
    st = hd.new_status()
    o = hd.hd_attn_fwd(q, k, v, n, mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.isfinite(o.float()).all()
    positions = _sample_positions(P, n, 12, 104)
    err = _check_prefill_rows(q, k, v, o, n, mode, 0, heads=[0, 5, 31], positions=positions, batches=[0, 1])
    assert err <= TOL_BF16, err


def test_long_context_expand_window_gather_sampled(hd):
    """n=4, L=32768 (nL=131072), 64/8 heads, W=4096 tokens (intra), with the
    expand over 4 x 152064 x 4096 bf16 tables and Zipf(1.1) ids, and the
    final-stream gather."""
    B, n, L, Hq, Hkv, D, V, dm, W = 1, 4, 32768, 64, 8, 128, 152064, 4096, 4096
    P = n * L
    ids = synth.ids_zipf(B, L, V, 1.1, 201)
    tables = synth.normal_device((n, V, dm), 202, std=0.02)
    st = hd.new_status()
    x = hd.hd_expand_embed(tables, synth.to_torch(ids, "i32", "cuda"), dev_status=st)
    g = hd.hd_final_stream_gather(x, n)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # expand: sampled rows bit-exact
    rng = synth.rng(203)
    for i in [0, L - 1] + rng.integers(0, L, size=64).tolist():
        for s in range(n):
            assert torch.equal(x[0, i * n + s], tables[s, int(ids[0, i])])
        assert torch.equal(g[0, i], x[0, i * n + n - 1])
    del x, g, tables
    torch.cuda.empty_cache()

    q = synth.normal_device((B, P, Hq, D), 204)
    k = synth.normal_device((B, P, Hkv, D), 205)
    v = synth.normal_device((B, P, Hkv, D), 206)
    o = hd.hd_attn_fwd(q, k, v, n, "intra", W, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    positions = _sample_positions(P, n, 10, 207) + [4095 * n, 4096 * n + 1, 4097 * n + 3]
    positions = sorted(set(positions))
    err = _check_prefill_rows(q, k, v, o, n, "intra", W, heads=[0, 63], positions=positions, batches=[0])
    assert err <= TOL_BF16, err


@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_decode_full_size_sampled(hd, mode):
    """Batch 64, n=4, 32768 tokens per stream, 64/8 heads, bf16 cache (32 GiB)."""
    B, n, T, Hq, Hkv, D = 64, 4, 32768, 64, 8, 128
    G = Hq // Hkv
    q = synth.normal_device((B, n, Hq, D), 301)
    kc = synth.normal_device((B, n, T, Hkv, D), 302)
    vc = synth.normal_device((B, n, T, Hkv, D), 303)
    ctx = torch.full((B,), T, dtype=torch.int32, device="cuda")
    st = hd.new_status()
    o = hd.hd_attn_decode(q, kc, vc, ctx, mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    worst = 0.0
    for b, kv in [(0, 0), (37, 5), (63, 7)]:
        kh = to_f64(kc[b:b + 1, :, :, kv:kv + 1])
        vh = to_f64(vc[b:b + 1, :, :, kv:kv + 1])
        qh = to_f64(q[b:b + 1, :, kv * G:(kv + 1) * G])
        rows = [(0, s, g) for s in range(n) for g in (0, G - 1)]
        ro, _ = oracle.decode_rows(qh, kh, vh, np.array([T]), n, mode, rows)
        got = np.stack([to_f64(o[b, s, kv * G + g]) for (_, s, g) in rows])
        worst = max(worst, max_abs(got, ro))
    assert worst <= TOL_BF16, worst
