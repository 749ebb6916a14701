"""GPU parity on EVERY output row of the full-size prefill workloads C1
(intra) and C2 (cross): n=4, L=4096 (nL=16384), batch 2, 32 query / 8 KV
heads, head_dim 128, bf16 in and out -- against the float64 oracle, computed
in blocks of query rows on the host cores (a thread pool over (batch, head,
block) units; numpy's BLAS one thread per worker).  Intra rows are checked
through the oracle on each de-interleaved stream with n = 1 (the pins show
intra-stream attention equals independent causal attention per stream), so
only the score blocks that can be visible are formed.

Plus the long-context workload C3 (n=4, L=32768, 64/8 heads, W=4096) on
sampled rows of every (head, stream)."""

import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, lib, to_f64

pytestmark = pytest.mark.gpu

BLOCK = 1024


@pytest.fixture(scope="module")
def hd():
    return lib()


def _workers():
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(16, os.cpu_count() or 1))


def _blas_one_thread():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        import contextlib
        return contextlib.nullcontext()


def _host(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_prefill_every_row(hd, mode):
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 1101)
    k = synth.normal_device((B, P, Hkv, D), 1102)
    v = synth.normal_device((B, P, Hkv, D), 1103)
    st = hd.new_status()
    o = hd.hd_attn_fwd(q, k, v, n, mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qh, kh, vh, oh = _host(q), _host(k), _host(v), _host(o)
    del q, k, v, o
    torch.cuda.empty_cache()
    if mode == "intra":
        # stream s of batch b: rows i*n + s, checked as one causal sequence
        views = [(b, s) for b in range(B) for s in range(n)]
        units = [(b, s, h, p0) for (b, s) in views for h in range(Hq) for p0 in range(0, L, BLOCK)]
    else:
        units = [(b, None, h, p0) for b in range(B) for h in range(Hq) for p0 in range(0, P, BLOCK)]

    def one(u):
        b, s, h, p0 = u
        if s is None:
            ro, _ = oracle.attn_rows_block(qh, kh, vh, n, "cross", b, h, p0, min(P, p0 + BLOCK))
            got = oh[b, p0:p0 + BLOCK, h]
        else:
            ro, _ = oracle.attn_rows_block(qh[b:b + 1, s::n], kh[b:b + 1, s::n], vh[b:b + 1, s::n], 1, "intra",
                                           0, h, p0, min(L, p0 + BLOCK))
            got = oh[b, s::n][p0:p0 + BLOCK, h]
        return float(np.max(np.abs(got - ro)))

    with _blas_one_thread(), cf.ThreadPoolExecutor(_workers()) as ex:
        errs = list(ex.map(one, units))
    worst = max(errs)
    assert worst <= TOL_BF16, (worst, units[int(np.argmax(errs))])


def test_long_context_rows_of_every_head_and_stream(hd):
    B, n, L, Hq, Hkv, D, W = 1, 4, 32768, 64, 8, 128, 4096
    P, G = n * L, Hq // Hkv
    q = synth.normal_device((B, P, Hq, D), 1201)
    k = synth.normal_device((B, P, Hkv, D), 1202)
    v = synth.normal_device((B, P, Hkv, D), 1203)
    st = hd.new_status()
    o = hd.hd_attn_fwd(q, k, v, n, "intra", W, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = synth.rng(1204)
    worst = 0.0
    for kv in range(Hkv):
        kh = to_f64(k[:, :, kv:kv + 1])
        vh = to_f64(v[:, :, kv:kv + 1])
        for h in range(kv * G, (kv + 1) * G):
            toks = [0, L - 1] + g.integers(0, L, size=2).tolist()
            pos = sorted({i * n + s for i in toks for s in range(n)})
            qh = np.zeros((1, P, 1, D))
            qh[0, pos, 0] = to_f64(q[0, pos, h])
            ro, _ = oracle.attn_rows(qh, kh, vh, n, "intra", [(0, 0, p) for p in pos], W)
            got = to_f64(o[0, pos, h])
            worst = max(worst, float(np.max(np.abs(got - ro))))
    assert worst <= TOL_BF16, worst


@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_backward_every_row(hd, mode):
    """dQ, dK, dV of the full-size backward workload (forward then backward
    through the library) against the blocked float64 oracle, every row."""
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P, G = n * L, Hq // Hkv
    q = synth.normal_device((B, P, Hq, D), 1301)
    k = synth.normal_device((B, P, Hkv, D), 1302)
    v = synth.normal_device((B, P, Hkv, D), 1303)
    dO = synth.normal_device((B, P, Hq, D), 1304)
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(q, k, v, n, mode, lse=True, dev_status=st)
    dq, dk, dv = hd.hd_attn_bwd(q, k, v, o, dO, lse, n, mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qh, kh, vh, gh = _host(q), _host(k), _host(v), _host(dO)
    dqh, dkh, dvh = _host(dq), _host(dk), _host(dv)
    del q, k, v, dO, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    if mode == "intra":
        units = [(b, s, kvh) for b in range(B) for s in range(n) for kvh in range(Hkv)]
    else:
        units = [(b, None, kvh) for b in range(B) for kvh in range(Hkv)]

    def one(u):
        b, s, kvh = u
        hs = slice(kvh * G, (kvh + 1) * G)
        if s is None:
            rq, rk, rv = oracle.attn_bwd_blocked(qh, kh, vh, gh, n, "cross", b, kvh)
            gq, gk, gv = dqh[b, :, hs], dkh[b, :, kvh], dvh[b, :, kvh]
        else:
            sl = lambda x: x[b:b + 1, s::n]  # noqa: E731
            rq, rk, rv = oracle.attn_bwd_blocked(sl(qh), sl(kh), sl(vh), sl(gh), 1, "intra", 0, kvh)
            gq, gk, gv = dqh[b, s::n, hs], dkh[b, s::n, kvh], dvh[b, s::n, kvh]
        return tuple(float(np.max(np.abs(g - r))) / max(1.0, float(np.max(np.abs(r))))
                     for g, r in ((gq, rq), (gk, rk), (gv, rv)))

    with _blas_one_thread(), cf.ThreadPoolExecutor(_workers()) as ex:
        errs = np.array(list(ex.map(one, units)))
    assert errs.max() <= TOL_BF16, (errs.max(axis=0), units[int(np.argmax(errs.max(axis=1)))])
