"""GPU parity of the attention backward (``hd_attn_bwd``) against the float64
oracle: small cases element by element (several tiles, ragged tails, GQA,
windows, n = 1, one token per stream, D = 64 and 128, both element types),
the forward -> backward chain through the library, and the full workload
sizes on sampled rows plus the softmax identities over every key.

Bound: the parity bound of the element type times the output's scale,
max|err| <= TOL * max(1, max|ref|).  Gradients are sums of many products and
can exceed 1; the bf16 path rounds P and dS to bf16 once before each tensor-
core product (relative 2^-9), so its error grows with the gradient's size."""

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, TOL_F32, dev, host_qkv, lib, max_abs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hd():
    return lib()


def _bound(ref, tol):
    return tol * max(1.0, float(np.max(np.abs(ref))))


def _round(x, dtype):
    x = np.asarray(x, dtype=np.float32)
    return synth.bf16_round(x) if dtype == "bf16" else x


CASES = [
    # dtype, mode, W, B, L, n, Hq, Hkv, D
    ("f32", "intra", 0, 1, 200, 2, 4, 2, 64),
    ("f32", "cross", 0, 1, 100, 3, 2, 1, 128),
    ("f32", "intra", 37, 2, 150, 2, 2, 2, 64),
    ("f32", "cross", 50, 1, 90, 2, 2, 2, 128),
    ("bf16", "intra", 0, 2, 300, 2, 4, 2, 128),
    ("bf16", "cross", 0, 1, 150, 3, 4, 1, 128),
    ("bf16", "intra", 100, 1, 400, 2, 2, 2, 128),
    ("bf16", "cross", 200, 1, 160, 4, 4, 2, 64),
    ("bf16", "intra", 0, 1, 257, 2, 2, 1, 64),
    ("bf16", "intra", 0, 1, 1, 3, 2, 1, 128),
    ("bf16", "cross", 0, 1, 128, 1, 2, 2, 128),
    ("bf16", "cross", 1, 1, 70, 3, 2, 2, 128),
]


@pytest.mark.parametrize("dtype,mode,W,B,L,n,Hq,Hkv,D", CASES)
def test_bwd_matches_oracle(hd, dtype, mode, W, B, L, n, Hq, Hkv, D):
    P = n * L
    scale = D ** -0.5
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 500 + L, dtype)
    dO = synth.normal((B, P, Hq, D), 600 + L, dtype=dtype)
    ro, rl = oracle.attn(q, k, v, n, mode, W, scale)
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, dO, n, mode, W, scale)
    st = hd.new_status()
    dq, dk, dv = hd.hd_attn_bwd(dev(q, dtype), dev(k, dtype), dev(v, dtype), dev(_round(ro, dtype), dtype),
                                dev(dO, dtype), dev(rl, "f32"), n, mode, W, scale, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        err = max_abs(to_f64(got), ref)
        assert err <= _bound(ref, tol), (name, err, float(np.max(np.abs(ref))))


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 70)])
def test_bwd_scores_beyond_the_exponent_range(hd, mode, W):
    """Queries scaled by 40: within a row many exponents s*scale - lse fall
    below -126, where the FMA-pipe exponential clamps to ~2^-126 instead of
    0; dQ, dK and dV still match the oracle and stay finite."""
    B, L, n, Hq, Hkv, D = 1, 300, 2, 4, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 720, "bf16")
    q = synth.bf16_round(q.astype(np.float32) * np.float32(40.0))
    dO = synth.normal((B, P, Hq, D), 723, dtype="bf16")
    ro, rl = oracle.attn(q, k, v, n, mode, W)
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    st = hd.new_status()
    dq, dk, dv = hd.hd_attn_bwd(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(_round(ro, "bf16"), "bf16"),
                                dev(dO, "bf16"), dev(rl, "f32"), n, mode, W, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        g = to_f64(got)
        assert np.isfinite(g).all(), name
        err = max_abs(g, ref)
        assert err <= _bound(ref, TOL_BF16), (name, err, float(np.max(np.abs(ref))))


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("cross", 300)])
def test_forward_backward_chain(hd, mode, W):
    """O and lse from the library's forward feed its backward."""
    B, L, n, Hq, Hkv, D = 1, 260, 3, 4, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 700, "bf16")
    dO = synth.normal((B, P, Hq, D), 703, dtype="bf16")
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    o, lse = hd.hd_attn_fwd(qd, kd, vd, n, mode, W, lse=True)
    dq, dk, dv = hd.hd_attn_bwd(qd, kd, vd, o, dev(dO, "bf16"), lse, n, mode, W)
    torch.cuda.synchronize()
    rdq, rdk, rdv = oracle.attn_bwd(q, k, v, dO, n, mode, W)
    for got, ref in ((dq, rdq), (dk, rdk), (dv, rdv)):
        assert max_abs(to_f64(got), ref) <= _bound(ref, TOL_BF16)


def test_bwd_repeatable_and_workspace_reuse(hd):
    """Two calls on one workspace give identical bits (no atomics, no state)."""
    B, L, n, Hq, Hkv, D = 1, 300, 2, 4, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 710, "bf16")
    dO = synth.normal((B, P, Hq, D), 713, dtype="bf16")
    ro, rl = oracle.attn(q, k, v, n, "intra")
    args = (dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), dev(_round(ro, "bf16"), "bf16"), dev(dO, "bf16"),
            dev(rl, "f32"), n, "intra")
    ws = torch.empty(hd.hd_attn_bwd_workspace(B, L, n, Hq, "intra"), dtype=torch.uint8, device="cuda")
    a = hd.hd_attn_bwd(*args, workspace=ws)
    ws.fill_(0xFF)
    b = hd.hd_attn_bwd(*args, workspace=ws)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ------------------------------------------------------------- full size

@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_bwd_full_size_sampled(hd, mode):
    """n=4, L=4096 (nL=16384), batch 2, 32/8 heads, head_dim 128, bf16: the
    bench's backward workload, forward then backward through the library."""
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P, G = n * L, Hq // Hkv
    q = synth.normal_device((B, P, Hq, D), 801)
    k = synth.normal_device((B, P, Hkv, D), 802)
    v = synth.normal_device((B, P, Hkv, D), 803)
    dO = synth.normal_device((B, P, Hq, D), 804)
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(q, k, v, n, mode, lse=True, dev_status=st)
    dq, dk, dv = hd.hd_attn_bwd(q, k, v, o, dO, lse, n, mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()

    # Identities over every key: rows of dS sum to zero, rows of P to one.
    # Bound: 2^-5 of the root-sum-square of the summed rows (the random-walk
    # size of per-element bf16 rounding is ~2^-10 of it), plus 1e-3.
    ns = n if mode == "intra" else 1
    dk64 = dk.double().view(B, P // ns, ns, Hkv, D)
    dv64 = dv.double().view(B, P // ns, ns, Hkv, D)
    sum_dk = dk64.sum(dim=1)
    want_dv = dO.double().view(B, P // ns, ns, Hkv, G, D).sum(dim=(1, 4))
    err_k = (sum_dk.abs() - 2.0 ** -5 * dk64.pow(2).sum(dim=1).sqrt() - 1e-3).max().item()
    err_v = ((dv64.sum(dim=1) - want_dv).abs() - 2.0 ** -5 * dv64.pow(2).sum(dim=1).sqrt() - 1e-3).max().item()
    assert err_k <= 0 and err_v <= 0, (err_k, err_v)

    # Sampled rows against the oracle, one GQA group at a time.
    worst = 0.0
    for b, kv in [(0, 0), (1, 5)]:
        kh = to_f64(k[b:b + 1, :, kv:kv + 1])
        vh = to_f64(v[b:b + 1, :, kv:kv + 1])
        qh = to_f64(q[b:b + 1, :, kv * G:(kv + 1) * G])
        oh = to_f64(dO[b:b + 1, :, kv * G:(kv + 1) * G])
        qpos = [0, 1, n - 1, 127 * n, 128 * n + 1, P // 2 + 2, P - n, P - 1]
        rows = [(0, g, p) for g in (0, G - 1) for p in qpos]
        ref = oracle.attn_bwd_dq_rows(qh, kh, vh, oh, n, mode, rows)
        got = np.stack([to_f64(dq[b, p, kv * G + g]) for (_, g, p) in rows])
        worst = max(worst, max_abs(got, ref) / max(1.0, float(np.max(np.abs(ref)))))
        kpos = list(range(P - 6, P)) + [(L - 40) * n + 1]
        krows = [(0, 0, p) for p in kpos]
        rk, rv = oracle.attn_bwd_dkv_rows(qh, kh, vh, oh, n, mode, krows)
        gk = np.stack([to_f64(dk[b, p, kv]) for p in kpos])
        gv = np.stack([to_f64(dv[b, p, kv]) for p in kpos])
        worst = max(worst, max_abs(gk, rk) / max(1.0, float(np.max(np.abs(rk)))))
        worst = max(worst, max_abs(gv, rv) / max(1.0, float(np.max(np.abs(rv)))))
    assert worst <= TOL_BF16, worst


FS_CASES = [
    # dtype, mode, W, B, L, n, Hq, Hkv, D
    ("bf16", "intra", 0, 2, 300, 4, 4, 2, 128),
    ("bf16", "cross", 0, 1, 260, 4, 4, 1, 128),
    ("bf16", "cross", 100, 1, 200, 3, 2, 2, 64),
    ("bf16", "cross", 2, 1, 150, 4, 2, 2, 128),   # window < n: some keys seen by no query
    ("f32", "intra", 0, 1, 130, 3, 2, 1, 64),
    ("f32", "cross", 50, 1, 90, 2, 2, 2, 128),
]


@pytest.mark.parametrize("dtype,mode,W,B,L,n,Hq,Hkv,D", FS_CASES)
def test_final_stream_bwd_matches_oracle(hd, dtype, mode, W, B, L, n, Hq, Hkv, D):
    P = n * L
    scale = D ** -0.5
    qf = synth.normal((B, L, Hq, D), 1400 + L, dtype=dtype)
    k = synth.normal((B, P, Hkv, D), 1401 + L, dtype=dtype)
    v = synth.normal((B, P, Hkv, D), 1402 + L, dtype=dtype)
    gf = synth.normal((B, L, Hq, D), 1403 + L, dtype=dtype)
    of, lf = oracle.attn_final_stream(qf, k, v, n, mode, W, scale)
    rq, rk, rv = oracle.attn_bwd_final_stream(qf, k, v, gf, n, mode, W, scale)
    st = hd.new_status()
    dk0 = torch.full(k.shape, 7.0, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    dq, dk, dv = hd.hd_attn_bwd_final_stream(dev(qf, dtype), dev(k, dtype), dev(v, dtype), dev(_round(of, dtype), dtype),
                                             dev(gf, dtype), dev(lf, "f32"), n, mode, W, scale, dk=dk0,
                                             dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        err = max_abs(to_f64(got), ref)
        assert err <= _bound(ref, tol), (name, err)
    if mode == "intra":  # keys of streams 0..n-2 are seen by no final-stream query
        assert not to_f64(dk)[:, np.arange(P) % n != n - 1].any()


def test_final_stream_bwd_chain(hd):
    """Forward and backward of the final-stream call through the library."""
    B, L, n, Hq, Hkv, D = 1, 260, 4, 4, 2, 128
    qf = synth.normal((B, L, Hq, D), 1501, dtype="bf16")
    k = synth.normal((B, n * L, Hkv, D), 1502, dtype="bf16")
    v = synth.normal((B, n * L, Hkv, D), 1503, dtype="bf16")
    gf = synth.normal((B, L, Hq, D), 1504, dtype="bf16")
    qd, kd, vd = dev(qf, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    for mode in ("intra", "cross"):
        of, lf = hd.hd_attn_fwd_final_stream(qd, kd, vd, n, mode, lse=True)
        grads = hd.hd_attn_bwd_final_stream(qd, kd, vd, of, dev(gf, "bf16"), lf, n, mode)
        torch.cuda.synchronize()
        for got, ref in zip(grads, oracle.attn_bwd_final_stream(qf, k, v, gf, n, mode)):
            assert max_abs(to_f64(got), ref) <= _bound(ref, TOL_BF16)
