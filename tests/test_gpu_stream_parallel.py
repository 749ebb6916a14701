"""GPU parity of the stream-parallel calls, with R ranks run one after
another on one device: what an all-gather would deliver is the stack of the
ranks' shards.  (Kernels of different ranks never wait on one another, so
running them in sequence is exact.)  Checked against the float64 oracle:
the re-interleave bit-exact, the cross-stream prefill rows of each rank, the
per-rank decode partials (including ranks that see no key), and their merge
= the full cross-stream decode; plus the merge kernel on its own."""

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


def _shard(x, n, R, r):
    """Rank r's streams of x [B, n*L, ...] in local order (reshape, no oracle)."""
    B, P = x.shape[:2]
    L, nl = P // n, n // R
    return np.ascontiguousarray(x.reshape((B, L, nl, R) + x.shape[2:])[:, :, :, r].reshape((B, L * nl) + x.shape[2:]))


@pytest.mark.parametrize("R", [2, 4])
def test_interleave_restores_the_expanded_order(hd, R):
    n, B, L = 4, 2, 37
    x = synth.normal((B, n * L, 8, 128), 1001, dtype="bf16")
    parts = np.stack([_shard(x, n, R, r) for r in range(R)])
    out = hd.hd_stream_interleave(dev(parts, "bf16"), n)
    torch.cuda.synchronize()
    want = oracle.stream_interleave(parts, n)
    assert np.array_equal(want, x)
    assert np.array_equal(out.float().cpu().numpy().view(np.uint32), want.astype(np.float32).view(np.uint32))


@pytest.mark.parametrize("R,W,dtype", [(2, 0, "bf16"), (4, 0, "bf16"), (2, 150, "bf16"), (4, 0, "f32")])
def test_cross_prefill_shards(hd, R, W, dtype):
    n, B, L, Hq, Hkv, D = 4, 1, 150, 4, 2, 128
    P = n * L
    q = synth.normal((B, P, Hq, D), 1011, dtype=dtype)
    k = synth.normal((B, P, Hkv, D), 1012, dtype=dtype)
    v = synth.normal((B, P, Hkv, D), 1013, dtype=dtype)
    ro, rl = oracle.attn(q, k, v, n, "cross", W)
    kparts = dev(np.stack([_shard(k, n, R, r) for r in range(R)]), dtype)
    vparts = dev(np.stack([_shard(v, n, R, r) for r in range(R)]), dtype)
    kd, vd = hd.hd_stream_interleave(kparts, n), hd.hd_stream_interleave(vparts, n)
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    for r in range(R):
        o, lse = hd.hd_attn_fwd_shard(dev(_shard(q, n, R, r), dtype), kd, vd, n, R, r, W, lse=True,
                                      out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert max_abs(to_f64(o), _shard(ro, n, R, r)) <= tol
        want_lse = _shard(np.transpose(rl, (0, 2, 1)), n, R, r)  # [B, P_loc, Hq]
        assert max_abs(np.transpose(to_f64(lse), (0, 2, 1)), want_lse) <= 1e-3


@pytest.mark.parametrize("R", [2, 4])
def test_intra_prefill_shards_need_no_exchange(hd, R):
    n, B, L, H, D = 4, 1, 130, 2, 128
    q = synth.normal((B, n * L, H, D), 1021, dtype="bf16")
    k = synth.normal((B, n * L, H, D), 1022, dtype="bf16")
    v = synth.normal((B, n * L, H, D), 1023, dtype="bf16")
    ro, _ = oracle.attn(q, k, v, n, "intra")
    for r in range(R):
        o = hd.hd_attn_fwd(*(dev(_shard(x, n, R, r), "bf16") for x in (q, k, v)), n // R, "intra")
        torch.cuda.synchronize()
        assert max_abs(to_f64(o), _shard(ro, n, R, r)) <= TOL_BF16


@pytest.mark.parametrize("R,T,W", [(2, 300, 0), (4, 300, 0), (4, 1, 0), (2, 70, 64), (4, 2, 5)])
def test_cross_decode_shards_and_merge(hd, R, T, W):
    n, B, Lmax, Hq, Hkv, D = 4, 2, 320, 8, 2, 128
    q = synth.normal((B, n, Hq, D), 1031, dtype="bf16")
    kc = synth.normal((B, n, Lmax, Hkv, D), 1032, dtype="bf16")
    vc = synth.normal((B, n, Lmax, Hkv, D), 1033, dtype="bf16")
    ctx = np.array([T, max(1, T // 2)], dtype=np.int32)
    ctx_d = dev(ctx, "i32")
    rows = [(b, s, h) for b in range(B) for s in range(n) for h in range(Hq)]
    # The all-gather of the ranks' stream queries restores q.
    qparts = np.stack([q[:, r::R] for r in range(R)])
    qd = hd.hd_stream_interleave(dev(qparts, "bf16"), n)
    torch.cuda.synchronize()
    assert np.array_equal(qd.float().cpu().numpy(), q)
    o_parts, l_parts = [], []
    for r in range(R):
        st = oracle.shard_streams(n, R, r)
        o, lse = hd.hd_attn_decode_shard(qd, dev(kc[:, st].copy(), "bf16"), dev(vc[:, st].copy(), "bf16"), ctx_d,
                                         R, r, W)
        torch.cuda.synchronize()
        ro, rl = oracle.decode_rows_streams(q, kc[:, st], vc[:, st], ctx, n, st, rows, W)
        got_o = to_f64(o).reshape(-1, D)
        got_l = to_f64(lse).reshape(-1)
        empty = np.isneginf(rl)
        assert np.array_equal(np.isneginf(got_l), empty)
        assert not got_o[empty].any()
        assert max_abs(got_o, ro) <= TOL_BF16
        assert max_abs(got_l[~empty], rl[~empty]) <= 1e-3
        o_parts.append(o)
        l_parts.append(lse)
    if T == 1:
        assert torch.isneginf(torch.stack(l_parts)).any()
    om, lm = hd.hd_attn_combine(torch.stack(o_parts), torch.stack(l_parts), out_dtype=torch.float32, lse=True)
    torch.cuda.synchronize()
    fo, fl = oracle.decode_rows(q, kc, vc, ctx, n, "cross", rows, W)
    assert max_abs(to_f64(om).reshape(-1, D), fo) <= TOL_BF16
    assert max_abs(to_f64(lm).reshape(-1), fl) <= 1e-3
    # The fused form: each rank merges only its own stream rows, reading the
    # R partials through their own pointers.
    fo4 = fo.reshape(B, n, Hq, D)
    fl3 = fl.reshape(B, n, Hq)
    for r in range(R):
        ol, ll = hd.hd_attn_combine_streams(o_parts, l_parts, n, R, r, out_dtype=torch.float32, lse=True)
        torch.cuda.synchronize()
        assert ol.shape == (B, n // R, Hq, D)
        assert max_abs(to_f64(ol), fo4[:, r::R]) <= TOL_BF16
        assert max_abs(to_f64(ll), fl3[:, r::R]) <= 1e-3


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("f32", "bf16")])
def test_combine_kernel(hd, in_dt, out_dt):
    R, rows, D = 3, 257, 64
    o = synth.normal((R, rows, D), 1041, dtype=in_dt)
    l = synth.normal((R, rows), 1042).astype(np.float32) * 4
    l[0, :7] = -np.inf          # some empty parts
    l[:, 10] = -np.inf          # a row with every part empty
    wo, wl = oracle.combine_partials(o, l)
    go, gl = hd.hd_attn_combine(dev(o, in_dt), dev(l, "f32"),
                                out_dtype=torch.bfloat16 if out_dt == "bf16" else torch.float32, lse=True)
    torch.cuda.synchronize()
    tol = TOL_BF16 if out_dt == "bf16" else TOL_F32
    assert max_abs(to_f64(go), wo) <= tol
    gl = to_f64(gl)
    assert np.array_equal(np.isneginf(gl), np.isneginf(wl))
    fin = np.isfinite(wl)
    assert max_abs(gl[fin], wl[fin]) <= 1e-5


def test_orchestration_runs_end_to_end_on_one_rank(hd):
    """StreamParallel's calls (NCCL all-gathers, re-interleave, shard kernels,
    merge) in a one-rank NCCL group on this GPU: with R = 1 every layer must
    equal the plain single-GPU result, here checked against the oracle."""
    import os
    import socket

    import torch.distributed as dist

    from stream_sequence_attention_b200 import stream_parallel as sp

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        n, B, L, Hq, Hkv, D = 4, 1, 130, 4, 2, 128
        view = sp.StreamParallel(n)
        assert (view.R, view.r, view.streams) == (1, 0, [0, 1, 2, 3])
        q, k, v = (synth.normal((B, n * L, H, D), 1051 + i, dtype="bf16") for i, H in enumerate((Hq, Hkv, Hkv)))
        qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
        oc = view.cross_attention(qd, kd, vd, out_dtype=torch.float32)
        oi = view.intra_attention(qd, kd, vd, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert max_abs(to_f64(oc), oracle.attn(q, k, v, n, "cross")[0]) <= TOL_BF16
        assert max_abs(to_f64(oi), oracle.attn(q, k, v, n, "intra")[0]) <= TOL_BF16
        ps = sp.PeerShards(view, B, L, Hkv, D)
        for _ in range(3):  # cycles both buffer pairs
            op = ps.cross_attention(qd, kd, vd, out_dtype=torch.float32)
        torch.cuda.synchronize()
        ps.close()
        assert max_abs(to_f64(op), oracle.attn(q, k, v, n, "cross")[0]) <= TOL_BF16
        Lmax, T = 200, 150
        qd_ = synth.normal((2, n, 8, D), 1061, dtype="bf16")
        kc = synth.normal((2, n, Lmax, Hkv, D), 1062, dtype="bf16")
        vc = synth.normal((2, n, Lmax, Hkv, D), 1063, dtype="bf16")
        ctx = np.array([T, 7], dtype=np.int32)
        od = view.cross_decode(dev(qd_, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"))
        torch.cuda.synchronize()
        ref, _ = oracle.decode(qd_, kc, vc, ctx, n, "cross")
        assert max_abs(to_f64(od), ref) <= TOL_BF16
        pdec = sp.PeerDecode(view, 2, 8, D)
        for _ in range(3):  # cycles both buffer sets
            op = pdec.cross_decode(dev(qd_, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"))
        torch.cuda.synchronize()
        pdec.close()
        assert max_abs(to_f64(op), ref) <= TOL_BF16
    finally:
        dist.destroy_process_group()


# (n, R, L, Hq, Hkv, D, W): ragged tails, GQA, windows, every rank count that
# divides n up to the 8-rank limit (128/R rows of each shard per key tile).
PARTS_CASES = [
    (4, 1, 150, 4, 2, 128, 0),
    (4, 2, 150, 4, 2, 128, 0),
    (4, 4, 150, 4, 2, 128, 0),
    (4, 2, 150, 4, 2, 128, 150),
    (8, 8, 70, 2, 1, 128, 0),
    (8, 2, 95, 4, 4, 64, 0),
    (2, 2, 300, 6, 2, 128, 37),
    (16, 4, 40, 2, 2, 128, 0),
]


def _parts_inputs(n, R, L, Hq, Hkv, D, seed):
    B, P = 2, n * L
    q = synth.normal((B, P, Hq, D), seed, dtype="bf16")
    k = synth.normal((B, P, Hkv, D), seed + 1, dtype="bf16")
    v = synth.normal((B, P, Hkv, D), seed + 2, dtype="bf16")
    return q, k, v


@pytest.mark.parametrize("n,R,L,Hq,Hkv,D,W", PARTS_CASES)
def test_parts_prefill_reads_shards_in_place(hd, n, R, L, Hq, Hkv, D, W):
    q, k, v = _parts_inputs(n, R, L, Hq, Hkv, D, 1071)
    ro, rl = oracle.attn(q, k, v, n, "cross", W)
    kp = dev(np.stack([_shard(k, n, R, r) for r in range(R)]), "bf16")
    vp = [dev(_shard(v, n, R, r), "bf16") for r in range(R)]  # list form for v, stacked form for k
    for r in range(R):
        st = hd.new_status()
        o, lse = hd.hd_attn_fwd_parts(dev(_shard(q, n, R, r), "bf16"), kp, vp, n, R, r, W, lse=True,
                                      out_dtype=torch.float32, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert max_abs(to_f64(o), _shard(ro, n, R, r)) <= TOL_BF16
        want_lse = _shard(np.transpose(rl, (0, 2, 1)), n, R, r)
        assert max_abs(np.transpose(to_f64(lse), (0, 2, 1)), want_lse) <= 1e-3


@pytest.mark.parametrize("n,R,L,Hq,Hkv,D,W", [c for c in PARTS_CASES if c[1] > 1] + [PARTS_CASES[0]])
def test_peer_gather_copies_and_attends(hd, n, R, L, Hq, Hkv, D, W):
    """The fused form with every 'peer' shard in local memory: the same
    kernel code as with peer pointers.  Run twice with different data through
    the same destination slots and flags (the flags are reset by the call)."""
    for rep in range(2):
        q, k, v = _parts_inputs(n, R, L, Hq, Hkv, D, 1081 + 10 * rep)
        ro, _ = oracle.attn(q, k, v, n, "cross", W)
        ks = [dev(_shard(k, n, R, r), "bf16") for r in range(R)]
        vs = [dev(_shard(v, n, R, r), "bf16") for r in range(R)]
        for r in range(R):
            kd = [torch.full_like(ks[0], 7.0) for _ in range(R)]
            vd = [torch.full_like(vs[0], 7.0) for _ in range(R)]
            st = hd.new_status()
            o = hd.hd_attn_fwd_peer_gather(dev(_shard(q, n, R, r), "bf16"), ks, vs, kd, vd, n, R, r, window=W,
                                           out_dtype=torch.float32, dev_status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            assert max_abs(to_f64(o), _shard(ro, n, R, r)) <= TOL_BF16
            for rho in range(R):  # every slot given: the own shard is copied as well
                if R > 1:
                    assert torch.equal(kd[rho].view(torch.int16), ks[rho].view(torch.int16))
                    assert torch.equal(vd[rho].view(torch.int16), vs[rho].view(torch.int16))
            if R > 1:  # own slot not given: the own shard is read in place
                kd2 = [None if rho == r else torch.full_like(ks[0], 7.0) for rho in range(R)]
                vd2 = [None if rho == r else torch.full_like(vs[0], 7.0) for rho in range(R)]
                o2 = hd.hd_attn_fwd_peer_gather(dev(_shard(q, n, R, r), "bf16"), ks, vs, kd2, vd2, n, R, r,
                                                window=W, out_dtype=torch.float32, dev_status=st)
                torch.cuda.synchronize()
                assert int(st.item()) == 0
                assert max_abs(to_f64(o2), _shard(ro, n, R, r)) <= TOL_BF16


def test_parts_at_full_size_sampled_rows(hd):
    """The cross-stream prefill workload (n=4, L=4096, batch 2, 32/8 heads)
    as rank 0 of 4: the fused gather form, sampled rows of every head against
    the oracle, and the copies bit-exact."""
    n, R, r, B, L, Hq, Hkv, D = 4, 4, 0, 2, 4096, 32, 8, 128
    nl = n // R
    g = synth.rng(1091)
    ql = synth.normal_device((B, nl * L, Hq, D), 1092)
    ks = [synth.normal_device((B, nl * L, Hkv, D), 1093 + i) for i in range(R)]
    vs = [synth.normal_device((B, nl * L, Hkv, D), 1103 + i) for i in range(R)]
    kd = [torch.zeros_like(ks[0]) for _ in range(R)]
    vd = [torch.zeros_like(vs[0]) for _ in range(R)]
    st = hd.new_status()
    o = hd.hd_attn_fwd_peer_gather(ql, ks, vs, kd, vd, n, R, r, out_dtype=torch.float32, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for rho in range(1, R):
        assert torch.equal(kd[rho].view(torch.int16), ks[rho].view(torch.int16))
        assert torch.equal(vd[rho].view(torch.int16), vs[rho].view(torch.int16))
    # the expanded order: position i*n + s holds shard s % R, local row i*nl + s // R
    kx = torch.stack(ks).view(R, B, L, nl, Hkv, D).permute(1, 2, 3, 0, 4, 5).reshape(B, n * L, Hkv, D)
    vx = torch.stack(vs).view(R, B, L, nl, Hkv, D).permute(1, 2, 3, 0, 4, 5).reshape(B, n * L, Hkv, D)
    toks = sorted({0, L - 1, *g.integers(0, L, size=3).tolist()})
    rows_loc = [i * nl + l for i in toks for l in range(nl)]
    worst = 0.0
    for b in range(B):
        kh, vh = to_f64(kx[b:b + 1]), to_f64(vx[b:b + 1])
        for h in range(Hq):
            qh = np.zeros((1, n * L, 1, D))
            pos = [i * n + r + R * l for i in toks for l in range(nl)]
            qh[0, pos, 0] = to_f64(ql[b, rows_loc, h])
            kvh = h // (Hq // Hkv)
            ro, _ = oracle.attn_rows(qh, kh[:, :, kvh:kvh + 1], vh[:, :, kvh:kvh + 1], n, "cross",
                                     [(0, 0, p) for p in pos])
            worst = max(worst, float(np.max(np.abs(to_f64(o[b, rows_loc, h]) - ro))))
    assert worst <= TOL_BF16, worst


@pytest.mark.parametrize("in_dt,out_dt,R", [("f32", "f32", 2), ("bf16", "bf16", 4), ("f32", "bf16", 8),
                                            ("bf16", "f32", 2)])
def test_combine_streams_kernel(hd, in_dt, out_dt, R):
    """The own-rows merge on random partials (some parts and some rows empty),
    each part through its own pointer, against the oracle's merge."""
    B, n, Hq, D = 3, 8, 5, 64
    o = [synth.normal((B, n, Hq, D), 1601 + i, dtype=in_dt) for i in range(R)]
    lse = [synth.normal((B, n, Hq), 1611 + i).astype(np.float32) * 3 for i in range(R)]
    lse[0][0, :, :2] = -np.inf          # empty parts
    for i in range(R):
        lse[i][1, 3, 4] = -np.inf       # a row with every part empty
    wo, wl = oracle.combine_partials(np.stack(o), np.stack(lse))
    tol = TOL_BF16 if out_dt == "bf16" else TOL_F32
    for r in range(R):
        go, gl = hd.hd_attn_combine_streams([dev(x, in_dt) for x in o], [dev(x, "f32") for x in lse], n, R, r,
                                            out_dtype=torch.bfloat16 if out_dt == "bf16" else torch.float32,
                                            lse=True)
        torch.cuda.synchronize()
        assert max_abs(to_f64(go), wo[:, r::R]) <= tol
        gl = to_f64(gl)
        want = wl[:, r::R]
        assert np.array_equal(np.isneginf(gl), np.isneginf(want))
        fin = np.isfinite(want)
        assert max_abs(gl[fin], want[fin]) <= 1e-5
