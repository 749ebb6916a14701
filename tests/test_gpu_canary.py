"""Out-of-bounds write checks (compute-sanitizer is closed on this machine):
every output, in-place buffer and workspace of every C-ABI call lives inside
a canary-filled byte buffer with guard bands before and after it.  After
the call the guards must be bit-identical (no stray store past a ragged
tail, a last tile or a row map) and every output element must have been
overwritten (no row left unwritten).  Shapes are ragged, span several tiles,
and cover both head dims, both output types, windows and both modes."""

import numpy as np
import pytest
import torch

from stream_sequence_attention_b200 import synth
from tests.gpu_util import Guarded, lib

pytestmark = pytest.mark.gpu

BF, F32 = torch.bfloat16, torch.float32


@pytest.fixture(scope="module")
def hd():
    return lib()


def _ok(*gs, written=True):
    for g in gs:
        assert g.guards_intact(), "a store landed outside the buffer"
        if written:
            assert g.fully_written(), "an output element was not written"


@pytest.mark.parametrize("dtype,n,B,L,V,d", [(F32, 2, 1, 64, 512, 128), (BF, 4, 2, 37, 1000, 4096), (BF, 3, 3, 5, 7, 8)])
def test_expand_and_gather_guarded(hd, dtype, n, B, L, V, d):
    tables = synth.normal_device((n, V, d), 41, std=0.02).to(dtype)
    ids = torch.randint(0, V, (B, L), dtype=torch.int32, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    x = Guarded((B, n * L, d), dtype)
    hd.hd_expand_embed(tables, ids, out=x.t)
    _ok(x)
    g = Guarded((B, L, d), dtype)
    hd.hd_final_stream_gather(x.t, n, out=g.t)
    _ok(g)
    assert torch.equal(g.t, x.t[:, n - 1::n])


FWD_CASES = [
    # B, n, L, Hq, Hkv, D, mode, W, out dtype
    (1, 4, 300, 4, 2, 128, "intra", 0, BF),
    (2, 3, 77, 8, 2, 64, "cross", 50, F32),
    (1, 1, 513, 2, 1, 128, "intra", 129, F32),
    (2, 2, 200, 6, 3, 64, "intra", 0, BF),
    (1, 5, 61, 4, 4, 128, "cross", 0, F32),
]


@pytest.mark.parametrize("B,n,L,Hq,Hkv,D,mode,W,odt", FWD_CASES)
@pytest.mark.parametrize("in_dt", [BF, F32])
def test_attn_fwd_guarded(hd, B, n, L, Hq, Hkv, D, mode, W, odt, in_dt):
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 51).to(in_dt)
    k = synth.normal_device((B, P, Hkv, D), 52).to(in_dt)
    v = synth.normal_device((B, P, Hkv, D), 53).to(in_dt)
    o = Guarded((B, P, Hq, D), odt)
    lse = Guarded((B, Hq, P), F32)
    hd.hd_attn_fwd(q, k, v, n, mode, W, out=o.t, lse=lse.t)
    _ok(o, lse)
    # final-stream queries (KV-mirror layer)
    of = Guarded((B, L, Hq, D), odt)
    lf = Guarded((B, Hq, L), F32)
    hd.hd_attn_fwd_final_stream(q[:, n - 1::n].contiguous(), k, v, n, mode, W, out=of.t, lse=lf.t)
    _ok(of, lf)


@pytest.mark.parametrize("B,n,L,Hq,Hkv,D,mode,W,dt", [
    (1, 4, 300, 4, 2, 128, "intra", 0, BF), (2, 3, 77, 8, 2, 64, "cross", 50, BF), (1, 2, 130, 2, 1, 64, "cross", 0, F32)])
def test_attn_bwd_guarded(hd, B, n, L, Hq, Hkv, D, mode, W, dt):
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 61).to(dt)
    k = synth.normal_device((B, P, Hkv, D), 62).to(dt)
    v = synth.normal_device((B, P, Hkv, D), 63).to(dt)
    dO = synth.normal_device((B, P, Hq, D), 64).to(dt)
    o, lse = hd.hd_attn_fwd(q, k, v, n, mode, W, lse=True)
    dq, dk, dv = Guarded(q.shape, dt), Guarded(k.shape, dt), Guarded(v.shape, dt)
    ws = Guarded((hd.hd_attn_bwd_workspace(B, L, n, Hq, mode),), torch.uint8)
    hd.hd_attn_bwd(q, k, v, o, dO, lse, n, mode, W, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    _ok(dq, dk, dv)
    _ok(ws, written=False)
    # final-stream backward
    qf, of_, dOf = (t[:, n - 1::n].contiguous() for t in (q, o, dO))
    _, lf = hd.hd_attn_fwd_final_stream(qf, k, v, n, mode, W, lse=True)
    dqf, dk2, dv2 = Guarded(qf.shape, dt), Guarded(k.shape, dt), Guarded(v.shape, dt)
    ws2 = Guarded((hd.hd_attn_bwd_workspace(B, L, 1, Hq, "intra"),), torch.uint8)
    hd.hd_attn_bwd_final_stream(qf, k, v, of_, dOf, lf, n, mode, W, dq=dqf.t, dk=dk2.t, dv=dv2.t, workspace=ws2.t)
    _ok(dqf, dk2, dv2)
    _ok(ws2, written=False)


@pytest.mark.parametrize("mode,W,odt", [("intra", 0, BF), ("cross", 0, F32), ("cross", 300, BF), ("intra", 7, F32)])
@pytest.mark.parametrize("n,Hq,Hkv", [(4, 32, 8), (8, 64, 8), (2, 4, 4)])
def test_decode_guarded(hd, mode, W, odt, n, Hq, Hkv):
    B, Lmax, D = 3, 700, 128
    q = synth.normal_device((B, n, Hq, D), 71)
    kc = synth.normal_device((B, n, Lmax, Hkv, D), 72)
    vc = synth.normal_device((B, n, Lmax, Hkv, D), 73)
    ctx = torch.tensor([700, 1, 333], dtype=torch.int32, device="cuda")
    o = Guarded((B, n, Hq, D), odt)
    lse = Guarded((B, n, Hq), F32)
    ws = Guarded((hd.hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, mode),), torch.uint8)
    hd.hd_attn_decode(q, kc, vc, ctx, mode, W, out=o.t, lse=lse.t, workspace=ws.t)
    _ok(o, lse)
    _ok(ws, written=False)
    o2 = Guarded((B, n, Hq, D), odt)
    l2 = Guarded((B, n, Hq), F32)
    hd.hd_attn_decode_noalloc(q, kc, vc, ctx, mode, W, out=o2.t, lse=l2.t)
    _ok(o2, l2)
    assert torch.equal(o2.t, o.t) and torch.equal(l2.t, lse.t)


@pytest.mark.parametrize("D,rot,layout,dt", [(128, 128, "half", BF), (64, 32, "interleaved", F32), (128, 64, "half", F32)])
def test_rope_guarded(hd, D, rot, layout, dt):
    B, P, Hq, Hkv = 2, 333, 6, 2
    q = Guarded((B, P, Hq, D), dt, init=synth.normal_device((B, P, Hq, D), 81).to(dt))
    k = Guarded((B, P, Hkv, D), dt, init=synth.normal_device((B, P, Hkv, D), 82).to(dt))
    q0, k0 = q.t.clone(), k.t.clone()
    hd.hd_rope(q.t, k.t, rot_dim=rot, layout=layout)
    _ok(q, k)
    assert not torch.equal(q.t, q0) and not torch.equal(k.t, k0)
    # decode form: positions from ctx_len
    qd = Guarded((B, 4, Hq, D), dt, init=synth.normal_device((B, 4, Hq, D), 83).to(dt))
    pos0 = torch.tensor([5, 900], dtype=torch.int32, device="cuda")
    hd.hd_rope(qd.t, None, rot_dim=rot, layout=layout, pos_base=-4, pos_mult=4, pos0=pos0)
    _ok(qd)


@pytest.mark.parametrize("R,n", [(2, 4), (4, 4), (2, 2)])
def test_stream_parallel_calls_guarded(hd, R, n):
    B, L, Hq, Hkv, D = 2, 150, 8, 2, 128
    nl = n // R
    parts_k = synth.normal_device((R, B, nl * L, Hkv, D), 91)
    parts_v = synth.normal_device((R, B, nl * L, Hkv, D), 92)
    q_loc = synth.normal_device((B, nl * L, Hq, D), 93)
    # re-interleave
    k = Guarded((B, n * L, Hkv, D), BF)
    v = Guarded((B, n * L, Hkv, D), BF)
    hd.hd_stream_interleave(parts_k, n, out=k.t)
    hd.hd_stream_interleave(parts_v, n, out=v.t)
    _ok(k, v)
    for r in range(R):
        o = Guarded((B, nl * L, Hq, D), BF)
        lse = Guarded((B, Hq, nl * L), F32)
        hd.hd_attn_fwd_shard(q_loc, k.t, v.t, n, R, r, out=o.t, lse=lse.t)
        _ok(o, lse)
        o2 = Guarded((B, nl * L, Hq, D), F32)
        l2 = Guarded((B, Hq, nl * L), F32)
        hd.hd_attn_fwd_parts(q_loc, parts_k, parts_v, n, R, r, out=o2.t, lse=l2.t)
        _ok(o2, l2)
        # fused gather: every slot, the own one included, is a guarded copy target
        kd = [Guarded((B, nl * L, Hkv, D), BF) for _ in range(R)]
        vd = [Guarded((B, nl * L, Hkv, D), BF) for _ in range(R)]
        flags = Guarded((max(1, hd.hd_attn_peer_flags_bytes(B, L, n) // 8),), torch.int64)
        o3 = Guarded((B, nl * L, Hq, D), BF)
        hd.hd_attn_fwd_peer_gather(q_loc, list(parts_k), list(parts_v), [g.t for g in kd], [g.t for g in vd], n, R, r,
                                   flags=flags.t, out=o3.t)
        _ok(o3, *kd, *vd)
        _ok(flags, written=False)
        for i in range(R):
            assert torch.equal(kd[i].t, parts_k[i]) and torch.equal(vd[i].t, parts_v[i])
    # cross decode partials and both merges
    Lmax = 400
    qd = synth.normal_device((B, n, Hq, D), 94)
    kc = synth.normal_device((B, nl, Lmax, Hkv, D), 95)
    vc = synth.normal_device((B, nl, Lmax, Hkv, D), 96)
    ctx = torch.tensor([400, 17], dtype=torch.int32, device="cuda")
    op = Guarded((B, n, Hq, D), F32)
    lp = Guarded((B, n, Hq), F32)
    ws = Guarded((hd.hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, "cross"),), torch.uint8)
    hd.hd_attn_decode_shard(qd, kc, vc, ctx, R, 0, out=op.t, lse=lp.t, workspace=ws.t)
    _ok(op, lp)
    _ok(ws, written=False)
    o_all = torch.stack([op.t] * R)
    l_all = torch.stack([lp.t] * R)
    oc = Guarded((B, n, Hq, D), BF)
    lc = Guarded((B, n, Hq), F32)
    hd.hd_attn_combine(o_all, l_all, out=oc.t, lse=lc.t)
    _ok(oc, lc)
    os_ = Guarded((B, nl, Hq, D), BF)
    ls_ = Guarded((B, nl, Hq), F32)
    hd.hd_attn_combine_streams([op.t] * R, [lp.t] * R, n, R, R - 1, out=os_.t, lse=ls_.t)
    _ok(os_, ls_)
