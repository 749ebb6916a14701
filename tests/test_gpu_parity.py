"""GPU parity: every C-ABI call against the float64 oracle on seeded inputs,
at sizes the oracle finishes in seconds that still span several tiles and a
ragged tail, plus the edge cases (n = 1, windows of 1 and >= L, out-of-range
token ids, a sequence of one token, masked-key perturbation)."""

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


# ------------------------------------------------------- expand / gather

@pytest.mark.parametrize("dtype,n,B,L,V,d", [
    ("f32", 2, 1, 64, 512, 128),      # tiny fp32 config
    ("bf16", 4, 2, 37, 1000, 4096),   # ragged, wide rows
    ("bf16", 3, 3, 5, 7, 8),          # one 16-byte vector per row
    ("f32", 1, 2, 9, 11, 12),
])
def test_expand_bit_exact(hd, dtype, n, B, L, V, d):
    tables = synth.normal((n, V, d), 31, std=0.02, dtype=dtype)
    ids = synth.ids_uniform(B, L, V, 32)
    st = hd.new_status()
    out = hd.hd_expand_embed(dev(tables, dtype), dev(ids, "i32"), dev_status=st)
    torch.cuda.synchronize()
    ref = oracle.expand(tables, ids)
    got = out.float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.astype(np.float32).view(np.uint32))
    assert int(st.item()) == 0


def test_expand_ids_at_a_four_byte_offset(hd):
    """ids need only int32 alignment: a view starting one token in (ids[:, 1:]
    of one sequence) is accepted and expands bit-exactly."""
    n, V, d = 3, 50, 64
    tables = synth.normal((n, V, d), 35, std=0.02, dtype="bf16")
    ids = synth.ids_uniform(1, 41, V, 36)
    ids_d = dev(ids, "i32")[:, 1:]
    assert ids_d.is_contiguous() and ids_d.data_ptr() % 16 == 4
    st = hd.new_status()
    out = hd.hd_expand_embed(dev(tables, "bf16"), ids_d, dev_status=st)
    torch.cuda.synchronize()
    ref = oracle.expand(tables, ids[:, 1:])
    assert np.array_equal(out.float().cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32))
    assert int(st.item()) == 0


def test_expand_bad_token_zero_row_and_status(hd):
    n, V, d = 2, 16, 64
    tables = synth.normal((n, V, d), 33, std=0.02, dtype="bf16")
    ids = np.array([[3, 16, 5, -1, 15]], dtype=np.int32)
    st = hd.new_status()
    out = hd.hd_expand_embed(dev(tables, "bf16"), dev(ids, "i32"), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == hd.HD_ERR_BAD_TOKEN
    got = out.float().cpu().numpy()
    for i, t in enumerate(ids[0]):
        for s in range(n):
            row = got[0, i * n + s]
            if 0 <= t < V:
                assert np.array_equal(row, tables[s, t])
            else:
                assert not row.any()


@pytest.mark.parametrize("dtype,n,B,L,d", [("f32", 2, 1, 64, 128), ("bf16", 4, 2, 33, 4096), ("bf16", 1, 1, 3, 8)])
def test_gather_bit_exact(hd, dtype, n, B, L, d):
    h = synth.normal((B, n * L, d), 34, dtype=dtype)
    out = hd.hd_final_stream_gather(dev(h, dtype), n)
    torch.cuda.synchronize()
    ref = oracle.final_stream_gather(h, n)
    assert np.array_equal(out.float().cpu().numpy().view(np.uint32), ref.astype(np.float32).view(np.uint32))


def test_tiny_fp32_config_chain(hd):
    """The tiny fp32 workload: expand, intra and cross attention, gather."""
    n, L, B, V, dm, H, D = 2, 64, 1, 512, 128, 2, 64
    tables = synth.normal((n, V, dm), 40, std=0.02)
    ids = synth.ids_uniform(B, L, V, 41)
    x = hd.hd_expand_embed(dev(tables, "f32"), dev(ids, "i32"))
    q, k, v = host_qkv(B, n * L, H, H, D, 42, "f32")
    qd, kd, vd = dev(q, "f32"), dev(k, "f32"), dev(v, "f32")
    for mode in ("intra", "cross"):
        o, lse = hd.hd_attn_fwd(qd, kd, vd, n, mode, 0, 1 / 8, lse=True)
        torch.cuda.synchronize()
        ro, rl = oracle.attn(q, k, v, n, mode, 0, 1 / 8)
        assert max_abs(to_f64(o), ro) <= TOL_F32, mode
        assert max_abs(to_f64(lse), rl) <= TOL_F32, mode
    g = hd.hd_final_stream_gather(x, n)
    torch.cuda.synchronize()
    assert np.array_equal(g.cpu().numpy(), oracle.final_stream_gather(oracle.expand(tables, ids), n))


# ---------------------------------------------------------- attention

ATTN_CASES = [
    # (dtype, B, n, L, Hq, Hkv, D, mode, W)
    ("f32", 1, 3, 50, 2, 1, 64, "intra", 0),
    ("f32", 2, 2, 41, 4, 2, 128, "cross", 0),
    ("f32", 1, 4, 30, 2, 2, 64, "intra", 7),
    ("f32", 1, 2, 40, 2, 1, 64, "cross", 9),
    ("bf16", 2, 3, 300, 4, 2, 128, "intra", 0),    # 3 query blocks, ragged
    ("bf16", 2, 3, 300, 4, 2, 128, "cross", 0),    # 8 query blocks, ragged
    ("bf16", 1, 4, 257, 4, 1, 128, "intra", 100),  # window inside the tile grid
    ("bf16", 1, 2, 300, 2, 2, 128, "cross", 200),  # window in physical positions
    ("bf16", 1, 2, 200, 2, 1, 128, "intra", 1),    # window of one key: O = v_self
    ("bf16", 1, 2, 130, 2, 2, 128, "intra", 1000), # window wider than the stream
    ("bf16", 2, 1, 384, 2, 2, 128, "intra", 0),    # n = 1: plain causal
    ("bf16", 1, 4, 200, 8, 2, 64, "intra", 0),     # head_dim 64
    ("bf16", 1, 4, 100, 8, 8, 64, "cross", 50),
    ("bf16", 1, 3, 1, 2, 1, 128, "intra", 0),      # one token
]


@pytest.mark.parametrize("dtype,B,n,L,Hq,Hkv,D,mode,W", ATTN_CASES)
@pytest.mark.parametrize("out_f32", [False, True])
def test_attn_fwd_matches_oracle(hd, dtype, B, n, L, Hq, Hkv, D, mode, W, out_f32):
    """Every case with float32 and bf16 output.  bf16 output is held to the
    bf16 bound whatever the input type (its rounding alone is up to 2^-9 of
    |O|)."""
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 50 + L + W, dtype)
    scale = D ** -0.5
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(dev(q, dtype), dev(k, dtype), dev(v, dtype), n, mode, W, scale,
                            out_dtype=torch.float32 if out_f32 else None, lse=True, dev_status=st)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, n, mode, W, scale)
    tol = TOL_F32 if (dtype == "f32" and out_f32) else TOL_BF16
    err = max_abs(to_f64(o), ro)
    assert err <= tol, f"max-abs {err}"
    assert max_abs(to_f64(lse), rl) <= (TOL_F32 if dtype == "f32" else 1e-3)
    assert int(st.item()) == 0


@pytest.mark.parametrize("mode,W,n", [("intra", 0, 4), ("cross", 0, 4), ("intra", 150, 2), ("cross", 300, 2),
                                      ("intra", 0, 1)])
@pytest.mark.parametrize("out_f32", [False, True])
def test_running_max_jumps(hd, mode, W, n, out_f32):
    """Keys whose scores grow tile after tile, so a row's maximum rises by far
    more than 2^8 (the kernel's rescale threshold, in log2 units) several
    times within a unit: the rows that jump redo their exponentials against
    the new maximum and rescale O.  Some rows see their first key tile fully
    masked (windows), so their maximum starts at -inf."""
    B, L, Hq, Hkv, D = 1, 700, 4, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 77, "bf16")
    q = synth.bf16_round(np.abs(q).astype(np.float32) * np.float32(0.5))
    # key j's features grow with its position: scores rise ~linearly along the
    # sequence, a tile of 128 keys later by ~10 log2 units or more
    grow = (1.0 + np.arange(P, dtype=np.float32) / 40.0)[None, :, None, None]
    k = synth.bf16_round(np.abs(k).astype(np.float32) * grow * np.float32(0.25))
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), n, mode, W,
                            out_dtype=torch.float32 if out_f32 else None, lse=True, dev_status=st)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, n, mode, W)
    assert np.isfinite(to_f64(o)).all()
    assert max_abs(to_f64(o), ro) <= TOL_BF16
    assert max_abs(to_f64(lse), rl) <= 1e-3 * max(1.0, float(np.abs(rl).max()))
    assert int(st.item()) == 0


@pytest.mark.parametrize("mode,W", [("intra", 0), ("cross", 0), ("cross", 100)])
def test_scores_beyond_the_exponent_range(hd, mode, W):
    """Scores spread so widely within a row (queries scaled by 40: a score
    spread of ~60 log2 units, hundreds between a row's extremes) that many
    exponents fall below -126: there the FMA-pipe exponential of the
    unmasked tiles clamps to ~2^-126 where MUFU gives 0, both negligible
    next to the row sum (>= 1).  O and lse still match the oracle and stay
    finite."""
    B, n, L, Hq, Hkv, D = 1, 2, 400, 4, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 91, "bf16")
    q = synth.bf16_round(q.astype(np.float32) * np.float32(40.0))
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), n, mode, W, lse=True, dev_status=st)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, n, mode, W)
    assert int(st.item()) == 0
    assert np.isfinite(to_f64(o)).all() and np.isfinite(to_f64(lse)).all()
    assert max_abs(to_f64(o), ro) <= TOL_BF16
    assert max_abs(to_f64(lse), rl) <= 1e-3 * max(1.0, float(np.abs(rl).max()))


@pytest.mark.parametrize("dtype,mode,W", [("bf16", "intra", 0), ("bf16", "cross", 0), ("bf16", "intra", 60),
                                          ("bf16", "cross", 90), ("f32", "intra", 0), ("f32", "cross", 33)])
def test_masked_keys_do_not_change_output_bits(hd, dtype, mode, W):
    """Perturbing every key/value that is invisible to a query row leaves that
    row bit-identical: masked-out cross-stream keys get exactly zero weight."""
    B, n, L, Hq, Hkv, D = 1, 4, 160, 2, 1, 128 if dtype == "bf16" else 64
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 60, dtype)
    o1 = hd.hd_attn_fwd(dev(q, dtype), dev(k, dtype), dev(v, dtype), n, mode, W)
    g = synth.rng(61)
    pk = np.arange(P)
    for p in (0, 3, P // 2 + 1, P - 1):
        hidden = ~oracle.visible(p, pk, n, mode, W)
        k2, v2 = k.copy(), v.copy()
        k2[:, hidden] = g.standard_normal(k2[:, hidden].shape).astype(np.float32) * 8
        v2[:, hidden] = g.standard_normal(v2[:, hidden].shape).astype(np.float32) * 8
        if dtype == "bf16":
            k2, v2 = synth.bf16_round(k2), synth.bf16_round(v2)
        o2 = hd.hd_attn_fwd(dev(q, dtype), dev(k2, dtype), dev(v2, dtype), n, mode, W)
        torch.cuda.synchronize()
        assert torch.equal(o1[:, p], o2[:, p]), p


def test_attn_dev_status_stays_clear(hd):
    B, n, L, H, D = 1, 2, 130, 2, 128
    q, k, v = host_qkv(B, n * L, H, H, D, 70, "bf16")
    st = hd.new_status()
    hd.hd_attn_fwd(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), n, "cross", dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


# -------------------------------------------------------------- decode

def _cache_case(B, n, Lmax, Hq, Hkv, D, seed):
    q = synth.normal((B, n, Hq, D), seed, dtype="bf16")
    kc = synth.normal((B, n, Lmax, Hkv, D), seed + 1, dtype="bf16")
    vc = synth.normal((B, n, Lmax, Hkv, D), seed + 2, dtype="bf16")
    return q, kc, vc


DECODE_CASES = [
    # (B, n, Lmax, Hq, Hkv, ctx, mode, W)
    (3, 4, 300, 16, 2, [300, 1, 77], "intra", 0),
    (3, 4, 300, 16, 2, [300, 1, 77], "cross", 0),
    (2, 4, 513, 64, 8, [513, 200], "cross", 0),     # 32 query rows per KV head
    (2, 2, 200, 8, 2, [200, 65], "intra", 50),
    (2, 3, 200, 6, 3, [199, 64], "cross", 70),
    (1, 1, 129, 4, 4, [129], "intra", 0),
    (2, 8, 100, 16, 2, [100, 3], "cross", 0),        # 64 query rows: two row groups
    # tensor-core cross decode (n*G <= 32 rows): many splits of one KV head,
    # a window across split boundaries, one stream with 32 heads per group
    (1, 4, 5000, 8, 1, [4999], "cross", 0),
    (1, 2, 3000, 32, 2, [2999], "cross", 1000),
    (2, 1, 700, 32, 1, [700, 333], "cross", 0),
    (2, 4, 70, 8, 1, [70, 5], "cross", 0),             # cache shorter than one 128-token box
]


@pytest.mark.parametrize("B,n,Lmax,Hq,Hkv,ctx,mode,W", DECODE_CASES)
def test_decode_matches_oracle(hd, B, n, Lmax, Hq, Hkv, ctx, mode, W):
    D = 128
    q, kc, vc = _cache_case(B, n, Lmax, Hq, Hkv, D, 80 + Lmax)
    ctx = np.array(ctx, dtype=np.int32)
    st = hd.new_status()
    o, lse = hd.hd_attn_decode(dev(q, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"), mode, W,
                               out_dtype=torch.float32, lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.decode(q, kc, vc, ctx, n, mode, W)
    assert max_abs(to_f64(o), ro) <= TOL_BF16
    assert max_abs(to_f64(lse), rl) <= 1e-3


def test_decode_bf16_output_and_two_calls(hd):
    B, n, Lmax, Hq, Hkv, D = 2, 4, 260, 32, 8, 128
    q, kc, vc = _cache_case(B, n, Lmax, Hq, Hkv, D, 90)
    ctx = np.array([260, 129], dtype=np.int32)
    args = (dev(q, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"))
    for mode in ("intra", "cross"):
        o1 = hd.hd_attn_decode(*args, mode)
        o2 = hd.hd_attn_decode(*args, mode)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2)
        ro, _ = oracle.decode(q, kc, vc, ctx, n, mode)
        assert max_abs(to_f64(o1), ro) <= TOL_BF16


def test_decode_equals_prefill_rows_on_gpu(hd):
    """Decode of the last token equals the prefill rows of that token."""
    B, n, L, Hq, Hkv, D = 1, 4, 150, 8, 2, 128
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 95, "bf16")
    kc = np.ascontiguousarray(k.reshape(B, L, n, Hkv, D).transpose(0, 2, 1, 3, 4))
    vc = np.ascontiguousarray(v.reshape(B, L, n, Hkv, D).transpose(0, 2, 1, 3, 4))
    qd = np.ascontiguousarray(q.reshape(B, L, n, Hq, D)[:, L - 1])
    ctx = np.array([L], dtype=np.int32)
    for mode in ("intra", "cross"):
        pre = hd.hd_attn_fwd(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), n, mode, out_dtype=torch.float32)
        dec = hd.hd_attn_decode(dev(qd, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"), mode,
                                out_dtype=torch.float32)
        torch.cuda.synchronize()
        last = pre.view(B, L, n, Hq, D)[:, L - 1]
        assert float((last - dec).abs().max()) <= 2 * TOL_BF16 / 4


def test_decode_bad_ctx_len_reports_and_zeros(hd):
    B, n, Lmax, Hq, Hkv, D = 2, 2, 64, 4, 2, 128
    q, kc, vc = _cache_case(B, n, Lmax, Hq, Hkv, D, 99)
    ctx = np.array([0, 65], dtype=np.int32)
    st = hd.new_status()
    o = hd.hd_attn_decode(dev(q, "bf16"), dev(kc, "bf16"), dev(vc, "bf16"), dev(ctx, "i32"), "intra",
                          dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == hd.HD_ERR_INVALID_ARG
    assert not o.float().abs().sum().item()


def test_same_buffers_under_different_shapes(hd):
    """The tensor maps are cached by (pointer, shape): one allocation viewed
    with two different geometries gives the right result for both."""
    buf_q = torch.empty(2 * 4 * 160 * 4 * 128, dtype=torch.bfloat16, device="cuda")
    buf_k = torch.empty(2 * 4 * 160 * 2 * 128, dtype=torch.bfloat16, device="cuda")
    buf_v = torch.empty_like(buf_k)
    for (B, n, L, Hq, Hkv, seed) in [(2, 4, 160, 4, 2, 61), (1, 2, 320, 8, 4, 62), (2, 4, 160, 4, 2, 63)]:
        P = n * L
        q, k, v = host_qkv(B, P, Hq, Hkv, 128, seed, "bf16")
        qd = buf_q.view(B, P, Hq, 128)
        kd = buf_k.view(B, P, Hkv, 128)
        vd = buf_v.view(B, P, Hkv, 128)
        qd.copy_(dev(q, "bf16"))
        kd.copy_(dev(k, "bf16"))
        vd.copy_(dev(v, "bf16"))
        o = hd.hd_attn_fwd(qd, kd, vd, n, "cross", out_dtype=torch.float32)
        torch.cuda.synchronize()
        ro, _ = oracle.attn(q, k, v, n, "cross")
        assert max_abs(to_f64(o), ro) <= TOL_BF16
