"""hd_attn_fwd_rope: attention with the rotary embedding fused in (query rows
rotated inside the attention kernel, k rotated in place), against the
float64 oracle's attn(rope(q), rope(k), v), and against the separate chain
hd_rope + hd_attn_fwd (k bit-identical; the query rows' cos/sin come from the
special-function unit inside the attention kernel, so O agrees with the
chain to the bf16 bound rather than bit for bit)."""

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, dev, host_qkv, lib, max_abs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hd():
    return lib()


CASES = [
    # B, n, L, Hq, Hkv, D, mode, W, rot, layout, base
    (2, 4, 300, 4, 2, 128, "intra", 0, 128, "half", 10000.0),
    (1, 4, 300, 4, 2, 128, "cross", 0, 128, "half", 10000.0),
    (1, 3, 257, 6, 2, 128, "intra", 100, 64, "half", 500000.0),      # partial rotary, window
    (1, 2, 300, 2, 2, 128, "cross", 200, 128, "interleaved", 1e6),   # window in positions
    (2, 1, 384, 2, 2, 128, "intra", 0, 128, "half", 10000.0),         # n = 1
    (1, 4, 200, 8, 2, 64, "intra", 0, 64, "interleaved", 10000.0),    # head_dim 64
    (1, 4, 100, 8, 8, 64, "cross", 50, 32, "half", 10000.0),
    (1, 3, 1, 2, 1, 128, "intra", 0, 40, "interleaved", 10000.0),     # one token, rot % 16 != 0
]


@pytest.mark.parametrize("B,n,L,Hq,Hkv,D,mode,W,rot,layout,base", CASES)
@pytest.mark.parametrize("out_f32", [False, True])
def test_fused_rope_attention(hd, B, n, L, Hq, Hkv, D, mode, W, rot, layout, base, out_f32):
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 300 + L + rot, "bf16")
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    q_before = qd.clone()
    odt = torch.float32 if out_f32 else None
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd_rope(qd, kd, vd, n, mode, W, rot_dim=rot, base=base, layout=layout, out_dtype=odt,
                                 lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(qd, q_before), "q must be left as given"
    kw = dict(layout=layout)
    qr, kr = oracle.rope(q, rot, base, **kw), oracle.rope(k, rot, base, **kw)
    err_k = np.abs(to_f64(kd) - kr)
    assert np.all(err_k <= 2.0 ** -8 * np.abs(kr) + 1e-5), "k is not rope(k)"
    ro, _ = oracle.attn(qr, kr, v, n, mode, W)
    assert max_abs(to_f64(o), ro) <= TOL_BF16
    # The kernel attends over rope(q), rope(k) rounded to bf16 (the rotated
    # rows are bf16 tiles); lse is checked against the oracle on those inputs,
    # where the rounding moves scores by up to 2^-8 of their size.
    _, rl = oracle.attn(synth.bf16_round(qr.astype(np.float32)), synth.bf16_round(kr.astype(np.float32)), v, n, mode, W)
    assert max_abs(to_f64(lse), rl) <= 1e-3
    # the separate chain: hd_rope on copies, then hd_attn_fwd
    q2, k2 = dev(q, "bf16"), dev(k, "bf16")
    hd.hd_rope(q2, k2, rot, base, layout=layout)
    o2, l2 = hd.hd_attn_fwd(q2, k2, vd, n, mode, W, out_dtype=odt, lse=True)
    torch.cuda.synchronize()
    assert torch.equal(k2, kd)
    assert float((o2.float() - o.float()).abs().max()) <= TOL_BF16
    assert float((l2 - lse).abs().max()) <= 1e-3


def test_fused_rope_full_size_sampled(hd):
    """The intra prefill workload (n=4 L=4096 B=2 32q/8kv D=128): k equal to
    the separate chain's bit for bit, O within the bf16 bound of it, and
    sampled rows against the oracle."""
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 321)
    k = synth.normal_device((B, P, Hkv, D), 322)
    v = synth.normal_device((B, P, Hkv, D), 323)
    k0 = k.clone()
    o = hd.hd_attn_fwd_rope(q, k, v, n, "intra")
    q2, k2 = q.clone(), k0.clone()
    hd.hd_rope(q2, k2)
    o2 = hd.hd_attn_fwd(q2, k2, v, n, "intra")
    torch.cuda.synchronize()
    assert torch.equal(k, k2)
    assert float((o.float() - o2.float()).abs().max()) <= TOL_BF16
    # sampled rows of stream 1, head 5, against the oracle on the de-interleaved stream
    s, h = 1, 5
    g = h // (Hq // Hkv)
    qs = oracle.rope(to_f64(q[0:1]), D)[:, s::n, h:h + 1]
    ks = oracle.rope(to_f64(k0[0:1]), D)[:, s::n, g:g + 1]
    vs = to_f64(v[0:1, s::n, g:g + 1])
    for i in (0, 1, 127, 128, 2049, 4095):
        ref, _ = oracle.attn(qs[:, :i + 1], ks[:, :i + 1], vs[:, :i + 1], 1, "intra")
        assert max_abs(to_f64(o[0:1, i * n + s, h]), ref[:, i, 0]) <= TOL_BF16
