"""GPU parity of hd_attn_fwd_final_stream (final-stream queries only, the
KV-mirror layers) against the float64 oracle, and against the final-stream
rows of the full hd_attn_fwd on the GPU."""

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


CASES = [
    # (dtype, B, n, L, Hq, Hkv, D, mode, W)
    ("bf16", 2, 4, 300, 4, 2, 128, "cross", 0),    # ragged, queries at stride n
    ("bf16", 2, 4, 300, 4, 2, 128, "intra", 0),
    ("bf16", 1, 3, 257, 4, 1, 128, "cross", 200),  # window in physical positions
    ("bf16", 1, 2, 200, 2, 2, 128, "intra", 50),
    ("bf16", 1, 4, 130, 8, 2, 64, "cross", 0),     # head_dim 64
    ("bf16", 1, 1, 140, 2, 2, 128, "cross", 0),    # n = 1: plain causal
    ("bf16", 2, 4, 1, 2, 1, 128, "cross", 0),      # one token
    ("f32", 1, 4, 70, 2, 1, 64, "cross", 0),
    ("f32", 2, 3, 45, 4, 2, 128, "intra", 9),
]


@pytest.mark.parametrize("dtype,B,n,L,Hq,Hkv,D,mode,W", CASES)
def test_final_stream_matches_oracle(hd, dtype, B, n, L, Hq, Hkv, D, mode, W):
    P = n * L
    q, k, v = host_qkv(B, P, Hq, Hkv, D, 700 + L + W, dtype)
    qf = np.ascontiguousarray(q[:, n - 1::n])
    st = hd.new_status()
    o, lse = hd.hd_attn_fwd_final_stream(dev(qf, dtype), dev(k, dtype), dev(v, dtype), n, mode, W,
                                         out_dtype=torch.float32, lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.attn_final_stream(qf, k, v, n, mode, W)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert max_abs(to_f64(o), ro) <= tol
    assert max_abs(to_f64(lse), rl) <= (TOL_F32 if dtype == "f32" else 1e-3)


@pytest.mark.parametrize("mode", ["intra", "cross"])
def test_final_stream_equals_full_call_rows_on_gpu(hd, mode):
    B, n, L, Hq, Hkv, D = 2, 4, 512, 8, 2, 128
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 801)
    k = synth.normal_device((B, P, Hkv, D), 802)
    v = synth.normal_device((B, P, Hkv, D), 803)
    full = hd.hd_attn_fwd(q, k, v, n, mode, out_dtype=torch.float32)
    fin = hd.hd_attn_fwd_final_stream(q[:, n - 1::n].contiguous(), k, v, n, mode, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert float((full[:, n - 1::n] - fin).abs().max()) <= 1e-2


def test_final_stream_full_size_sampled(hd):
    """KV-mirror layer at the bench's size: n=4, L=4096, batch 2, 32/8 heads, cross mode."""
    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * L
    qf = synth.normal_device((B, L, Hq, D), 811)
    k = synth.normal_device((B, P, Hkv, D), 812)
    v = synth.normal_device((B, P, Hkv, D), 813)
    o = hd.hd_attn_fwd_final_stream(qf, k, v, n, "cross")
    torch.cuda.synchronize()
    G = Hq // Hkv
    worst = 0.0
    for b, h in [(0, 0), (1, 31)]:
        kv = h // G
        kh = to_f64(k[b:b + 1, :, kv:kv + 1])
        vh = to_f64(v[b:b + 1, :, kv:kv + 1])
        rows = [0, 1, 127, 128, 2047, L - 1]
        qrows = {i * n + n - 1: to_f64(qf[b, i, h]) for i in rows}
        ref, _ = oracle.attn_rows(_QRows(qrows, (1, P, 1, D)), kh, vh, n, "cross",
                                  [(0, 0, i * n + n - 1) for i in rows])
        got = np.stack([to_f64(o[b, i, h]) for i in rows])
        worst = max(worst, max_abs(got, ref))
    assert worst <= TOL_BF16


class _QRows:
    """Stands in for q[b, p, h, :] with a few prefetched rows (one head)."""

    def __init__(self, rows, shape):
        self.rows = rows
        self.shape = shape

    def __getitem__(self, idx):
        return self.rows[idx[1]]
