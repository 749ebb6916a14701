"""GPU parity of ``hd_rope`` against the float64 oracle: both pairings,
partial rotary, head dims 8 to 256, q only, per-sequence decode offsets,
positions near 2^30 (where a float32 angle would be far off), and the full
prefill workload on sampled rows.

Bound: one rounding of the rotated value to the output type plus the float32
rotation: bf16 |err| <= 2^-8 |ref| + 1e-5; float32 |err| <= 1e-5."""

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import dev, lib, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hd():
    return lib()


def _check(got, ref, dtype):
    err = np.abs(got - ref)
    bound = (2.0 ** -8 * np.abs(ref) + 1e-5) if dtype == "bf16" else np.full_like(ref, 1e-5)
    assert np.all(err <= bound), float(np.max(err - bound))


CASES = [
    # dtype, layout, B, P, Hq, Hkv, D, rot, base, pos_base, pos_mult, pos0
    ("bf16", "half", 2, 4 * 300, 32, 8, 128, 128, 10000.0, 0, 0, None),
    ("f32", "interleaved", 1, 3 * 50, 4, 2, 64, 64, 500000.0, 0, 0, None),
    ("bf16", "half", 2, 4, 8, 2, 128, 64, 10000.0, -4, 4, [7, 1000]),
    ("f32", "half", 1, 37, 3, 0, 80, 80, 10000.0, 12345, 0, None),
    ("bf16", "interleaved", 1, 100, 2, 2, 256, 128, 1e6, 2 ** 30, 0, None),
    ("f32", "half", 3, 10, 2, 2, 8, 8, 10.0, 5, 2, [0, 1, 2 ** 20]),
]


@pytest.mark.parametrize("dtype,layout,B,P,Hq,Hkv,D,rot,base,pos_base,pos_mult,pos0", CASES)
def test_rope_matches_oracle(hd, dtype, layout, B, P, Hq, Hkv, D, rot, base, pos_base, pos_mult, pos0):
    q = synth.normal((B, P, Hq, D), 900 + D, dtype=dtype)
    k = synth.normal((B, P, Hkv, D), 901 + D, dtype=dtype) if Hkv else None
    qd = dev(q, dtype)
    kd = dev(k, dtype) if k is not None else None
    p0 = None if pos0 is None else torch.tensor(pos0, dtype=torch.int32, device="cuda")
    hd.hd_rope(qd, kd, rot, base, pos_base, pos_mult, p0, layout)
    torch.cuda.synchronize()
    kw = dict(layout=layout, pos_base=pos_base, pos_mult=pos_mult, pos0=pos0)
    _check(to_f64(qd), oracle.rope(q, rot, base, **kw), dtype)
    if k is not None:
        _check(to_f64(kd), oracle.rope(k, rot, base, **kw), dtype)


def test_rope_full_size_sampled(hd):
    """q [2, 16384, 32, 128], k [2, 16384, 8, 128] bf16 at positions p = i*n + s."""
    B, P, Hq, Hkv, D = 2, 16384, 32, 128 // 16, 128
    q = synth.normal_device((B, P, Hq, D), 911)
    k = synth.normal_device((B, P, Hkv, D), 912)
    q0, k0 = q.clone(), k.clone()
    hd.hd_rope(q, k)
    torch.cuda.synchronize()
    for b, p in [(0, 0), (0, 1), (1, 4095), (0, 8191), (1, 16383)]:
        for x, x0 in ((q, q0), (k, k0)):
            ref = oracle.rope(to_f64(x0[b:b + 1, p:p + 1]), D, 10000.0, pos_base=p)
            _check(to_f64(x[b:b + 1, p:p + 1]), ref, "bf16")
