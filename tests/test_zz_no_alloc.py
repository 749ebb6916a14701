"""hd_attn_decode_noalloc: decode with the library's own fixed scratch, for
callers that cannot give the library device memory.

Run last (file name) so a stop-at-first-failure run has covered everything
else first; it also passes alone in a fresh process.  The new entry point is
called through the C ABI twice in a row.  It runs the same kernels on the
same work plan as hd_attn_decode (caller-provided workspace), only with
another scratch address, so both results must be bit-identical; they are
also checked against the float64 oracle within the bf16 parity bound.  Sizes
needing more scratch than the fixed maximum are refused on the host.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from stream_sequence_attention_b200 import synth
from tests.gpu_util import TOL_BF16, lib, to_f64

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call_noalloc(hd, q, kc, vc, ctx, o, lse, mode, window=0):
    B, n, Hq, D = q.shape
    Lmax, Hkv = kc.shape[2], kc.shape[3]
    st = hd.new_status()
    code = hd.lib().hd_attn_decode_noalloc(
        _ptr(q), _ptr(kc), _ptr(vc), _ptr(ctx), _ptr(o), _ptr(lse), B, n, Lmax, Hq, Hkv, D,
        hd.HD_INTRA if mode == "intra" else hd.HD_CROSS, window, D ** -0.5, hd.HD_BF16, hd.HD_F32, _ptr(st),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return code, st


@pytest.mark.parametrize("mode,window", [("intra", 0), ("cross", 0), ("cross", 300)])
def test_noalloc_matches_workspace_decode_twice(mode, window):
    hd = lib()
    B, n, Lmax, Hq, Hkv, D = 4, 4, 1000, 32, 8, 128
    q = synth.normal_device((B, n, Hq, D), 501)
    kc = synth.normal_device((B, n, Lmax, Hkv, D), 502)
    vc = synth.normal_device((B, n, Lmax, Hkv, D), 503)
    ctx = torch.tensor([1000, 1, 517, 64], dtype=torch.int32, device="cuda")
    ref, ref_lse = hd.hd_attn_decode(q, kc, vc, ctx, mode, window, out_dtype=torch.float32, lse=True)
    oo, ol = oracle.decode(to_f64(q), to_f64(kc), to_f64(vc), ctx.cpu().numpy(), n, mode, window)
    for call in range(2):
        o = torch.full((B, n, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, n, Hq), float("nan"), dtype=torch.float32, device="cuda")
        code, st = _call_noalloc(hd, q, kc, vc, ctx, o, lse, mode, window)
        torch.cuda.synchronize()
        assert code == hd.HD_OK, hd.status_string(code)
        assert int(st.item()) == 0
        # same kernels, same plan, same summation order: bit-identical
        assert torch.equal(o, ref), call
        assert torch.equal(lse, ref_lse), call
        assert float(np.abs(to_f64(o) - oo).max()) <= TOL_BF16, call
        assert float(np.abs(to_f64(lse) - ol).max()) <= 1e-3, call


def test_noalloc_refuses_sizes_beyond_the_scratch():
    hd = lib()
    # batch 512, 8 streams, 64 query heads: the split partials need far more
    # than the fixed scratch, so the call is refused before any launch.
    B, n, Lmax, Hq, Hkv, D = 512, 8, 4096, 64, 8, 128
    need = hd.hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, "cross")
    assert need > (64 << 20)
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    code = hd.lib().hd_attn_decode_noalloc(fake, fake, fake, fake, fake, None, B, n, Lmax, Hq, Hkv, D,
                                           hd.HD_CROSS, 0, 0.1, hd.HD_BF16, hd.HD_BF16, None, None)
    assert code == hd.HD_ERR_UNSUPPORTED


def test_noalloc_after_other_work_on_the_device():
    """The scratch keeps the last call's contents; a later call with other
    sizes must not read stale partials."""
    hd = lib()
    D = 128
    for (B, n, Lmax, Hq, Hkv, ctxs) in [(2, 2, 300, 8, 2, [300, 7]), (3, 4, 129, 16, 4, [1, 129, 64])]:
        q = synth.normal_device((B, n, Hq, D), 600 + B)
        kc = synth.normal_device((B, n, Lmax, Hkv, D), 610 + B)
        vc = synth.normal_device((B, n, Lmax, Hkv, D), 620 + B)
        ctx = torch.tensor(ctxs, dtype=torch.int32, device="cuda")
        for mode in ("intra", "cross"):
            ref = hd.hd_attn_decode(q, kc, vc, ctx, mode, out_dtype=torch.float32)
            o = hd.hd_attn_decode_noalloc(q, kc, vc, ctx, mode, out_dtype=torch.float32)
            torch.cuda.synchronize()
            assert np.isfinite(o.cpu().numpy()).all()
            assert torch.equal(o, ref)
