"""The FMA-pipe exponential of the attention kernels (exp2_fma, an optional
replacement for part of the MUFU exponentials, and its packed f32x2 form
exp2_fma2) against the MUFU form and float64 2**x, over its whole input
range: no NaN or negative result, exact zero below 2^-126 (as the
flush-to-zero MUFU form gives, -inf included; the packed form clamps there
to ~2^-126), relative error below 1e-4 elsewhere; and exp2_sat2 behind the
saturating shift, on exponents up to 8.  A small probe library is compiled
from tests/probes/exp2_fma_probe.cu against the kernels' shared header."""

import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def probe():
    from stream_sequence_attention_b200 import build as hd_build

    out = os.path.join(tempfile.mkdtemp(prefix="hd_probe_"), "exp2_probe.so")
    cmd = [hd_build._nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "stream_sequence_attention_b200", "csrc"),
           "-I", os.path.join(ROOT, "include"), "-o", out, os.path.join(ROOT, "tests", "probes", "exp2_fma_probe.cu")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return ctypes.CDLL(out)


def test_exp2_fma_whole_range(probe):
    special = [-np.inf, -1e30, -1000.0, -200.0, -127.5, -127.0, -126.6, -126.5, -126.0001, -126.0, -125.9,
               -125.5, -125.0, -100.0, -64.3, -10.0, -1.0, -0.5, -1e-7, 0.0, 1e-7, 0.5, 0.49999997, 1.0, 10.0,
               100.0, 127.0]
    sweep = np.linspace(-140.0, 20.0, 200001)
    x = np.concatenate([np.array(special), sweep]).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    fo = torch.empty_like(xt)
    mo = torch.empty_like(xt)
    po = torch.empty_like(xt)
    so = torch.empty_like(xt)
    rc = probe.exp2_probe(ctypes.c_void_p(xt.data_ptr()), ctypes.c_void_p(fo.data_ptr()),
                          ctypes.c_void_p(mo.data_ptr()), ctypes.c_void_p(po.data_ptr()),
                          ctypes.c_void_p(so.data_ptr()), len(x))
    assert rc == 0
    f = fo.cpu().numpy().astype(np.float64)
    m = mo.cpu().numpy().astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    assert np.isfinite(f).all(), x[~np.isfinite(f)][:8]
    assert (np.signbit(fo.cpu().numpy()) == 0).all()
    below = x < -126.0
    assert (f[below] == 0.0).all()
    assert (m[below] == 0.0).all()  # the MUFU form flushes there too
    normal = x >= -125.0
    rel = np.abs(f[normal] - exact[normal]) / exact[normal]
    assert rel.max() < 1e-4, float(rel.max())
    assert (np.abs(f[normal] - m[normal]) / exact[normal]).max() < 1.2e-4
    edge = (x >= -126.0) & (x < -125.0)  # results near 2^-126: absolute bound
    assert (np.abs(f[edge] - exact[edge]) <= 2.0 ** -136).all()
    # the packed form: the same values for x >= -126 (where the attention
    # kernel uses it: exponents of unmasked tiles), clamped to ~2^-126 below
    pr = po.cpu().numpy().astype(np.float64)
    assert np.isfinite(pr).all() and (pr >= 0).all()
    ok = x >= -126.0
    assert np.array_equal(pr[ok], f[ok])
    assert (pr[~ok] <= 2.0 ** -125).all()
    # the saturating form, on exponents x <= 8 (the attention kernel's:
    # up to its rescale threshold): the shift through y = sat((x + 126) / 134)
    # costs about 134 * 2^-25 in x; x below -126 lands on ~2^-126
    sr = so.cpu().numpy().astype(np.float64)
    inr = x <= 8.0
    assert np.isfinite(sr[inr]).all() and (sr[inr] >= 0).all()
    sn = inr & (x >= -125.0)
    rel = np.abs(sr[sn] - exact[sn]) / exact[sn]
    assert rel.max() < 1e-4, (float(rel.max()), float(x[sn][np.argmax(rel)]))
    assert (sr[inr & (x < -125.0)] <= 2.0 ** -124).all()
