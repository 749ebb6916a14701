"""The diagnostics (clock-counter builds and probes) stay usable: their
modules import without a GPU, their probe sources are not part of libhd.so,
and the probes cross-compile for sm_100a against the kernels' shared header
(no GPU needed to compile)."""

import importlib
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "stream_sequence_attention_b200")
PROBES = ["softmax_probe.cu", "mma_probe.cu"]


@pytest.mark.parametrize("mod", ["diag_trace", "diag_softmax", "diag_mma", "diag_ab"])
def test_diag_modules_import(mod):
    m = importlib.import_module(f"stream_sequence_attention_b200.{mod}")
    assert callable(m.main)


def test_probe_sources_stay_out_of_the_library():
    from stream_sequence_attention_b200 import build

    srcs = [os.path.basename(s) for s in build.sources()]
    for p in PROBES:
        assert os.path.exists(os.path.join(PKG, "diag", p))
        assert p not in srcs


@pytest.mark.parametrize("probe", PROBES)
def test_probe_compiles(probe, tmp_path):
    from stream_sequence_attention_b200 import build

    out = str(tmp_path / (probe + ".o"))
    cmd = [build._nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-c",
           "-I", os.path.join(PKG, "csrc"), "-I", os.path.join(ROOT, "include"), "-o", out,
           os.path.join(PKG, "diag", probe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
