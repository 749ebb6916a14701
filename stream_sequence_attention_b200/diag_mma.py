"""Diagnostic: cycles per tcgen05.mma step for the attention kernels' issue
patterns (continuous, bursts with commits, the forward's two-head order,
and that order with a wait on every commit).

Compiles ``diag/mma_probe.cu`` (against the kernels' shared header, not part
of libhd.so) and prints the cycles per MMA averaged over one CTA per SM.

    python -m stream_sequence_attention_b200.diag_mma
"""

import ctypes
import os
import subprocess
import tempfile

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
NAMES = ["128 SS MMAs, one commit", "16 x [8 SS; commit]", "16 x [8 TS; commit]",
         "forward order, two heads: [8 TS; 8 SS; commit] x 2 per tile", "the same, waiting on each commit"]


def main():
    import torch

    from stream_sequence_attention_b200 import build as hd_build

    out = os.path.join(tempfile.mkdtemp(prefix="hd_diag_"), "mma_probe.so")
    cmd = [hd_build._nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-I", os.path.join(HERE, "csrc"), "-I", os.path.join(os.path.dirname(HERE), "include"),
           "-o", out, os.path.join(HERE, "diag", "mma_probe.cu")]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(out)
    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    buf = (ctypes.c_ulonglong * (2 * ctas))()
    for pat, name in enumerate(NAMES):
        lib.run_mma(pat, ctas, buf)  # first run: warm-up
        rc = lib.run_mma(pat, ctas, buf)
        if rc != 0:
            raise RuntimeError(f"probe returned {rc}")
        a = np.frombuffer(buf, dtype=np.uint64).reshape(ctas, 2).astype(np.float64)
        per = a[:, 0] / a[:, 1]
        print(f"{name}: {per.mean():.1f} clk per MMA (min {per.min():.1f}, max {per.max():.1f})")


if __name__ == "__main__":
    main()
