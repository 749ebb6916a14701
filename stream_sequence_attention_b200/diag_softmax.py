"""Diagnostic: clock64 timing of the phases of the attention kernel's softmax.

Compiles ``diag/softmax_probe.cu`` (against the kernels' shared header, not
part of libhd.so) and prints, per choice of FMA-pipe exponential pairs and
for one and two warps per SM sub-partition, the cycles one warp spends per
128-score row in: the tensor-memory load, the row max, the exponents, the
exponentials with bf16 pack and row sum, and the tensor-memory store of P.
One CTA per SM, the scores held in tensor memory, 200 iterations.

    python -m stream_sequence_attention_b200.diag_softmax
"""

import ctypes
import os
import subprocess
import tempfile

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
NAMES = {0: "none", 1: "1 in 3", 2: "1 in 2", 3: "2 in 5", 4: "3 in 8", 5: "1 in 4"}


def main():
    import torch

    from stream_sequence_attention_b200 import build as hd_build

    out = os.path.join(tempfile.mkdtemp(prefix="hd_diag_"), "softmax_probe.so")
    cmd = [hd_build._nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-I", os.path.join(HERE, "csrc"), "-I", os.path.join(os.path.dirname(HERE), "include"),
           "-o", out, os.path.join(HERE, "diag", "softmax_probe.cu")]
    subprocess.run(cmd, check=True)
    lib = ctypes.CDLL(out)
    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    iters = 200
    buf = (ctypes.c_ulonglong * (ctas * 64))()
    print(f"cycles per warp and 128-score row ({ctas} CTAs, {iters} iterations)")
    for sel in NAMES:
        for threads in (128, 256):
            rc = lib.softmax_probe(sel, ctas, threads, iters, buf)
            if rc != 0:
                raise RuntimeError(f"probe returned {rc}")
            c = np.frombuffer(buf, dtype=np.uint64).reshape(ctas, 8, 8)[:, : threads // 32, :5].astype(np.float64)
            m = c.mean(axis=(0, 1)) / iters
            print(f"FMA-pipe pairs {NAMES[sel]:6s}, {threads // 128} warp(s) per sub-partition: load {m[0]:.0f}, "
                  f"max {m[1]:.0f}, exponents {m[2]:.0f}, exponentials+pack+sum {m[3]:.0f}, store {m[4]:.0f}, "
                  f"total {m.sum():.0f}")


if __name__ == "__main__":
    main()
