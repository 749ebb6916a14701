"""Per-role clock counters of the tcgen05 attention kernels (diagnostic).

    python -m stream_sequence_attention_b200.diag_trace [--mode intra|cross] [-D SWITCH=VALUE ...]
    python -m stream_sequence_attention_b200.diag_trace --kernel bwd [--mode intra|cross]

``--kernel bwd`` builds with ``-DHD_BW_TRACE=1`` instead and runs one
``hd_attn_bwd`` call of the bench's backward workload (the same shapes, O
and lse from the forward): per tile of the dK/dV kernel, the cycles its
elementwise warps wait for S, form P, wait for dP and form dS, their
epilogue per unit, and the MMA warp's waits for P, for dS and for the Q/dO/K/V
stages and accumulators.

Builds a diagnostic copy of the library with ``-DHD_TC_TRACE=1`` (plus any
extra switches) next to libhd.so as ``libhd_trace.so``, runs one forward
call of the bench's prefill workload (n=4, L=4096, B=2, 32q/8kv, D=128,
bf16) after three warm-up calls, and prints, averaged over the CTAs, the
cycles per tile each softmax warpgroup spends waiting for its scores, in the
score load, in the mask and row max, in the exponentials up to publishing P,
in the row sum, and (per tile, amortised) in the epilogue's wait for the last
P V and in writing O out; the score load to P published on masked tiles
and on a unit's first tile; and the MMA issuer's cycles waiting for P and for
its Q/K/V/O stages.  The counters perturb the kernel (clock reads and a few
more registers): compare them with each other, not with the timed build.
"""

from __future__ import annotations

import argparse
import ctypes
import os

import numpy as np


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--mode", default="intra", choices=["intra", "cross"])
    ap.add_argument("-D", dest="defines", action="append", default=[])
    ap.add_argument("--kernel", default="fwd", choices=["fwd", "bwd"])
    a = ap.parse_args()
    import torch

    from stream_sequence_attention_b200 import build, hd, synth

    if a.kernel == "bwd":
        return trace_bwd(a, torch, build, hd, synth)

    out = os.path.join(os.path.dirname(build.LIB), "libhd_trace.so")
    build.build(extra=["-DHD_TC_TRACE=1"] + [f"-D{d}" for d in a.defines], out=out)
    hd.LIB_PATH = out
    hd._lib = None
    L = hd.lib()
    L.hd_tc_trace_fetch.argtypes = [ctypes.c_void_p, ctypes.c_int]
    B, n, Lt, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * Lt
    q = synth.normal_device((B, P, Hq, D), 1)
    k = synth.normal_device((B, P, Hkv, D), 2)
    v = synth.normal_device((B, P, Hkv, D), 3)
    o = torch.empty_like(q)
    for _ in range(3):
        hd.hd_attn_fwd(q, k, v, n, a.mode, out=o)
    torch.cuda.synchronize()
    L.hd_tc_trace_clear()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hd.hd_attn_fwd(q, k, v, n, a.mode, out=o)
    e1.record()
    torch.cuda.synchronize()
    slots = 32
    buf = (ctypes.c_ulonglong * (1024 * slots))()
    L.hd_tc_trace_fetch(buf, 1024 * slots)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    c = np.frombuffer(buf, dtype=np.uint64).reshape(1024, slots)[:sms].astype(np.float64)
    print(f"{a.mode}: {e0.elapsed_time(e1):.3f} ms (trace build), {sms} CTAs")
    print(f"  MMA issuer per CTA: waiting for P {c[:, 24].mean() / 1e6:.3f} M clk, for Q/K/V/O "
          f"{c[:, 25].mean() / 1e6:.3f} M clk, total {c[:, 26].mean() / 1e6:.3f} M clk")
    names = ["wait for S", "score load", "mask + max", "exp -> P published", "row sum",
             "epilogue: wait for last P V", "epilogue: O out"]
    for sl in (0, 1):
        b = sl * 12
        tiles = c[:, b + 7].sum()
        per = [c[:, b + i].sum() / tiles for i in range(7)]
        print(f"  softmax slot {sl}: {tiles / sms:.1f} tiles per CTA; clk per tile: " +
              ", ".join(f"{nm} {x:.0f}" for nm, x in zip(names, per)))
        masked = c[:, b + 9].sum()
        print(f"    score load to P published: masked tiles {c[:, b + 8].sum() / max(masked, 1):.0f} clk "
              f"({masked / sms:.1f} per CTA), first tiles of units {c[:, b + 10].sum() / sms:.0f} clk per CTA")


def trace_bwd(a, torch, build, hd, synth):
    out = os.path.join(os.path.dirname(build.LIB), "libhd_trace_bwd.so")
    build.build(extra=["-DHD_BW_TRACE=1"] + [f"-D{d}" for d in a.defines], out=out)
    hd.LIB_PATH = out
    hd._lib = None
    L = hd.lib()
    L.hd_bw_trace_fetch.argtypes = [ctypes.c_void_p, ctypes.c_int]
    B, n, Lt, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * Lt
    q = synth.normal_device((B, P, Hq, D), 1)
    k = synth.normal_device((B, P, Hkv, D), 2)
    v = synth.normal_device((B, P, Hkv, D), 3)
    dO = synth.normal_device((B, P, Hq, D), 4)
    o, lse = hd.hd_attn_fwd(q, k, v, n, a.mode, lse=True)
    for _ in range(3):
        hd.hd_attn_bwd(q, k, v, o, dO, lse, n, a.mode)
    torch.cuda.synchronize()
    L.hd_bw_trace_clear()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hd.hd_attn_bwd(q, k, v, o, dO, lse, n, a.mode)
    e1.record()
    torch.cuda.synchronize()
    slots = 16
    buf = (ctypes.c_ulonglong * (1024 * slots))()
    L.hd_bw_trace_fetch(buf, 1024 * slots)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    c = np.frombuffer(buf, dtype=np.uint64).reshape(1024, slots)[:sms].astype(np.float64)
    tiles = c[:, 4].sum()
    print(f"{a.mode} backward: {e0.elapsed_time(e1):.3f} ms (trace build, whole call), {sms} CTAs, "
          f"{tiles / sms:.1f} dK/dV tiles per CTA")
    names = ["wait for S", "form P", "wait for dP", "form dS"]
    print("  dK/dV elementwise warps, clk per tile: " +
          ", ".join(f"{nm} {c[:, i].sum() / tiles:.0f}" for i, nm in enumerate(names)) +
          f"; epilogue {c[:, 5].mean() / 1e3:.1f} K clk per CTA")
    print(f"  dK/dV MMA warp per CTA: waiting for P {c[:, 8].mean() / 1e6:.3f} M clk, for dS "
          f"{c[:, 9].mean() / 1e6:.3f} M clk, for Q/dO/K/V and accumulators {c[:, 10].mean() / 1e6:.3f} M clk, "
          f"total {c[:, 11].mean() / 1e6:.3f} M clk")


if __name__ == "__main__":
    main()
