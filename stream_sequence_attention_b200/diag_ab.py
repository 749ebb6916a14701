"""Diagnostic: interleaved A/B timing of library variants built from the
committed source with compile-time switches.

    python -m stream_sequence_attention_b200.diag_ab \\
        --variant base= --variant p0=HD_TC_POLY_EVERY=0 --variant p4=HD_TC_POLY_EVERY=4 [--kernel bwd]

Each ``--variant NAME=SWITCH[,SWITCH...]`` builds a copy of libhd.so with
``-DSWITCH`` for every switch listed (none for ``NAME=``).  The variants'
outputs on a small case are compared with the first variant's (max abs
difference), then the bench's workloads (n=4, L=4096, B=2, 32q/8kv, D=128,
bf16; intra and cross) are timed round-robin across the variants with CUDA
events, L2 flushed (512 MiB write) before each launch, and the medians are
printed.  ``--kernel fwd`` times hd_attn_fwd, ``--kernel bwd`` hd_attn_bwd.
"""

from __future__ import annotations

import argparse
import os
import statistics
import tempfile


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--variant", action="append", required=True, help="NAME=SWITCH[,SWITCH...]")
    ap.add_argument("--kernel", default="fwd", choices=["fwd", "bwd"])
    ap.add_argument("--rounds", type=int, default=6)
    a = ap.parse_args()
    import torch

    from stream_sequence_attention_b200 import build, hd, synth

    tmp = tempfile.mkdtemp(prefix="hd_ab_")
    libs = {}
    for spec in a.variant:
        name, _, sw = spec.partition("=")
        flags = [f"-D{x}" for x in sw.split(",") if x]
        out = os.path.join(tmp, f"libhd_{name}.so")
        build.build(extra=flags, out=out)
        # loaded through the binding, which sets the argument types
        hd.LIB_PATH = out
        hd._lib = None
        libs[name] = hd.lib()
        print(f"built {name}: {' '.join(flags) or '(no switches)'}", flush=True)

    def use(name):
        hd._lib = libs[name]

    names = list(libs)
    # agreement on a small case (two heads per KV head, ragged tail, both modes)
    B, n, L, Hq, Hkv, D = 1, 4, 300, 4, 2, 128
    P = n * L
    q, k, v, dO = (synth.normal_device((B, P, H, D), s) for s, H in ((11, Hq), (12, Hkv), (13, Hkv), (14, Hq)))
    ref = {}
    for name in names:
        use(name)
        res = []
        for mode in ("intra", "cross"):
            o, lse = hd.hd_attn_fwd(q, k, v, n, mode, lse=True)
            res.append(o.float())
            if a.kernel == "bwd":
                res.extend(t.float() for t in hd.hd_attn_bwd(q, k, v, o, dO, lse, n, mode))
        torch.cuda.synchronize()
        if not ref:
            ref = {"base": res}
        diff = max(float((x - y).abs().max()) for x, y in zip(res, ref["base"]))
        print(f"{name}: max |difference| from {names[0]} on the small case {diff:.3e}", flush=True)

    B, n, L, Hq, Hkv, D = 2, 4, 4096, 32, 8, 128
    P = n * L
    q = synth.normal_device((B, P, Hq, D), 1)
    k = synth.normal_device((B, P, Hkv, D), 2)
    v = synth.normal_device((B, P, Hkv, D), 3)
    dO = synth.normal_device((B, P, Hq, D), 4)
    o = torch.empty_like(q)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    fwd = {}
    if a.kernel == "bwd":
        use(names[0])
        for mode in ("intra", "cross"):
            oo, ll = hd.hd_attn_fwd(q, k, v, n, mode, lse=True)
            fwd[mode] = (oo, ll)

    def call(mode):
        if a.kernel == "fwd":
            hd.hd_attn_fwd(q, k, v, n, mode, out=o)
        else:
            hd.hd_attn_bwd(q, k, v, fwd[mode][0], dO, fwd[mode][1], n, mode)

    for name in names:
        use(name)
        for mode in ("intra", "cross"):
            for _ in range(3):
                call(mode)
    torch.cuda.synchronize()
    times = {(nm, m): [] for nm in names for m in ("intra", "cross")}
    for _ in range(a.rounds):
        for name in names:
            use(name)
            for mode in ("intra", "cross"):
                for _ in range(3):
                    flush.fill_(1)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    call(mode)
                    e1.record()
                    e1.synchronize()
                    times[(name, mode)].append(e0.elapsed_time(e1))
    for name in names:
        print(f"{name}: " + "  ".join(f"{m} {statistics.median(times[(name, m)]):.4f} ms "
                                      f"(min {min(times[(name, m)]):.4f})" for m in ("intra", "cross")), flush=True)


if __name__ == "__main__":
    main()
