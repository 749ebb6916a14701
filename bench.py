"""Benchmark of the Hidden Decoding hot path on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload intra|cross|long|decode|mirror|bwd|bwd_cross|rope]
                    [--no-extras]

Default workload (intra): n=4 streams, L=4096 tokens (nL=16384), batch 2,
32 query / 8 KV heads, head_dim 128, bf16.  One step is one pass of the
prefill hot path over one batch: hd_expand_embed (4 tables of 152064 x 4096,
Zipf(1.1) ids) -> hd_attn_fwd (intra-stream, causal) -> hd_final_stream_gather
(final-stream rows of the expanded [B, nL, 4096] sequence).  The metric is
useful attention TFLOP/s (visible pairs x 4 x head_dim per second of step
time); the decode workload (batch 64, 32768 tokens per stream, both modes) is
reported alongside in GB/s against HBM, and the cross-stream layer, the
KV-mirror layer and the backward (dQ, dK, dV; useful FLOPs = pairs x 10 x D)
in TFLOP/s.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream, with an L2 flush (a 512 MiB write) between steps
outside the events; a barrier and a device synchronise on both sides; the
max over ranks.  With N > 1 every rank runs its own batch (data-parallel,
weak scaling; no collective on the data path).

--impl reference times the float64 CPU oracle on this machine's host cores
(rank 0 only) on bounded samples of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "intra": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, mode="intra", W=0, V=152064, dm=4096),
    "cross": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, mode="cross", W=0, V=152064, dm=4096),
    "long": dict(B=1, n=4, L=32768, Hq=64, Hkv=8, D=128, mode="intra", W=4096, V=152064, dm=4096),
    "decode": dict(B=64, n=4, T=32768, Hq=64, Hkv=8, D=128),
    "mirror": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, mode="cross", W=0, V=152064, dm=4096, final=True),
    "bwd": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, mode="intra", W=0, bwd=True),
    "bwd_cross": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, mode="cross", W=0, bwd=True),
    "rope": dict(B=2, n=4, L=4096, Hq=32, Hkv=8, D=128, rope=True),
}
NAMES = {
    "intra": "bf16 prefill, intra-stream, n=4 L=4096 B=2 32q/8kv D=128",
    "cross": "bf16 prefill, cross-stream, n=4 L=4096 B=2 32q/8kv D=128",
    "long": "long-context intra-stream W=4096, n=4 L=32768 B=1 64q/8kv D=128",
    "decode": "decode B=64 n=4 ctx=32768 64q/8kv D=128, intra+cross",
    "mirror": "bf16 KV-mirror layer: final-stream queries, cross-stream keys, n=4 L=4096 B=2 32q/8kv D=128",
    "bwd": "bf16 attention backward (dQ, dK, dV), intra-stream, n=4 L=4096 B=2 32q/8kv D=128",
    "bwd_cross": "bf16 attention backward (dQ, dK, dV), cross-stream, n=4 L=4096 B=2 32q/8kv D=128",
    "rope": "bf16 RoPE in place on q and k at positions i*n+s, n=4 L=4096 B=2 32q/8kv D=128",
}
FLUSH_BYTES = 512 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="intra", choices=list(WORKLOADS))
    ap.add_argument("--no-extras", action="store_true", help="skip the side measurements")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (small ncu captures)")
    ap.add_argument("--profile", action="store_true",
                    help="timed steps only (no e2e, side measurements or CPU oracle): for ncu captures")
    return ap.parse_args()


# --------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


HOST_MARKER = b"// ------------------------------------------------------------------- host"


def kernel_source_sha(names):
    """Hash of the device part of the named sources (each file up to its
    host-code marker): a recorded traffic figure stays valid across host-side
    edits and turns stale when a kernel changes."""
    h = hashlib.sha256()
    for nm in names:
        with open(os.path.join(ROOT, "stream_sequence_attention_b200", "csrc", nm), "rb") as f:
            src = f.read()
        cut = src.find(HOST_MARKER)
        h.update(src if cut < 0 else src[:cut])
    return h.hexdigest()[:16]


def recorded_traffic(kernel, sources, workload):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel source changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    e = t.get(kernel, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha(sources):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    INTERVAL_MS = 20

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []  # (arrival time, line)

    def start(self):
        """Start sampling; returns once the first sample has arrived (at most
        a few seconds), so that a short timed region still gets samples."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.INTERVAL_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
            return
        t0 = time.monotonic()
        while not self.lines and self.proc.poll() is None and time.monotonic() - t0 < 5.0:
            time.sleep(0.005)

    def mark(self):
        """Call right before the timed region."""
        self.t_begin = time.monotonic()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self):
        """Call right after the timed region.  Keeps the samples that arrived
        within one interval of it."""
        if self.proc is None:
            return None
        t_end = time.monotonic()
        time.sleep(2 * self.INTERVAL_MS / 1000)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        slack = self.INTERVAL_MS / 1000
        t_begin = getattr(self, "t_begin", t_end)
        window = [ln for (t, ln) in self.lines if t_begin - slack <= t <= t_end + slack]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in window:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ GPU workloads

class Prefill:
    """expand -> attention -> final-stream gather on device-resident inputs."""

    def __init__(self, cfg, seed_base, torch, hd, synth):
        self.cfg = c = cfg
        self.torch, self.hd = torch, hd
        P = c["n"] * c["L"]
        self.P = P
        ids = synth.ids_zipf(c["B"], c["L"], c["V"], 1.1, seed_base + 1)
        self.ids_host = torch.from_numpy(ids).pin_memory()
        self.ids = self.ids_host.cuda()
        self.tables = synth.normal_device((c["n"], c["V"], c["dm"]), seed_base + 2, std=0.02)
        self.final = bool(c.get("final"))
        qrows = c["L"] if self.final else P
        self.q = synth.normal_device((c["B"], qrows, c["Hq"], c["D"]), seed_base + 3)
        self.k = synth.normal_device((c["B"], P, c["Hkv"], c["D"]), seed_base + 4)
        self.v = synth.normal_device((c["B"], P, c["Hkv"], c["D"]), seed_base + 5)
        self.x = torch.empty((c["B"], P, c["dm"]), dtype=torch.bfloat16, device="cuda")
        self.o = torch.empty_like(self.q)
        self.g = torch.empty((c["B"], c["L"], c["dm"]), dtype=torch.bfloat16, device="cuda")
        self.status = hd.new_status()

    def step(self, ev=None):
        c, hd = self.cfg, self.hd
        hd.hd_expand_embed(self.tables, self.ids, self.x, dev_status=self.status)
        if ev is not None:
            ev[0].record()
        if self.final:
            hd.hd_attn_fwd_final_stream(self.q, self.k, self.v, c["n"], c["mode"], c["W"], out=self.o,
                                        dev_status=self.status)
        else:
            hd.hd_attn_fwd(self.q, self.k, self.v, c["n"], c["mode"], c["W"], out=self.o, dev_status=self.status)
        if ev is not None:
            ev[1].record()
        hd.hd_final_stream_gather(self.x, c["n"], out=self.g)

    launches_per_step = 3

    def e2e_buffers(self):
        torch = self.torch
        self.h_q = torch.empty_like(self.q, device="cpu").pin_memory()
        self.h_k = torch.empty_like(self.k, device="cpu").pin_memory()
        self.h_v = torch.empty_like(self.v, device="cpu").pin_memory()
        self.h_q.copy_(self.q)
        self.h_k.copy_(self.k)
        self.h_v.copy_(self.v)
        self.h_g = torch.empty_like(self.g, device="cpu").pin_memory()
        self.h_o = torch.empty_like(self.o, device="cpu").pin_memory()
        return (self.ids_host.numel() * 4 + 2 * (self.h_q.numel() + self.h_k.numel() + self.h_v.numel()),
                2 * (self.h_g.numel() + self.h_o.numel()))

    def e2e_step(self):
        """Host inputs -> device, the step, results -> host (pinned buffers)."""
        self.ids.copy_(self.ids_host, non_blocking=True)
        self.q.copy_(self.h_q, non_blocking=True)
        self.k.copy_(self.h_k, non_blocking=True)
        self.v.copy_(self.h_v, non_blocking=True)
        self.step()
        self.h_o.copy_(self.o, non_blocking=True)
        self.h_g.copy_(self.g, non_blocking=True)

    def e2e_pipelined(self, K, dist=None):
        """K end-to-end steps with the copies overlapped: three CUDA streams,
        two device buffer slots.  Step i copies its inputs (ids, q, k, v) from
        pinned host memory into slot i%2, runs expand -> attention -> gather
        on it, and copies O and the gathered rows back; the H2D of step i+1
        and the D2H of step i-1 run while step i computes.  Inputs (0.4 GB)
        exceed L2, so no flush.  Returns the wall time of the K steps (ms,
        CUDA events on the compute stream, after every stream has joined)."""
        torch, hd, c = self.torch, self.hd, self.cfg
        if not hasattr(self, "slots"):
            self.slots = [dict(ids=self.ids, q=self.q, k=self.k, v=self.v, x=self.x, o=self.o, g=self.g)]
            self.slots.append({k: torch.empty_like(t) for k, t in self.slots[0].items()})
        s_c = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        start.record(s_c)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(K):
            b = i % 2
            sl = self.slots[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_out[b])  # slot b's step i-2 has computed and been copied out
                sl["ids"].copy_(self.ids_host, non_blocking=True)
                sl["q"].copy_(self.h_q, non_blocking=True)
                sl["k"].copy_(self.h_k, non_blocking=True)
                sl["v"].copy_(self.h_v, non_blocking=True)
                ev_in[b].record(s_in)
            s_c.wait_event(ev_in[b])
            hd.hd_expand_embed(self.tables, sl["ids"], sl["x"], dev_status=self.status, stream=s_c)
            if self.final:
                hd.hd_attn_fwd_final_stream(sl["q"], sl["k"], sl["v"], c["n"], c["mode"], c["W"], out=sl["o"],
                                            dev_status=self.status, stream=s_c)
            else:
                hd.hd_attn_fwd(sl["q"], sl["k"], sl["v"], c["n"], c["mode"], c["W"], out=sl["o"],
                               dev_status=self.status, stream=s_c)
            hd.hd_final_stream_gather(sl["x"], c["n"], out=sl["g"], stream=s_c)
            ev_done[b].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                self.h_o.copy_(sl["o"], non_blocking=True)
                self.h_g.copy_(sl["g"], non_blocking=True)
                ev_out[b].record(s_out)
        s_c.wait_stream(s_in)
        s_c.wait_stream(s_out)
        end.record(s_c)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return start.elapsed_time(end)

    def flops(self):
        from stream_sequence_attention_b200 import accounting as acc
        c = self.cfg
        if self.final:
            return acc.attn_flops_final_stream(c["B"], c["L"], c["n"], c["Hq"], c["D"], c["mode"], c["W"])
        return acc.attn_flops(c["B"], c["L"], c["n"], c["Hq"], c["D"], c["mode"], c["W"])


class Decode:
    """hd_attn_decode, intra then cross, against a resident per-stream cache."""

    def __init__(self, cfg, seed_base, torch, hd, synth):
        self.cfg = c = cfg
        self.torch, self.hd = torch, hd
        self.q = synth.normal_device((c["B"], c["n"], c["Hq"], c["D"]), seed_base + 1)
        self.kc = synth.normal_device((c["B"], c["n"], c["T"], c["Hkv"], c["D"]), seed_base + 2)
        self.vc = synth.normal_device((c["B"], c["n"], c["T"], c["Hkv"], c["D"]), seed_base + 3)
        self.ctx = torch.full((c["B"],), c["T"], dtype=torch.int32, device="cuda")
        self.o = {m: torch.empty_like(self.q) for m in ("intra", "cross")}
        wsb = max(hd.hd_attn_decode_workspace(c["B"], c["n"], c["T"], c["Hq"], c["Hkv"], c["D"], m)
                  for m in ("intra", "cross"))
        self.ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        self.status = hd.new_status()

    def run(self, mode):
        self.hd.hd_attn_decode(self.q, self.kc, self.vc, self.ctx, mode, out=self.o[mode], workspace=self.ws,
                               dev_status=self.status)

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.run("intra")
        if ev is not None:
            ev[1].record()
        self.run("cross")

    launches_per_step = 4  # decode + combine, per mode

    def bytes_per_mode(self):
        from stream_sequence_attention_b200 import accounting as acc
        c = self.cfg
        return acc.decode_bytes(c["B"], c["n"], c["T"], c["Hq"], c["Hkv"], c["D"])

    def e2e_buffers(self):
        torch = self.torch
        self.h_q = torch.empty_like(self.q, device="cpu").pin_memory()
        self.h_q.copy_(self.q)
        self.h_o = {m: torch.empty_like(self.q, device="cpu").pin_memory() for m in self.o}
        return 2 * self.h_q.numel(), 2 * 2 * self.h_q.numel()

    def e2e_step(self):
        self.q.copy_(self.h_q, non_blocking=True)
        self.step()
        for m in self.o:
            self.h_o[m].copy_(self.o[m], non_blocking=True)


class Backward:
    """hd_attn_bwd on device-resident q, k, v, o, lse and dO (o and lse from
    the library's forward of the same inputs)."""

    def __init__(self, cfg, seed_base, torch, hd, synth):
        self.cfg = c = cfg
        self.torch, self.hd = torch, hd
        P = c["n"] * c["L"]
        self.q = synth.normal_device((c["B"], P, c["Hq"], c["D"]), seed_base + 3)
        self.k = synth.normal_device((c["B"], P, c["Hkv"], c["D"]), seed_base + 4)
        self.v = synth.normal_device((c["B"], P, c["Hkv"], c["D"]), seed_base + 5)
        self.dO = synth.normal_device((c["B"], P, c["Hq"], c["D"]), seed_base + 6)
        self.status = hd.new_status()
        self.o, self.lse = hd.hd_attn_fwd(self.q, self.k, self.v, c["n"], c["mode"], c["W"], lse=True,
                                          dev_status=self.status)
        self.dq = torch.empty_like(self.q)
        self.dk = torch.empty_like(self.k)
        self.dv = torch.empty_like(self.v)
        self.ws = torch.empty(hd.hd_attn_bwd_workspace(c["B"], c["L"], c["n"], c["Hq"], c["mode"]),
                              dtype=torch.uint8, device="cuda")

    def step(self, ev=None):
        c = self.cfg
        if ev is not None:
            ev[0].record()
        self.hd.hd_attn_bwd(self.q, self.k, self.v, self.o, self.dO, self.lse, c["n"], c["mode"], c["W"],
                            dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws, dev_status=self.status)
        if ev is not None:
            ev[1].record()

    launches_per_step = 3  # lse/delta preparation, dK/dV, dQ

    def e2e_buffers(self):
        torch = self.torch
        self.h_in = [torch.empty_like(t, device="cpu").pin_memory() for t in
                     (self.q, self.k, self.v, self.o, self.dO, self.lse)]
        for h, t in zip(self.h_in, (self.q, self.k, self.v, self.o, self.dO, self.lse)):
            h.copy_(t)
        self.h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in (self.dq, self.dk, self.dv)]
        bi = sum(h.numel() * h.element_size() for h in self.h_in)
        bo = sum(h.numel() * h.element_size() for h in self.h_out)
        return bi, bo

    def e2e_step(self):
        for t, h in zip((self.q, self.k, self.v, self.o, self.dO, self.lse), self.h_in):
            t.copy_(h, non_blocking=True)
        self.step()
        for h, t in zip(self.h_out, (self.dq, self.dk, self.dv)):
            h.copy_(t, non_blocking=True)

    def flops(self):
        from stream_sequence_attention_b200 import accounting as acc
        c = self.cfg
        return acc.attn_bwd_flops(c["B"], c["L"], c["n"], c["Hq"], c["D"], c["mode"], c["W"])


class Rope:
    """hd_rope in place on device-resident q and k (one launch)."""

    def __init__(self, cfg, seed_base, torch, hd, synth):
        self.cfg = c = cfg
        self.torch, self.hd = torch, hd
        P = c["n"] * c["L"]
        self.q = synth.normal_device((c["B"], P, c["Hq"], c["D"]), seed_base + 3)
        self.k = synth.normal_device((c["B"], P, c["Hkv"], c["D"]), seed_base + 4)
        self.status = hd.new_status()

    def step(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.hd.hd_rope(self.q, self.k)
        if ev is not None:
            ev[1].record()

    launches_per_step = 1

    def nbytes(self):
        return 2 * (self.q.numel() + self.k.numel()) * self.q.element_size()

    def e2e_buffers(self):
        torch = self.torch
        self.h = [torch.empty_like(t, device="cpu").pin_memory() for t in (self.q, self.k)]
        for h, t in zip(self.h, (self.q, self.k)):
            h.copy_(t)
        n = sum(h.numel() * h.element_size() for h in self.h)
        return n, n

    def e2e_step(self):
        for t, h in zip((self.q, self.k), self.h):
            t.copy_(h, non_blocking=True)
        self.step()
        for h, t in zip(self.h, (self.q, self.k)):
            h.copy_(t, non_blocking=True)


def timed(torch, work, K, flush, dist=None, use_e2e=False, parts=None):
    """Run K steps with per-step CUDA events (flush outside them).  Returns
    (per-step ms list, dominant-kernel ms list); with ``parts`` (a list) it
    also receives per-step (ms before the dominant kernel, ms after it)."""
    st = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush()
        st[i].record()
        if use_e2e:
            work.e2e_step()
        else:
            work.step(kev[i])
        en[i].record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    steps = [a.elapsed_time(b) for a, b in zip(st, en)]
    kern = [] if use_e2e else [a.elapsed_time(b) for a, b in kev]
    if parts is not None and not use_e2e:
        parts.extend((a.elapsed_time(k0), k1.elapsed_time(b)) for a, (k0, k1), b in zip(st, kev, en))
    return steps, kern


def max_over_ranks(torch, dist, x, device="cuda"):
    """The slowest rank's time: every rank's share counts only when all are done."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload, rank):
    """Seed base of a rank's inputs: every rank draws its own batch."""
    return 1000 * (list(WORKLOADS).index(workload) + 1) + 97 * rank


def run_ours(args, rank, world, dist):
    import torch

    from stream_sequence_attention_b200 import build as hd_build
    from stream_sequence_attention_b200 import hd, synth

    hd_build.build()
    hd.lib()
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    peaks = load_peaks()
    wl = args.workload
    cfg = dict(WORKLOADS[wl])
    if args.batch:
        cfg["B"] = args.batch
    K = args.steps if args.steps is not None else (100 if wl != "decode" else 40)
    W = args.warmup if args.warmup is not None else 5
    W = max(W, 3)
    seed_base = rank_seed(wl, rank)
    if wl == "decode":
        work = Decode(cfg, seed_base, torch, hd, synth)
    elif cfg.get("bwd"):
        work = Backward(cfg, seed_base, torch, hd, synth)
    elif cfg.get("rope"):
        work = Rope(cfg, seed_base, torch, hd, synth)
    else:
        work = Prefill(cfg, seed_base, torch, hd, synth)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush = lambda: flush_buf.fill_(1)  # noqa: E731

    for _ in range(W):
        flush()
        work.step()
    torch.cuda.synchronize()
    if int(work.status.item()) != 0:
        raise RuntimeError(f"device status {hd.status_string(int(work.status.item()))}")

    clocks = ClockSampler(int(os.environ.get("LOCAL_RANK", 0)))
    clocks.start()
    clocks.mark()
    parts = []
    steps, kern = timed(torch, work, K, flush, dist, parts=parts)
    clk = clocks.stop()
    if args.profile:
        return {"profile": True, "ms_per_step": sum(steps) / K, "kernel_ms": statistics.mean(kern)}, work, peaks
    total_ms = sum(steps)
    total_ms = max_over_ranks(torch, dist, total_ms)
    ms_per_step = total_ms / K
    kern_ms = statistics.mean(kern)

    # e2e through the public API with host buffers
    bi, bo = work.e2e_buffers()
    for _ in range(2):
        work.e2e_step()
    if hasattr(work, "e2e_pipelined"):
        work.e2e_pipelined(2, dist)
        e2e_total = work.e2e_pipelined(args.e2e_steps, dist)
        e2e_mode = "pipelined: the H2D of step i+1 and the D2H of step i-1 overlap step i (three streams, two slots)"
    else:
        e2e_steps, _ = timed(torch, work, args.e2e_steps, flush, dist, use_e2e=True)
        e2e_total = sum(e2e_steps)
        e2e_mode = "serial: H2D, step, D2H per step"
    e2e_ms = max_over_ranks(torch, dist, e2e_total) / args.e2e_steps

    out = {}
    if wl == "decode":
        nbytes = 2 * work.bytes_per_mode()
        value = world * nbytes / (ms_per_step * 1e-3) / 1e9
        metric, unit = "decode GB/s vs HBM (intra+cross, B=64 n=4 ctx=32768)", "GB/s"
        achieved = work.bytes_per_mode() / (kern_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "kernel": "decode_kernel (intra) + combine",
                "peak_source": peaks["source"] + " hbm_gbs",
                "traffic": recorded_traffic("decode_kernel", ["decode.cu"], "decode_intra")}
        e2e_value = world * nbytes / (e2e_ms * 1e-3) / 1e9
        dtype = "bf16"
    elif cfg.get("rope"):
        nbytes = work.nbytes()
        value = world * nbytes / (ms_per_step * 1e-3) / 1e9
        metric, unit = "RoPE GB/s vs HBM (q and k in place, n=4 L=4096 B=2 32q/8kv)", "GB/s"
        achieved = nbytes / (kern_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "kernel": "rope_kernel<true>",
                "peak_source": peaks["source"] + " hbm_gbs",
                "traffic": recorded_traffic("rope_kernel", ["rope.cu"], wl)}
        e2e_value = world * nbytes / (e2e_ms * 1e-3) / 1e9
        dtype = "bf16"
    elif cfg.get("bwd"):
        fl = work.flops()
        value = world * fl / (ms_per_step * 1e-3) / 1e12
        metric = "useful attn backward TFLOP/s at n=4 (%s)" % cfg["mode"]
        unit = "TFLOP/s"
        achieved = fl / (kern_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16"], 4),
                "kernel": "hd_attn_bwd (bwd_prep + attn_bwd_dkv_kernel<128> + attn_bwd_dq_kernel<128>)",
                "peak_source": peaks["source"] + " bf16_tflops (burst)",
                "flops_convention": "useful = visible pairs x 10 x D; the kernels execute 14 x D per pair",
                "traffic": recorded_traffic("attn_bwd", ["attn_bwd_tc.cu", "attn_bwd_f32.cu", "hd_common.cuh"],
                                            wl)}
        e2e_value = world * fl / (e2e_ms * 1e-3) / 1e12
        dtype = "bf16"
    else:
        fl = work.flops()
        value = world * fl / (ms_per_step * 1e-3) / 1e12
        metric = "useful attn TFLOP/s at n=4 (%s)" % (cfg["mode"] + (", final-stream queries" if cfg.get("final") else ""))
        unit = "TFLOP/s"
        achieved = fl / (kern_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16"], 4), "kernel": "attn_tc_kernel<128>",
                "peak_source": peaks["source"] + " bf16_tflops (burst)",
                "traffic": recorded_traffic("attn_tc_kernel", ["attn_tc.cu", "hd_common.cuh"], wl)}
        e2e_value = world * fl / (e2e_ms * 1e-3) / 1e12
        dtype = "bf16"
    out.update({
        "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic (seeded; device-drawn N(0,1) q/k/v, N(0,0.02) tables, Zipf(1.1) ids)",
        "config": {"workload": NAMES[wl], "global_batch": cfg["B"] * world,
                   "seq_len": cfg.get("L", cfg.get("T")) * cfg["n"], "parallelism": f"dp{world}",
                   "l2": "flushed between timed steps (512 MiB write, outside the step events)"},
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": unit, "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
                "ms_per_step": round(e2e_ms, 3), "mode": e2e_mode},
        "gpu_launches": work.launches_per_step * K,
        "clocks": clk,
    })
    if isinstance(work, Prefill):
        # expand runs before the attention in the step, the gather after it
        from stream_sequence_attention_b200 import accounting as acc
        exp_ms = statistics.mean(p[0] for p in parts)
        gat_ms = statistics.mean(p[1] for p in parts)
        eb = acc.expand_bytes(cfg["B"], cfg["L"], cfg["n"], cfg["dm"])
        gb = acc.gather_bytes(cfg["B"], cfg["L"], cfg["dm"])
        uniq = int(torch.unique(work.ids).numel())
        out["expand"] = {"ms": round(exp_ms, 4), "GB/s": round(eb / (exp_ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(eb / (exp_ms * 1e-3) / 1e9 / peaks["hbm"], 4),
                         "unique_rows_per_table": uniq, "rows_per_table": cfg["B"] * cfg["L"],
                         "note": "Zipf(1.1) ids repeat rows; L2 hits on repeats can lift this figure above HBM"}
        out["gather"] = {"ms": round(gat_ms, 4), "GB/s": round(gb / (gat_ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(gb / (gat_ms * 1e-3) / 1e9 / peaks["hbm"], 4)}
    return out, work, peaks


def extras(torch, peaks, rank):
    """Side measurements on one GPU: decode GB/s (both modes), the
    cross-stream prefill layer, the KV-mirror layer, the long-context
    workload (expand, windowed intra attention, gather), RoPE, rank 0's
    stream-parallel share and the backward."""
    from stream_sequence_attention_b200 import hd, synth

    res = {}
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush = lambda: flush_buf.fill_(1)  # noqa: E731

    def time_fn(fn, K=10, W=3):
        for _ in range(W):
            flush()
            fn()
        ts = []
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    dec = Decode(WORKLOADS["decode"], 7001 + rank, torch, hd, synth)
    nb = dec.bytes_per_mode()
    for mode in ("intra", "cross"):
        ms = time_fn(lambda: dec.run(mode))
        gbs = nb / (ms * 1e-3) / 1e9
        res[f"decode_{mode}"] = {"ms": round(ms, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 4)}
    del dec
    torch.cuda.empty_cache()
    cr = Prefill(WORKLOADS["cross"], 7101 + rank, torch, hd, synth)
    c = WORKLOADS["cross"]
    ms = time_fn(lambda: hd.hd_attn_fwd(cr.q, cr.k, cr.v, c["n"], "cross", out=cr.o))
    tf = cr.flops() / (ms * 1e-3) / 1e12
    res["cross_prefill"] = {"ms": round(ms, 3), "TFLOP/s": round(tf, 1), "frac_bf16": round(tf / peaks["bf16"], 4)}
    del cr
    torch.cuda.empty_cache()
    mi = Prefill(WORKLOADS["mirror"], 7201 + rank, torch, hd, synth)
    c = WORKLOADS["mirror"]
    ms = time_fn(lambda: hd.hd_attn_fwd_final_stream(mi.q, mi.k, mi.v, c["n"], "cross", out=mi.o))
    tf = mi.flops() / (ms * 1e-3) / 1e12
    res["mirror_final_stream_cross"] = {"ms": round(ms, 3), "TFLOP/s": round(tf, 1),
                                        "frac_bf16": round(tf / peaks["bf16"], 4)}
    del mi
    torch.cuda.empty_cache()
    # Long-context workload: expand over 4 tables of 152064 x 4096 with
    # Zipf(1.1) ids -> intra-stream attention with a 4096-token window ->
    # final-stream gather, n=4 L=32768 B=1 64q/8kv D=128; each part timed.
    from stream_sequence_attention_b200 import accounting as acc
    lc = Prefill(WORKLOADS["long"], 7601 + rank, torch, hd, synth)
    c = WORKLOADS["long"]
    ms_e = time_fn(lambda: hd.hd_expand_embed(lc.tables, lc.ids, lc.x, dev_status=lc.status))
    ms_a = time_fn(lambda: hd.hd_attn_fwd(lc.q, lc.k, lc.v, c["n"], c["mode"], c["W"], out=lc.o,
                                          dev_status=lc.status))
    ms_g = time_fn(lambda: hd.hd_final_stream_gather(lc.x, c["n"], out=lc.g))
    torch.cuda.synchronize()
    if int(lc.status.item()) != 0:
        raise RuntimeError(f"device status {hd.status_string(int(lc.status.item()))}")
    tf = lc.flops() / (ms_a * 1e-3) / 1e12
    eb = acc.expand_bytes(c["B"], c["L"], c["n"], c["dm"])
    gb = acc.gather_bytes(c["B"], c["L"], c["dm"])
    res["long_context"] = {
        "workload": NAMES["long"] + ", expand 4 x 152064 x 4096 Zipf(1.1) ids, final-stream gather",
        "attn_ms": round(ms_a, 3), "attn_TFLOP/s": round(tf, 1), "attn_frac_bf16": round(tf / peaks["bf16"], 4),
        "expand_ms": round(ms_e, 4), "expand_GB/s": round(eb / (ms_e * 1e-3) / 1e9, 1),
        "expand_unique_rows_per_table": int(torch.unique(lc.ids).numel()), "expand_rows_per_table": c["B"] * c["L"],
        "gather_ms": round(ms_g, 4), "gather_GB/s": round(gb / (ms_g * 1e-3) / 1e9, 1),
        "gather_frac_hbm": round(gb / (ms_g * 1e-3) / 1e9 / peaks["hbm"], 4),
        "step_ms": round(ms_e + ms_a + ms_g, 3),
        "repeats": 10, "l2": "flushed before each timed launch"}
    del lc
    torch.cuda.empty_cache()
    # A plain device-to-device copy of as many bytes as each gather moves
    # (torch copy_, i.e. the driver's memcpy, not this library's kernel): the
    # rate HBM gives a copy of that size, fixed launch and drain costs
    # included, beside the gather's own.
    res["copy_same_bytes_as_gather"] = {}
    for wl in ("intra", "long"):
        c = WORKLOADS[wl]
        gb = acc.gather_bytes(c["B"], c["L"], c["dm"])
        src = torch.empty(gb // 2, dtype=torch.uint8, device="cuda")
        dst = torch.empty_like(src)
        ms_c = time_fn(lambda: dst.copy_(src))
        res["copy_same_bytes_as_gather"][wl] = {
            "bytes": gb, "ms": round(ms_c, 4), "GB/s": round(gb / (ms_c * 1e-3) / 1e9, 1),
            "frac_hbm": round(gb / (ms_c * 1e-3) / 1e9 / peaks["hbm"], 4)}
        del src, dst
    torch.cuda.empty_cache()
    # RoPE fused into the attention (intra workload): hd_rope on q and k then
    # hd_attn_fwd, against hd_attn_fwd_rope (k rotated in place, q rotated
    # inside the attention kernel).  Repeated rotation of the same buffers
    # changes the values, not the work.
    c = WORKLOADS["intra"]
    B, P = c["B"], c["n"] * c["L"]
    rq = synth.normal_device((B, P, c["Hq"], c["D"]), 7701 + rank)
    rk = synth.normal_device((B, P, c["Hkv"], c["D"]), 7702 + rank)
    rv = synth.normal_device((B, P, c["Hkv"], c["D"]), 7703 + rank)
    ro = torch.empty_like(rq)
    ms_sep = time_fn(lambda: (hd.hd_rope(rq, rk), hd.hd_attn_fwd(rq, rk, rv, c["n"], "intra", out=ro)))
    ms_fused = time_fn(lambda: hd.hd_attn_fwd_rope(rq, rk, rv, c["n"], "intra", out=ro))
    fl = acc.attn_flops(B, c["L"], c["n"], c["Hq"], c["D"], "intra", 0)
    res["rope_fused_intra"] = {"separate_ms": round(ms_sep, 3), "fused_ms": round(ms_fused, 3),
                               "fused_attn_TFLOP/s": round(fl / (ms_fused * 1e-3) / 1e12, 1),
                               "note": "separate = hd_rope(q, k) + hd_attn_fwd; fused = hd_attn_fwd_rope "
                                       "(rope(k) + attention with q rotated in the kernel)"}
    del rq, rk, rv, ro
    torch.cuda.empty_cache()
    rp = Rope(WORKLOADS["rope"], 7401 + rank, torch, hd, synth)
    ms = time_fn(lambda: rp.step())
    gbs = rp.nbytes() / (ms * 1e-3) / 1e9
    res["rope"] = {"ms": round(ms, 3), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm"], 4)}
    del rp
    torch.cuda.empty_cache()
    res.update(stream_parallel_rank(torch, peaks, rank, time_fn))
    for wl in ("bwd", "bwd_cross"):
        bw = Backward(WORKLOADS[wl], 7301 + rank, torch, hd, synth)
        ms = time_fn(lambda: bw.step())
        tf = bw.flops() / (ms * 1e-3) / 1e12
        res[f"backward_{WORKLOADS[wl]['mode']}"] = {"ms": round(ms, 3), "TFLOP/s": round(tf, 1),
                                                  "frac_bf16": round(tf / peaks["bf16"], 4)}
        del bw
        torch.cuda.empty_cache()
    return res


def stream_parallel_rank(torch, peaks, rank, time_fn, R=4):
    """Rank 0's share of a stream-parallel step with R ranks, timed on one GPU:
    the re-interleave of the all-gathered K/V shards and the local queries'
    cross-stream attention (cross workload sizes), and the cross-stream decode
    partial over the rank's cache streams plus the merge of R partials
    (decode workload sizes).  The all-gathers themselves need R GPUs."""
    from stream_sequence_attention_b200 import accounting as acc
    from stream_sequence_attention_b200 import hd, synth

    res = {}
    c = WORKLOADS["cross"]
    B, n, L, Hq, Hkv, D = c["B"], c["n"], c["L"], c["Hq"], c["Hkv"], c["D"]
    nl = n // R
    q_loc = synth.normal_device((B, L * nl, Hq, D), 7501 + rank)
    kparts = synth.normal_device((R, B, L * nl, Hkv, D), 7502 + rank)
    vparts = synth.normal_device((R, B, L * nl, Hkv, D), 7503 + rank)
    k = torch.empty((B, n * L, Hkv, D), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    o = torch.empty_like(q_loc)
    ms_il = time_fn(lambda: (hd.hd_stream_interleave(kparts, n, out=k), hd.hd_stream_interleave(vparts, n, out=v)))
    il_bytes = 2 * 2 * k.numel() * k.element_size()
    ms_at = time_fn(lambda: hd.hd_attn_fwd_shard(q_loc, k, v, n, R, 0, out=o))
    fl = B * Hq * acc.pairs_cross_shard(L, n, R, 0) * 4 * D
    # The same rows straight from the gathered shards (no re-interleave), and
    # the fused form that copies the R-1 other shards inside the kernel (here
    # from this GPU's memory, so the copies compete for HBM, not NVLink).
    ms_parts = time_fn(lambda: hd.hd_attn_fwd_parts(q_loc, kparts, vparts, n, R, 0, out=o))
    kd = torch.empty_like(kparts)
    vd = torch.empty_like(vparts)
    flags = torch.empty(max(1, hd.hd_attn_peer_flags_bytes(B, L, n) // 8), dtype=torch.int64, device="cuda")
    ms_fused = time_fn(lambda: hd.hd_attn_fwd_peer_gather(q_loc, list(kparts), list(vparts), kd, vd, n, R, 0,
                                                          flags=flags, out=o))
    tf = lambda ms: round(fl / (ms * 1e-3) / 1e12, 1)  # noqa: E731
    res[f"sp_R{R}_rank0_cross_prefill"] = {
        "interleave_ms": round(ms_il, 3), "interleave_GB/s": round(il_bytes / (ms_il * 1e-3) / 1e9, 1),
        "attn_ms": round(ms_at, 3), "attn_TFLOP/s": tf(ms_at),
        "attn_frac_bf16": round(fl / (ms_at * 1e-3) / 1e12 / peaks["bf16"], 4),
        "parts_ms": round(ms_parts, 3), "parts_TFLOP/s": tf(ms_parts),
        "peer_gather_ms": round(ms_fused, 3), "peer_gather_TFLOP/s": tf(ms_fused),
        "allgather_bytes_in_per_rank": (R - 1) * 2 * kparts[0].numel() * 2}
    del q_loc, kparts, vparts, k, v, o, kd, vd, flags
    torch.cuda.empty_cache()
    d = WORKLOADS["decode"]
    B, n, T, Hq, Hkv, D = d["B"], d["n"], d["T"], d["Hq"], d["Hkv"], d["D"]
    q = synth.normal_device((B, n, Hq, D), 7511 + rank)
    kc = synth.normal_device((B, n // R, T, Hkv, D), 7512 + rank)
    vc = synth.normal_device((B, n // R, T, Hkv, D), 7513 + rank)
    ctx = torch.full((B,), T, dtype=torch.int32, device="cuda")
    op = torch.empty((B, n, Hq, D), dtype=torch.float32, device="cuda")
    lp = torch.empty((B, n, Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(hd.hd_attn_decode_workspace(B, n, T, Hq, Hkv, D, "cross"), dtype=torch.uint8, device="cuda")
    ms_dec = time_fn(lambda: hd.hd_attn_decode_shard(q, kc, vc, ctx, R, 0, out=op, lse=lp, workspace=ws))
    dec_bytes = 2 * kc.numel() * 2 + q.numel() * 2 + op.numel() * 4
    o_all = op.unsqueeze(0).expand(R, -1, -1, -1, -1).contiguous()
    l_all = lp.unsqueeze(0).expand(R, -1, -1, -1).contiguous()
    out = torch.empty((B, n, Hq, D), dtype=torch.bfloat16, device="cuda")
    ms_cb = time_fn(lambda: hd.hd_attn_combine(o_all, l_all, out=out))
    # The fused merge of rank 0's own stream rows from R partials read through
    # their own pointers (here R local copies; on R GPUs, peers' memory).
    o_list = [op] + [op.clone() for _ in range(R - 1)]
    l_list = [lp] + [lp.clone() for _ in range(R - 1)]
    out_loc = torch.empty((B, n // R, Hq, D), dtype=torch.bfloat16, device="cuda")
    ms_cs = time_fn(lambda: hd.hd_attn_combine_streams(o_list, l_list, n, R, 0, out=out_loc))
    res[f"sp_R{R}_rank0_cross_decode"] = {
        "partial_ms": round(ms_dec, 3), "partial_GB/s": round(dec_bytes / (ms_dec * 1e-3) / 1e9, 1),
        "partial_frac_hbm": round(dec_bytes / (ms_dec * 1e-3) / 1e9 / peaks["hbm"], 4),
        "merge_ms": round(ms_cb, 4), "merge_own_rows_ms": round(ms_cs, 4),
        "allgather_bytes_in_per_rank": (R - 1) * (q.numel() // R * 2 + op.numel() * 4 + lp.numel() * 4)}
    del q, kc, vc, op, lp, ws, o_all, l_all, out, o_list, l_list, out_loc
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------ CPU oracle arm

def oracle_sample_rate(wl, budget_s, seed=5):
    """Run the float64 oracle on host cores on sampled output rows of the
    workload for about ``budget_s`` seconds; returns (units/s, unit, sample
    description, threads)."""
    import numpy as np

    import oracle
    from stream_sequence_attention_b200 import synth

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    cfg = WORKLOADS[wl]
    g = synth.rng(seed)
    if wl == "decode":
        n, T, D = cfg["n"], cfg["T"], cfg["D"]
        G = cfg["Hq"] // cfg["Hkv"]
        # one KV head of one sequence, host-drawn at full context length
        q = synth.normal((1, n, G, D), seed + 1, dtype="bf16")
        kc = synth.normal((1, n, T, 1, D), seed + 2, dtype="bf16")
        vc = synth.normal((1, n, T, 1, D), seed + 3, dtype="bf16")
        t0 = time.perf_counter()
        rows = 0
        while time.perf_counter() - t0 < budget_s:
            for mode in ("intra", "cross"):
                oracle.decode_rows(q, kc, vc, np.array([T]), n, mode, [(0, int(g.integers(n)), int(g.integers(G)))])
                rows += 1
        dt = time.perf_counter() - t0
        # bytes each row's arithmetic reads from the cache: intra T, cross n*T entries of K and V
        per_row_bytes = 0.5 * (2 * T * D * 2) + 0.5 * (2 * n * T * D * 2)
        return rows * per_row_bytes / dt / 1e9, "GB/s", f"{rows} decode rows (one KV head, ctx {T}), {dt:.1f} s", threads
    if cfg.get("rope"):
        n, L, D, H = cfg["n"], cfg["L"], cfg["D"], cfg["Hq"] + cfg["Hkv"]
        P = n * L
        x = synth.normal((1, 256, H, D), seed + 1, dtype="bf16")
        t0 = time.perf_counter()
        rows = 0
        while time.perf_counter() - t0 < budget_s:
            oracle.rope(x, D, 10000.0, pos_base=int(g.integers(P - 256)))
            rows += 256
        dt = time.perf_counter() - t0
        # bytes the GPU call moves for these rows: q and k read and written once (bf16)
        return (rows * H * D * 2 * 2 / dt / 1e9, "GB/s",
                f"{rows} positions x {H} heads in blocks of 256 consecutive positions, {dt:.1f} s", threads)
    n, L, D, mode, W = cfg["n"], cfg["L"], cfg["D"], cfg["mode"], cfg["W"]
    P = n * L
    q = synth.normal((1, P, 1, D), seed + 1, dtype="bf16")
    k = synth.normal((1, P, 1, D), seed + 2, dtype="bf16")
    v = synth.normal((1, P, 1, D), seed + 3, dtype="bf16")
    pk = np.arange(P)
    if cfg.get("bwd"):
        dO = synth.normal((1, P, 1, D), seed + 4, dtype="bf16")
        t0 = time.perf_counter()
        rows, pairs = 0, 0
        while time.perf_counter() - t0 < budget_s:
            p = int(g.integers(P))
            keys = oracle.attn_bwd_query_rows(q, k, v, dO, n, mode, [(0, 0, p)], W, D ** -0.5)[0][0]
            pairs += len(keys)
            rows += 1
        dt = time.perf_counter() - t0
        return (pairs * 10 * D / dt / 1e12, "TFLOP/s",
                f"{rows} uniformly sampled query rows of one (batch, head): each row's dQ and its dK/dV terms, "
                f"{dt:.1f} s", threads)
    t0 = time.perf_counter()
    rows, pairs = 0, 0
    while time.perf_counter() - t0 < budget_s:
        p = int(g.integers(P))
        oracle.attn_rows(q, k, v, n, mode, [(0, 0, p)], W, D ** -0.5)
        pairs += int(np.count_nonzero(oracle.visible(p, pk, n, mode, W)))
        rows += 1
    dt = time.perf_counter() - t0
    return (pairs * 4 * D / dt / 1e12, "TFLOP/s",
            f"{rows} uniformly sampled output rows of one (batch, head), {dt:.1f} s", threads)


def run_reference(args):
    wl = args.workload
    K = args.steps if args.steps is not None else 10
    W = args.warmup if args.warmup is not None else 3
    budget_total = 90.0
    per_step = max(0.05, budget_total / max(1, K + W))
    for _ in range(W):
        oracle_sample_rate(wl, per_step, seed=11)
    vals = []
    t0 = time.perf_counter()
    for i in range(K):
        v, unit, sample, threads = oracle_sample_rate(wl, per_step, seed=100 + i)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    if wl == "decode":
        metric = "decode GB/s vs HBM (intra+cross, B=64 n=4 ctx=32768)"
    elif WORKLOADS[wl].get("bwd"):
        metric = "useful attn backward TFLOP/s at n=4 (%s)" % WORKLOADS[wl]["mode"]
    elif WORKLOADS[wl].get("rope"):
        metric = "RoPE GB/s vs HBM (q and k in place, n=4 L=4096 B=2 32q/8kv)"
    else:
        metric = "useful attn TFLOP/s at n=4 (%s)" % WORKLOADS[wl]["mode"]
    return {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": K,
        "warmup": W, "ms_per_step": round(1000 * wall / K, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded host draws)",
        "config": {"workload": NAMES[wl], "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": f"per step: {sample}"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as td

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    out, work, peaks = run_ours(args, rank, world, dist)
    import torch

    del work
    torch.cuda.empty_cache()
    if args.profile:
        if rank == 0:
            print(json.dumps(out), flush=True)
        return
    if rank == 0:
        # The side measurements are single-GPU figures (the N = 1 run reports
        # them); with several ranks they would only hold the other GPUs idle.
        if not args.no_extras and args.workload != "decode" and world == 1:
            out["also"] = extras(torch, peaks, rank)
        v, unit, sample, threads = oracle_sample_rate(args.workload, 15.0)
        out["cpu_baseline"] = {"value": v, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample}
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
