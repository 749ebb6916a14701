"""The fused peer-gather cross-stream prefill through real CUDA IPC: two
processes on one GPU, each owning one rank's K/V shard buffers (PeerShards),
exchanging IPC handles over a gloo group, and each running
hd_attn_fwd_peer_gather that reads the other process's buffers through the
mapped addresses.  The processes take turns on the GPU (a host barrier
between their launches), so no kernel ever runs beside the other process's;
no kernel waits on anything outside its own launch.  Three layers cycle the
two buffer pairs.  Then the cross-stream decode with the partials' exchange
fused into the merge (PeerDecode): three steps cycle its two buffer sets.
Each rank's rows are checked against the float64 oracle."""

import json
import os
import socket
import subprocess
import sys

import pytest

from tests.gpu_util import TOL_BF16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CHILD = r"""
import datetime, json, sys
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, ROOT)
import oracle
from stream_sequence_attention_b200 import hd, synth, stream_parallel as sp
from tests.gpu_util import dev, max_abs, to_f64
rank, port = int(sys.argv[1]), sys.argv[2]
R = 2
torch.cuda.set_device(0)
dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=R,
                        timeout=datetime.timedelta(seconds=120))
n, B, L, Hq, Hkv, D = 4, 2, 150, 4, 2, 128
nl = n // R

def shard(x):
    P = x.shape[1]
    return np.ascontiguousarray(x.reshape((B, P // n, nl, R) + x.shape[2:])[:, :, :, rank].reshape(
        (B, (P // n) * nl) + x.shape[2:]))

view = sp.StreamParallel(n)
ps = sp.PeerShards(view, B, L, Hkv, D)
errs = []
for layer in range(3):
    q = synth.normal((B, n * L, Hq, D), 1401 + 10 * layer, dtype="bf16")
    k = synth.normal((B, n * L, Hkv, D), 1402 + 10 * layer, dtype="bf16")
    v = synth.normal((B, n * L, Hkv, D), 1403 + 10 * layer, dtype="bf16")
    ps.stage(dev(shard(k), "bf16"), dev(shard(v), "bf16"))
    ps.fence()
    st = hd.new_status()
    for turn in range(R):
        if turn == rank:
            o = ps.attend(dev(shard(q), "bf16"), out_dtype=torch.float32, dev_status=st)
            torch.cuda.synchronize()
        dist.barrier()
    ro, _ = oracle.attn(q, k, v, n, "cross")
    errs.append([int(st.item()), max_abs(to_f64(o), shard(ro))])
ps.close()
# Cross-stream decode: each rank's partial over its cache streams, merged
# for its own stream rows from both processes' exported partials.
Lmax, T, Hd = 300, 257, 8
pdec = sp.PeerDecode(view, B, Hd, D)
for step in range(3):
    qd = synth.normal((B, n, Hd, D), 1501 + 10 * step, dtype="bf16")
    kc = synth.normal((B, n, Lmax, Hkv, D), 1502 + 10 * step, dtype="bf16")
    vc = synth.normal((B, n, Lmax, Hkv, D), 1503 + 10 * step, dtype="bf16")
    ctx = np.array([T, T // 3], dtype=np.int32)
    st = hd.new_status()
    for turn in range(R):
        if turn == rank:
            pdec.partial(dev(qd, "bf16"), dev(kc[:, rank::R].copy(), "bf16"), dev(vc[:, rank::R].copy(), "bf16"),
                         dev(ctx, "i32"), dev_status=st)
            torch.cuda.synchronize()
        dist.barrier()
    pdec.fence()
    for turn in range(R):
        if turn == rank:
            od = pdec.merge(out_dtype=torch.float32)
            torch.cuda.synchronize()
        dist.barrier()
    ref, _ = oracle.decode(qd, kc, vc, ctx, n, "cross")
    errs.append([int(st.item()), max_abs(to_f64(od), ref[:, rank::R])])
pdec.close()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "errs": errs}))
"""


def test_peer_gather_through_ipc_two_processes():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = str(s.getsockname()[1])
    code = CHILD.replace("ROOT", repr(ROOT))
    procs = [subprocess.Popen([sys.executable, "-c", code, str(r), port], stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    try:
        for p in procs:
            out, err = p.communicate(timeout=300)
            assert p.returncode == 0, err[-3000:]
            outs.append(json.loads(out.strip().splitlines()[-1]))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    for o in outs:
        for status, err in o["errs"]:
            assert status == 0
            assert err <= TOL_BF16, (o["rank"], err)
