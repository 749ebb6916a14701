"""The bounded-wait failure path of the tcgen05 attention kernel, on the GPU,
without a fault: with HD_TEST_STALL_FIRST_S=1 the MMA warp of CTA 0 never
signals its S tiles (a flag nothing sets), so the softmax wait runs out after
its one-second limit.  The kernel must return with HD_ERR_TIMEOUT in the
status word and leave the context usable for the next launches.  Runs in a
child process because the hook is read once per process."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu

CHILD = r"""
import json, sys, torch
sys.path.insert(0, ROOT)
from stream_sequence_attention_b200 import build, hd, synth
build.build(); hd.lib()
q = synth.normal_device((1, 2 * 256, 4, 128), 1)
k = synth.normal_device((1, 2 * 256, 2, 128), 2)
v = synth.normal_device((1, 2 * 256, 2, 128), 3)
st = hd.new_status()
hd.hd_attn_fwd(q, k, v, 2, "intra", dev_status=st)
torch.cuda.synchronize()
status = int(st.item())
# the context is still usable: other kernels run and give exact results
h = synth.normal_device((1, 2 * 64, 16), 4)
g = hd.hd_final_stream_gather(h, 2)
torch.cuda.synchronize()
usable = bool(torch.equal(g, h[:, 1::2]))
print(json.dumps({"status": status, "usable": usable}))
"""


def test_attention_wait_times_out_cleanly():
    env = dict(os.environ, HD_TEST_STALL_FIRST_S="1")
    code = CHILD.replace("ROOT", repr(ROOT))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["status"] == 4  # HD_ERR_TIMEOUT
    assert out["usable"]


CHILD_BWD = r"""
import json, sys, torch
sys.path.insert(0, ROOT)
from stream_sequence_attention_b200 import build, hd, synth
build.build(); hd.lib()
q = synth.normal_device((1, 2 * 256, 4, 128), 1)
k = synth.normal_device((1, 2 * 256, 2, 128), 2)
v = synth.normal_device((1, 2 * 256, 2, 128), 3)
dO = synth.normal_device((1, 2 * 256, 4, 128), 4)
o, lse = hd.hd_attn_fwd(q, k, v, 2, "intra", lse=True)
st = hd.new_status()
hd.hd_attn_bwd(q, k, v, o, dO, lse, 2, "intra", dev_status=st)
torch.cuda.synchronize()
status = int(st.item())
h = synth.normal_device((1, 2 * 64, 16), 5)
g = hd.hd_final_stream_gather(h, 2)
torch.cuda.synchronize()
print(json.dumps({"status": status, "usable": bool(torch.equal(g, h[:, 1::2]))}))
"""

CHILD_DEC = r"""
import json, sys, torch
sys.path.insert(0, ROOT)
from stream_sequence_attention_b200 import build, hd, synth
build.build(); hd.lib()
q = synth.normal_device((2, 4, 16, 128), 1)
kc = synth.normal_device((2, 4, 256, 2, 128), 2)
vc = synth.normal_device((2, 4, 256, 2, 128), 3)
ctx = torch.full((2,), 256, dtype=torch.int32, device="cuda")
st = hd.new_status()
hd.hd_attn_decode(q, kc, vc, ctx, "cross", dev_status=st)
torch.cuda.synchronize()
status = int(st.item())
h = synth.normal_device((1, 2 * 64, 16), 5)
g = hd.hd_final_stream_gather(h, 2)
torch.cuda.synchronize()
print(json.dumps({"status": status, "usable": bool(torch.equal(g, h[:, 1::2]))}))
"""


CHILD_GATHER = r"""
import json, sys, torch
sys.path.insert(0, ROOT)
from stream_sequence_attention_b200 import build, hd, synth
build.build(); hd.lib()
n, R, r, L = 4, 2, 0, 300
q = synth.normal_device((1, 2 * L, 4, 128), 1)
ks = [synth.normal_device((1, 2 * L, 2, 128), 2 + i) for i in range(R)]
vs = [synth.normal_device((1, 2 * L, 2, 128), 4 + i) for i in range(R)]
kd = [torch.empty_like(ks[0]) for _ in range(R)]
vd = [torch.empty_like(vs[0]) for _ in range(R)]
st = hd.new_status()
hd.hd_attn_fwd_peer_gather(q, ks, vs, kd, vd, n, R, r, dev_status=st)
torch.cuda.synchronize()
status = int(st.item())
h = synth.normal_device((1, 2 * 64, 16), 5)
g = hd.hd_final_stream_gather(h, 2)
torch.cuda.synchronize()
print(json.dumps({"status": status, "usable": bool(torch.equal(g, h[:, 1::2]))}))
"""

CHILDREN = {"bwd": CHILD_BWD, "dec": CHILD_DEC, "dec_intra": CHILD_DEC.replace('"cross"', '"intra"'),
            "gather": CHILD_GATHER}


@pytest.mark.parametrize("var,child", [("HD_TEST_STALL_BWD", "bwd"), ("HD_TEST_STALL_DECODE", "dec"),
                                       ("HD_TEST_STALL_DECODE", "dec_intra"), ("HD_TEST_STALL_GATHER", "gather")])
def test_backward_decode_and_gather_waits_time_out_cleanly(var, child):
    """The same bounded-wait path in the dK/dV backward kernel (its MMA warp of
    CTA 0 never signals S), in both decode kernels (cross mode: the tcgen05
    kernel; intra mode: the warp-MMA kernel; the producer of the first CTA
    issues no loads), and in the fused peer-gather attention (CTA 0 never
    publishes its first copied piece, so the first key tile never becomes
    ready for any CTA)."""
    env = dict(os.environ, **{var: "1"})
    code = CHILDREN[child].replace("ROOT", repr(ROOT))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["status"] == 4  # HD_ERR_TIMEOUT
    assert out["usable"]
