"""Host-side checks of the C ABI: the library loads without a GPU, exports
every function ``include/hd.h`` declares, and rejects bad arguments before
touching the device."""

import ctypes
import os
import re

import pytest

from stream_sequence_attention_b200 import build as hd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hd.h")


@pytest.fixture(scope="module")
def L():
    hd_build.build()
    from stream_sequence_attention_b200 import hd
    return hd.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(hd_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("hd_expand_embed", "hd_attn_fwd", "hd_attn_decode", "hd_attn_decode_workspace",
                 "hd_final_stream_gather", "hd_status_string", "hd_version"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_binding_names_match_header():
    from stream_sequence_attention_b200 import hd
    assert sorted(hd.EXPORTS) == declared_functions()


def test_status_strings_and_version(L):
    from stream_sequence_attention_b200 import hd
    assert hd.status_string(0) == "HD_OK"
    assert hd.status_string(4) == "HD_ERR_TIMEOUT"
    assert hd.status_string(5) == "HD_ERR_BAD_TOKEN"
    assert hd.status_string(99) == "HD_ERR_UNKNOWN"
    assert hd.version() >= 100


def test_bad_arguments_rejected_on_host(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)  # never dereferenced: every call below fails validation first
    # n = 0
    assert L.hd_expand_embed(fake, fake, fake, 1, 4, 0, 10, 8, hd.HD_BF16, None, None) == hd.HD_ERR_INVALID_ARG
    # ids not int32-aligned (a 4-byte offset is allowed; 2 bytes is not)
    assert L.hd_expand_embed(fake, vp(0x10002), fake, 1, 4, 2, 10, 8, hd.HD_BF16, None, None) \
        == hd.HD_ERR_INVALID_ARG
    # row bytes not a multiple of 16 (d = 4 bf16)
    assert L.hd_expand_embed(fake, fake, fake, 1, 4, 2, 10, 4, hd.HD_BF16, None, None) == hd.HD_ERR_INVALID_ARG
    # Hq % Hkv != 0
    assert L.hd_attn_fwd(fake, fake, fake, fake, None, 1, 8, 2, 3, 2, 64, 0, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    # unsupported head dim
    assert L.hd_attn_fwd(fake, fake, fake, fake, None, 1, 8, 2, 2, 2, 96, 0, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_UNSUPPORTED
    # L = 0 and bad mode
    assert L.hd_attn_fwd(fake, fake, fake, fake, None, 1, 0, 2, 2, 2, 64, 0, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_fwd(fake, fake, fake, fake, None, 1, 8, 2, 2, 2, 64, 7, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    # misaligned q
    assert L.hd_attn_fwd(vp(0x10008), fake, fake, fake, None, 1, 8, 2, 2, 2, 64, 0, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    # decode: only bf16 / D = 128
    assert L.hd_attn_decode(fake, fake, fake, fake, fake, None, 1, 2, 8, 2, 2, 64, 0, 0, 0.1, 1, 1,
                            fake, 1 << 20, None, None) == hd.HD_ERR_UNSUPPORTED
    assert L.hd_attn_decode(fake, fake, fake, fake, fake, None, 1, 2, 8, 2, 2, 128, 0, 0, 0.1, 0, 1,
                            fake, 1 << 20, None, None) == hd.HD_ERR_UNSUPPORTED
    # gather: negative sizes
    assert L.hd_final_stream_gather(fake, fake, -1, 4, 2, 8, hd.HD_F32, None) == hd.HD_ERR_INVALID_ARG
    # empty work is a no-op that succeeds without a device
    assert L.hd_final_stream_gather(None, None, 0, 4, 2, 8, hd.HD_F32, None) == hd.HD_OK
    assert L.hd_expand_embed(None, None, None, 0, 4, 2, 10, 8, hd.HD_F32, None, None) == hd.HD_OK


def test_bwd_workspace_and_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    # two floats per (b, head, stream, token), tokens padded to 128 per stream
    assert L.hd_attn_bwd_workspace(2, 100, 4, 8, hd.HD_INTRA) == 2 * 8 * 4 * 128 * 8
    assert L.hd_attn_bwd_workspace(2, 100, 4, 8, hd.HD_CROSS) == 2 * 8 * 1 * 512 * 8
    assert L.hd_attn_bwd_workspace(0, 100, 4, 8, hd.HD_CROSS) == 0
    assert L.hd_attn_bwd_workspace(1, 8, 2, 2, 7) == 0

    def bwd(*, q=fake, lse=fake, ws=fake, ws_bytes=1 << 20, Hq=2, Hkv=2, D=64, mode=0, scale=0.1, dt=1, B=1):
        return L.hd_attn_bwd(q, fake, fake, fake, fake, lse, fake, fake, fake, B, 8, 2, Hq, Hkv, D, mode, 0, scale,
                             dt, ws, ws_bytes, None, None)
    assert bwd(Hq=3) == hd.HD_ERR_INVALID_ARG
    assert bwd(D=96) == hd.HD_ERR_UNSUPPORTED
    assert bwd(mode=5) == hd.HD_ERR_INVALID_ARG
    assert bwd(scale=-1.0) == hd.HD_ERR_INVALID_ARG
    assert bwd(lse=None) == hd.HD_ERR_INVALID_ARG
    assert bwd(ws=None) == hd.HD_ERR_INVALID_ARG
    assert bwd(ws=vp(0x10010)) == hd.HD_ERR_INVALID_ARG  # workspace not 256-byte aligned
    assert bwd(q=vp(0x10008)) == hd.HD_ERR_INVALID_ARG
    assert bwd(ws_bytes=16) == hd.HD_ERR_INVALID_ARG
    assert bwd(B=0) == hd.HD_OK


def test_attn_fwd_rope_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)  # never dereferenced: every call below fails validation first
    args = lambda rot, layout, dt: (fake, fake, fake, fake, None, 1, 300, 4, 4, 2, 128, 0, 0, 0.1,  # noqa
                                    rot, 10000.0, layout, dt, dt, None, None)
    # rot_dim not a multiple of 16 in the rotate-half form, or above D
    assert L.hd_attn_fwd_rope(*args(40, hd.HD_ROPE_HALF, hd.HD_BF16)) == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_fwd_rope(*args(256, hd.HD_ROPE_HALF, hd.HD_BF16)) == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_fwd_rope(*args(12, hd.HD_ROPE_INTERLEAVED, hd.HD_BF16)) == hd.HD_ERR_INVALID_ARG
    # bad layout; float32 inputs are not taken (the rotation runs in the tensor-core kernel)
    assert L.hd_attn_fwd_rope(*args(128, 7, hd.HD_BF16)) == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_fwd_rope(*args(128, hd.HD_ROPE_HALF, hd.HD_F32)) == hd.HD_ERR_UNSUPPORTED


def test_rope_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)

    def rope(*, q=fake, k=fake, D=128, rot=128, base=10000.0, layout=0, dt=1, B=1, P=4, pos_base=0):
        return L.hd_rope(q, k, None, B, P, 4, 2, D, rot, base, pos_base, 0, layout, dt, None)
    assert rope(rot=6) == hd.HD_ERR_INVALID_ARG          # not a multiple of 8
    assert rope(rot=136) == hd.HD_ERR_INVALID_ARG        # > D
    assert rope(D=260, rot=256) == hd.HD_ERR_INVALID_ARG  # D > 256
    assert rope(base=0.0) == hd.HD_ERR_INVALID_ARG
    assert rope(base=float("nan")) == hd.HD_ERR_INVALID_ARG
    assert rope(layout=3) == hd.HD_ERR_INVALID_ARG
    assert rope(q=vp(0x10008)) == hd.HD_ERR_INVALID_ARG
    assert rope(pos_base=1 << 40) == hd.HD_ERR_INVALID_ARG
    assert rope(B=0) == hd.HD_OK
    assert rope(q=None, k=None) == hd.HD_OK


def test_stream_parallel_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    # R must divide n, 0 <= r < R
    assert L.hd_attn_fwd_shard(fake, fake, fake, fake, None, 1, 8, 4, 3, 0, 2, 2, 128, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_fwd_shard(fake, fake, fake, fake, None, 1, 8, 4, 2, 2, 2, 2, 128, 0, 0.1, 1, 1, None, None) \
        == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_decode_shard(fake, fake, fake, fake, fake, fake, 1, 4, 3, 0, 8, 2, 2, 128, 0, 0.1, 1, 0,
                                  fake, 1 << 20, None, None) == hd.HD_ERR_INVALID_ARG
    # the decode partial needs its lse
    assert L.hd_attn_decode_shard(fake, fake, fake, fake, fake, None, 1, 4, 2, 0, 8, 2, 2, 128, 0, 0.1, 1, 0,
                                  fake, 1 << 20, None, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_stream_interleave(fake, fake, 3, 1, 4, 4, 8, hd.HD_BF16, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_stream_interleave(fake, fake, 2, 1, 4, 4, 4, hd.HD_BF16, None) == hd.HD_ERR_INVALID_ARG  # 8-byte rows
    assert L.hd_stream_interleave(None, None, 2, 0, 4, 4, 8, hd.HD_BF16, None) == hd.HD_OK
    assert L.hd_attn_combine(fake, fake, fake, None, 2, 10, 6, 0, 0, None) == hd.HD_ERR_INVALID_ARG  # D % 4
    assert L.hd_attn_combine(fake, fake, fake, None, 0, 10, 8, 0, 0, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_attn_combine(None, None, None, None, 2, 0, 8, 0, 0, None) == hd.HD_OK


def test_rank_shard_calls_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    arr = lambda *p: (vp * len(p))(*p)  # noqa: E731
    k4, v4 = arr(fake, fake, fake, fake), arr(fake, fake, fake, fake)

    def parts(k, v, B=1, L_=8, n=4, R=4, r=0, in_dt=hd.HD_BF16):
        return L.hd_attn_fwd_parts(fake, k, v, fake, None, B, L_, n, R, r, 2, 2, 128, 0, 0.1, in_dt, hd.HD_BF16,
                                   None, None)

    assert parts(k4, v4, B=0) == hd.HD_OK
    assert parts(k4, v4, n=6, R=3) == hd.HD_ERR_INVALID_ARG            # n must divide 128
    assert parts(k4, v4, R=3) == hd.HD_ERR_INVALID_ARG                 # R must divide n
    assert parts(k4, v4, r=4) == hd.HD_ERR_INVALID_ARG
    assert parts(k4, v4, n=16, R=16) == hd.HD_ERR_INVALID_ARG          # more ranks than supported
    assert parts(k4, v4, in_dt=hd.HD_F32) == hd.HD_ERR_UNSUPPORTED     # tensor-core path only
    assert parts(arr(fake, None, fake, fake), v4) == hd.HD_ERR_INVALID_ARG
    assert parts(k4, arr(fake, fake, vp(0x10008), fake)) == hd.HD_ERR_INVALID_ARG  # 16-byte alignment
    assert parts(None, v4) == hd.HD_ERR_INVALID_ARG
    # one flag word per (sequence, 128-key tile)
    assert L.hd_attn_peer_flags_bytes(2, 4096, 4) == 2 * 128 * 8
    assert L.hd_attn_peer_flags_bytes(1, 150, 4) == 5 * 8
    assert L.hd_attn_peer_flags_bytes(-1, 150, 4) == 0

    def gather(kd, vd, flags=fake, nbytes=1 << 20, R=4):
        return L.hd_attn_fwd_peer_gather(fake, k4, v4, kd, vd, flags, nbytes, fake, None, 1, 8, 4, R, 0, 2, 2, 128,
                                         0, 0.1, hd.HD_BF16, hd.HD_BF16, None, None)

    assert gather(k4, v4, nbytes=7) == hd.HD_ERR_INVALID_ARG           # flags smaller than one word per tile
    assert gather(k4, v4, flags=None) == hd.HD_ERR_INVALID_ARG
    assert gather(k4, v4, flags=vp(0x10004)) == hd.HD_ERR_INVALID_ARG  # 8-byte alignment
    assert gather(None, v4) == hd.HD_ERR_INVALID_ARG
    assert gather(arr(None, fake, None, fake), v4) == hd.HD_ERR_INVALID_ARG  # a peer's slot missing
    # IPC helpers reject null arguments without touching CUDA
    off = ctypes.c_size_t(0)
    assert L.hd_ipc_export(None, ctypes.create_string_buffer(64), ctypes.byref(off)) == hd.HD_ERR_INVALID_ARG
    assert L.hd_ipc_open(None, None) == hd.HD_ERR_INVALID_ARG
    assert L.hd_ipc_close(None) == hd.HD_ERR_INVALID_ARG


def test_combine_streams_bad_arguments(L):
    from stream_sequence_attention_b200 import hd
    vp = ctypes.c_void_p
    fake = vp(0x10000)
    arr = lambda *p: (vp * len(p))(*p)  # noqa: E731
    o2, l2 = arr(fake, fake), arr(fake, fake)

    def call(o, l, B=2, n=4, Hq=8, D=128, R=2, r=0, out=fake):
        return L.hd_attn_combine_streams(o, l, out, None, B, n, Hq, D, R, r, hd.HD_F32, hd.HD_BF16, None)

    assert call(o2, l2, B=0) == hd.HD_OK
    assert call(o2, l2, R=3) == hd.HD_ERR_INVALID_ARG          # R must divide n
    assert call(o2, l2, r=2) == hd.HD_ERR_INVALID_ARG
    assert call(o2, l2, D=6) == hd.HD_ERR_INVALID_ARG          # D % 4
    assert call(arr(fake, None), l2) == hd.HD_ERR_INVALID_ARG
    assert call(o2, arr(fake, vp(0x10002))) == hd.HD_ERR_INVALID_ARG  # lse alignment
    assert call(o2, l2, out=vp(0x10008)) == hd.HD_ERR_INVALID_ARG     # 16-byte output
    assert call(None, l2) == hd.HD_ERR_INVALID_ARG
