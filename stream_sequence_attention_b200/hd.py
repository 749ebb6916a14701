"""Python binding of the C ABI in ``include/hd.h`` (ctypes, marshalling only).

Each function takes torch tensors that already live on the current CUDA
device, checks dtype / shape / contiguity, and passes raw pointers, sizes and
the current CUDA stream to the library.  Every step of the computation runs in
the library's kernels; there is no fallback: if ``libhd.so`` is missing or a
call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhd.so")

HD_OK, HD_ERR_INVALID_ARG, HD_ERR_UNSUPPORTED, HD_ERR_CUDA, HD_ERR_TIMEOUT, HD_ERR_BAD_TOKEN = range(6)
HD_F32, HD_BF16 = 0, 1
HD_INTRA, HD_CROSS = 0, 1
HD_ROPE_HALF, HD_ROPE_INTERLEAVED = 0, 1

_MODES = {"intra": HD_INTRA, "cross": HD_CROSS, HD_INTRA: HD_INTRA, HD_CROSS: HD_CROSS}

EXPORTS = (
    "hd_expand_embed",
    "hd_attn_fwd",
    "hd_attn_fwd_final_stream",
    "hd_attn_bwd",
    "hd_attn_bwd_final_stream",
    "hd_attn_bwd_workspace",
    "hd_attn_decode",
    "hd_attn_decode_workspace",
    "hd_attn_decode_noalloc",
    "hd_attn_decode_shard",
    "hd_attn_fwd_shard",
    "hd_attn_combine_streams",
    "hd_attn_fwd_parts",
    "hd_attn_fwd_peer_gather",
    "hd_attn_peer_flags_bytes",
    "hd_ipc_export",
    "hd_ipc_open",
    "hd_ipc_close",
    "hd_stream_interleave",
    "hd_attn_combine",
    "hd_final_stream_gather",
    "hd_rope",
    "hd_attn_fwd_rope",
    "hd_status_string",
    "hd_version",
)


class HDError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhd.so (built in-tree by ``stream_sequence_attention_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m stream_sequence_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.hd_expand_embed.argtypes = [vp, vp, vp, i32, i32, i32, i64, i32, i32, vp, vp]
        L.hd_expand_embed.restype = i32
        L.hd_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32, vp, vp]
        L.hd_attn_fwd.restype = i32
        L.hd_attn_fwd_final_stream.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                               i32, vp, vp]
        L.hd_attn_fwd_final_stream.restype = i32
        L.hd_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                  i32, vp, sz, vp, vp]
        L.hd_attn_bwd.restype = i32
        L.hd_attn_bwd_final_stream.argtypes = L.hd_attn_bwd.argtypes
        L.hd_attn_bwd_final_stream.restype = i32
        L.hd_attn_bwd_workspace.argtypes = [i32, i32, i32, i32, i32]
        L.hd_attn_bwd_workspace.restype = sz
        L.hd_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                     vp, sz, vp, vp]
        L.hd_attn_decode.restype = i32
        L.hd_attn_decode_workspace.argtypes = [i32, i32, i32, i32, i32, i32, i32]
        L.hd_attn_decode_workspace.restype = sz
        L.hd_attn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                             i32, i32, vp, vp]
        L.hd_attn_decode_noalloc.restype = i32
        L.hd_final_stream_gather.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp]
        L.hd_final_stream_gather.restype = i32
        L.hd_attn_decode_shard.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                           i32, i32, vp, sz, vp, vp]
        L.hd_attn_decode_shard.restype = i32
        L.hd_attn_fwd_shard.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                        vp, vp]
        L.hd_attn_fwd_shard.restype = i32
        L.hd_attn_combine_streams.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp]
        L.hd_attn_combine_streams.restype = i32
        L.hd_attn_fwd_parts.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                        vp, vp]
        L.hd_attn_fwd_parts.restype = i32
        L.hd_attn_fwd_peer_gather.argtypes = [vp, vp, vp, vp, vp, vp, sz, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                              i32, i32, f32, i32, i32, vp, vp]
        L.hd_attn_fwd_peer_gather.restype = i32
        L.hd_attn_peer_flags_bytes.argtypes = [i32, i32, i32]
        L.hd_attn_peer_flags_bytes.restype = sz
        L.hd_ipc_export.argtypes = [vp, vp, ctypes.POINTER(sz)]
        L.hd_ipc_export.restype = i32
        L.hd_ipc_open.argtypes = [vp, ctypes.POINTER(vp)]
        L.hd_ipc_open.restype = i32
        L.hd_ipc_close.argtypes = [vp]
        L.hd_ipc_close.restype = i32
        L.hd_attn_fwd_rope.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                       ctypes.c_double, i32, i32, i32, vp, vp]
        L.hd_attn_fwd_rope.restype = i32
        L.hd_stream_interleave.argtypes = [vp, vp, i32, i32, i32, i32, i64, i32, vp]
        L.hd_stream_interleave.restype = i32
        L.hd_attn_combine.argtypes = [vp, vp, vp, vp, i32, i64, i32, i32, i32, vp]
        L.hd_attn_combine.restype = i32
        L.hd_rope.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_double, i64, i64, i32, i32, vp]
        L.hd_rope.restype = i32
        L.hd_status_string.argtypes = [i32]
        L.hd_status_string.restype = ctypes.c_char_p
        L.hd_version.argtypes = []
        L.hd_version.restype = i32
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().hd_status_string(int(code)).decode()


def version() -> int:
    return lib().hd_version()


def _check(fn, code):
    if code != HD_OK:
        raise HDError(fn, code)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HD_BF16
    if t.dtype == torch.float32:
        return HD_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word for the ``dev_status`` arguments."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def hd_expand_embed(tables: torch.Tensor, ids: torch.Tensor, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """tables [n, V, d], ids [B, L] int32 -> out [B, n*L, d]."""
    _need(tables, "tables")
    _need(ids, "ids")
    n, V, d = tables.shape
    B, L = ids.shape
    if ids.dtype != torch.int32:
        raise TypeError("ids must be int32")
    if out is None:
        out = torch.empty((B, n * L, d), dtype=tables.dtype, device=tables.device)
    _need(out, "out")
    if out.shape != (B, n * L, d) or out.dtype != tables.dtype:
        raise ValueError("out has the wrong shape or dtype")
    _check("hd_expand_embed", lib().hd_expand_embed(
        _ptr(tables), _ptr(ids), _ptr(out), B, L, n, V, d, _dt(tables), _ptr(dev_status), _stream(stream)))
    return out


def hd_final_stream_gather(h: torch.Tensor, n: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h [B, n*L, d] -> out [B, L, d] (rows of the final stream)."""
    _need(h, "h")
    B, P, d = h.shape
    if P % n:
        raise ValueError("sequence length is not a multiple of n")
    L = P // n
    if out is None:
        out = torch.empty((B, L, d), dtype=h.dtype, device=h.device)
    _need(out, "out")
    if out.shape != (B, L, d) or out.dtype != h.dtype:
        raise ValueError("out has the wrong shape or dtype")
    _check("hd_final_stream_gather", lib().hd_final_stream_gather(
        _ptr(h), _ptr(out), B, L, n, d, _dt(h), _stream(stream)))
    return out


_ROPE_LAYOUTS = {"half": HD_ROPE_HALF, "interleaved": HD_ROPE_INTERLEAVED}


def hd_rope(q: torch.Tensor | None, k: torch.Tensor | None = None, rot_dim: int | None = None,
            base: float = 10000.0, pos_base: int = 0, pos_mult: int = 0, pos0: torch.Tensor | None = None,
            layout: str = "half", stream=None):
    """Rotary embedding in place on q [B, P, Hq, D] and k [B, P, Hkv, D]
    (either may be None): row r of sequence b at position
    pos_base + pos_mult * pos0[b] + r.  Returns (q, k)."""
    ref = q if q is not None else k
    if ref is None:
        raise ValueError("q or k is required")
    for t, nm in ((q, "q"), (k, "k"), (pos0, "pos0")):
        if t is not None:
            _need(t, nm)
    B, P, _, D = ref.shape
    Hq = q.shape[2] if q is not None else 0
    Hkv = k.shape[2] if k is not None else 0
    if q is not None and k is not None and (k.shape[:2] != q.shape[:2] or k.shape[3] != D or k.dtype != q.dtype):
        raise ValueError("q and k disagree")
    if pos0 is not None and (pos0.dtype != torch.int32 or pos0.shape != (B,)):
        raise ValueError("pos0 must be int32 [B]")
    _check("hd_rope", lib().hd_rope(
        _ptr(q), _ptr(k), _ptr(pos0), B, P, Hq, Hkv, D, int(rot_dim or D), float(base), int(pos_base),
        int(pos_mult), _ROPE_LAYOUTS[layout], _dt(ref), _stream(stream)))
    return q, k


def hd_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode="intra", window: int = 0,
                scale: float | None = None, out: torch.Tensor | None = None, out_dtype=None,
                lse: torch.Tensor | bool | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """Stream-Factorized Attention forward.

    q [B, n*L, Hq, D], k/v [B, n*L, Hkv, D] -> O [B, n*L, Hq, D] (and lse
    [B, Hq, n*L] float32 when ``lse`` is True or a tensor).
    """
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, nm)
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, P, Hkv, D) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q/k/v shapes or dtypes disagree")
    if P % n:
        raise ValueError("sequence length is not a multiple of n")
    L = P // n
    if scale is None:
        scale = D ** -0.5
    odt = out_dtype or q.dtype
    if out is None:
        out = torch.empty((B, P, Hq, D), dtype=odt, device=q.device)
    _need(out, "out")
    if out.shape != q.shape:
        raise ValueError("out has the wrong shape")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, Hq, P), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    if isinstance(lse, torch.Tensor):
        _need(lse, "lse")
    _check("hd_attn_fwd", lib().hd_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, n, Hq, Hkv, D, _MODES[mode], int(window),
        float(scale), _dt(q), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_fwd_rope(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode="intra", window: int = 0,
                     scale: float | None = None, rot_dim: int | None = None, base: float = 10000.0,
                     layout: str = "half", out: torch.Tensor | None = None, out_dtype=None,
                     lse: torch.Tensor | bool | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """hd_attn_fwd on rope(q), rope(k) at the contiguous positions of the
    expanded sequence, the rotation fused in: k is rotated in place, q is
    rotated inside the attention kernel and left as given.  bf16 only."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, nm)
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, P, Hkv, D) or v.shape != k.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q/k/v shapes or dtypes disagree")
    if P % n:
        raise ValueError("sequence length is not a multiple of n")
    L = P // n
    rot = int(rot_dim or D)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, P, Hq, D), dtype=out_dtype or q.dtype, device=q.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, Hq, P), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    _check("hd_attn_fwd_rope", lib().hd_attn_fwd_rope(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, n, Hq, Hkv, D, _MODES[mode], int(window),
        float(scale), rot, float(base), _ROPE_LAYOUTS[layout], _dt(q), _dt(out), _ptr(dev_status),
        _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_fwd_final_stream(q_final: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, mode="intra",
                             window: int = 0, scale: float | None = None, out: torch.Tensor | None = None,
                             out_dtype=None, lse: torch.Tensor | bool | None = None,
                             dev_status: torch.Tensor | None = None, stream=None):
    """Attention of the final-stream queries only (KV-mirror layers).

    q_final [B, L, Hq, D], k/v [B, n*L, Hkv, D] -> O [B, L, Hq, D] (and lse
    [B, Hq, L] float32 when asked): the rows of :func:`hd_attn_fwd` at the
    positions i*n + n-1.
    """
    for t, nm in ((q_final, "q_final"), (k, "k"), (v, "v")):
        _need(t, nm)
    B, L, Hq, D = q_final.shape
    Hkv = k.shape[2]
    if k.shape != (B, n * L, Hkv, D) or v.shape != k.shape or k.dtype != q_final.dtype or v.dtype != q_final.dtype:
        raise ValueError("q_final/k/v shapes or dtypes disagree")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, L, Hq, D), dtype=out_dtype or q_final.dtype, device=q_final.device)
    _need(out, "out")
    if out.shape != q_final.shape:
        raise ValueError("out has the wrong shape")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q_final.device)
    elif lse is False:
        lse = None
    _check("hd_attn_fwd_final_stream", lib().hd_attn_fwd_final_stream(
        _ptr(q_final), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, n, Hq, Hkv, D, _MODES[mode], int(window),
        float(scale), _dt(q_final), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_bwd_workspace(B: int, L: int, n: int, Hq: int, mode="intra") -> int:
    return int(lib().hd_attn_bwd_workspace(B, L, n, Hq, _MODES[mode]))


def hd_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dO: torch.Tensor,
                lse: torch.Tensor, n: int, mode="intra", window: int = 0, scale: float | None = None,
                dq: torch.Tensor | None = None, dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """Backward of :func:`hd_attn_fwd`: returns (dq, dk, dv).

    q/o/dO [B, n*L, Hq, D], k/v [B, n*L, Hkv, D] (one dtype), lse [B, Hq, n*L]
    float32 from the forward.  ``workspace`` (uint8, at least
    :func:`hd_attn_bwd_workspace` bytes) is allocated when not given.
    """
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dO, "dO"), (lse, "lse")):
        _need(t, nm)
    B, P, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, P, Hkv, D) or v.shape != k.shape or o.shape != q.shape or dO.shape != q.shape:
        raise ValueError("q/k/v/o/dO shapes disagree")
    if any(t.dtype != q.dtype for t in (k, v, o, dO)):
        raise ValueError("q/k/v/o/dO dtypes disagree")
    if lse.shape != (B, Hq, P) or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 [B, Hq, n*L]")
    if P % n:
        raise ValueError("sequence length is not a multiple of n")
    L = P // n
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, ref, nm in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _need(t, nm)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{nm} has the wrong shape or dtype")
    need = hd_attn_bwd_workspace(B, L, n, Hq, mode)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _check("hd_attn_bwd", lib().hd_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, L, n, Hq, Hkv, D,
        _MODES[mode], int(window), float(scale), _dt(q), _ptr(workspace), workspace.numel(), _ptr(dev_status),
        _stream(stream)))
    return dq, dk, dv


def hd_attn_bwd_final_stream(q_final: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_final: torch.Tensor,
                             dO_final: torch.Tensor, lse_final: torch.Tensor, n: int, mode="intra", window: int = 0,
                             scale: float | None = None, dq: torch.Tensor | None = None,
                             dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
                             workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                             stream=None):
    """Backward of :func:`hd_attn_fwd_final_stream`: returns (dq_final, dk, dv).

    q_final/o_final/dO_final [B, L, Hq, D], k/v [B, n*L, Hkv, D] (one dtype),
    lse_final [B, Hq, L] float32 from the forward."""
    for t, nm in ((q_final, "q_final"), (k, "k"), (v, "v"), (o_final, "o_final"), (dO_final, "dO_final"),
                  (lse_final, "lse_final")):
        _need(t, nm)
    B, L, Hq, D = q_final.shape
    Hkv = k.shape[2]
    if k.shape != (B, n * L, Hkv, D) or v.shape != k.shape or o_final.shape != q_final.shape or \
            dO_final.shape != q_final.shape:
        raise ValueError("q_final/k/v/o_final/dO_final shapes disagree")
    if any(t.dtype != q_final.dtype for t in (k, v, o_final, dO_final)):
        raise ValueError("dtypes disagree")
    if lse_final.shape != (B, Hq, L) or lse_final.dtype != torch.float32:
        raise ValueError("lse_final must be float32 [B, Hq, L]")
    if scale is None:
        scale = D ** -0.5
    dq = torch.empty_like(q_final) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, ref, nm in ((dq, q_final, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        _need(t, nm)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{nm} has the wrong shape or dtype")
    need = hd_attn_bwd_workspace(B, L, 1, Hq, "intra")
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q_final.device)
    _need(workspace, "workspace")
    _check("hd_attn_bwd_final_stream", lib().hd_attn_bwd_final_stream(
        _ptr(q_final), _ptr(k), _ptr(v), _ptr(o_final), _ptr(dO_final), _ptr(lse_final), _ptr(dq), _ptr(dk),
        _ptr(dv), B, L, n, Hq, Hkv, D, _MODES[mode], int(window), float(scale), _dt(q_final), _ptr(workspace),
        workspace.numel(), _ptr(dev_status), _stream(stream)))
    return dq, dk, dv


def hd_attn_decode_workspace(B: int, n: int, Lmax: int, Hq: int, Hkv: int, D: int, mode="intra") -> int:
    return int(lib().hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, _MODES[mode]))


def hd_attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, ctx_len: torch.Tensor,
                   mode="intra", window: int = 0, scale: float | None = None, out: torch.Tensor | None = None,
                   out_dtype=None, lse: torch.Tensor | bool | None = None, workspace: torch.Tensor | None = None,
                   dev_status: torch.Tensor | None = None, stream=None):
    """q [B, n, Hq, D], caches [B, n, Lmax, Hkv, D], ctx_len [B] int32 ->
    O [B, n, Hq, D] (and lse [B, n, Hq] when asked)."""
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (ctx_len, "ctx_len")):
        _need(t, nm)
    B, n, Hq, D = q.shape
    _, _, Lmax, Hkv, _ = k_cache.shape
    if k_cache.shape != (B, n, Lmax, Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shapes disagree with q")
    if ctx_len.dtype != torch.int32 or ctx_len.shape != (B,):
        raise ValueError("ctx_len must be int32 [B]")
    if scale is None:
        scale = D ** -0.5
    odt = out_dtype or q.dtype
    if out is None:
        out = torch.empty((B, n, Hq, D), dtype=odt, device=q.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, n, Hq), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    ws_bytes = hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, mode)
    if ws_bytes == 0:
        raise HDError("hd_attn_decode_workspace", HD_ERR_UNSUPPORTED)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError("workspace too small")
    _check("hd_attn_decode", lib().hd_attn_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(ctx_len), _ptr(out), _ptr(lse), B, n, Lmax, Hq, Hkv, D,
        _MODES[mode], int(window), float(scale), _dt(q), _dt(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, ctx_len: torch.Tensor,
                           mode="intra", window: int = 0, scale: float | None = None,
                           out: torch.Tensor | None = None, out_dtype=None, lse: torch.Tensor | bool | None = None,
                           dev_status: torch.Tensor | None = None, stream=None):
    """Same as :func:`hd_attn_decode` but the library uses its own fixed
    device scratch instead of a workspace, for callers that cannot hand it
    device memory (see ``hd_attn_decode_noalloc`` in ``include/hd.h``: sizes
    needing more than 64 MiB of scratch are refused, and concurrent calls on
    unordered streams race)."""
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (ctx_len, "ctx_len")):
        _need(t, nm)
    B, n, Hq, D = q.shape
    _, _, Lmax, Hkv, _ = k_cache.shape
    if k_cache.shape != (B, n, Lmax, Hkv, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shapes disagree with q")
    if ctx_len.dtype != torch.int32 or ctx_len.shape != (B,):
        raise ValueError("ctx_len must be int32 [B]")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, n, Hq, D), dtype=out_dtype or q.dtype, device=q.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, n, Hq), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    _check("hd_attn_decode_noalloc", lib().hd_attn_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(ctx_len), _ptr(out), _ptr(lse), B, n, Lmax, Hq, Hkv, D,
        _MODES[mode], int(window), float(scale), _dt(q), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


# ------------------------------------------------------- stream parallelism

def hd_stream_interleave(parts: torch.Tensor, n: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """parts [R, B, (n/R)*L, ...] (rank r's streams r + R*l) -> out [B, n*L, ...]
    in the expanded order."""
    _need(parts, "parts")
    R, B, PL = parts.shape[:3]
    rest = tuple(parts.shape[3:])
    if n % R or PL % (n // R):
        raise ValueError("shard shapes do not match n")
    L = PL // (n // R)
    row = 1
    for x in rest:
        row *= x
    if out is None:
        out = torch.empty((B, n * L) + rest, dtype=parts.dtype, device=parts.device)
    _need(out, "out")
    if out.shape != (B, n * L) + rest or out.dtype != parts.dtype:
        raise ValueError("out has the wrong shape or dtype")
    _check("hd_stream_interleave", lib().hd_stream_interleave(
        _ptr(parts), _ptr(out), R, B, L, n, row, _dt(parts), _stream(stream)))
    return out


def hd_attn_combine(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: torch.Tensor | None = None,
                    out_dtype=None, lse: torch.Tensor | bool | None = None, stream=None):
    """Merge partial results over disjoint key sets: o_parts [R, ..., D],
    lse_parts [R, ...] float32 -> O [..., D] (and lse [...] when asked)."""
    _need(o_parts, "o_parts")
    _need(lse_parts, "lse_parts")
    R = o_parts.shape[0]
    D = o_parts.shape[-1]
    if lse_parts.shape != o_parts.shape[:-1] or lse_parts.dtype != torch.float32:
        raise ValueError("lse_parts must be float32 with o_parts' shape minus the last dim")
    rows = lse_parts[0].numel()
    if out is None:
        out = torch.empty(o_parts.shape[1:], dtype=out_dtype or o_parts.dtype, device=o_parts.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    elif lse is False:
        lse = None
    _check("hd_attn_combine", lib().hd_attn_combine(
        _ptr(o_parts), _ptr(lse_parts), _ptr(out), _ptr(lse), R, rows, D, _dt(o_parts), _dt(out), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_fwd_shard(q_loc: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n: int, R: int, r: int,
                      window: int = 0, scale: float | None = None, out: torch.Tensor | None = None, out_dtype=None,
                      lse: torch.Tensor | bool | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """Cross-stream attention of rank r's queries q_loc [B, (n/R)*L, Hq, D]
    against all streams' k/v [B, n*L, Hkv, D] (expanded order)."""
    for t, nm in ((q_loc, "q_loc"), (k, "k"), (v, "v")):
        _need(t, nm)
    B, PL, Hq, D = q_loc.shape
    Hkv = k.shape[2]
    if n % R or PL % (n // R):
        raise ValueError("shard shapes do not match n")
    L = PL // (n // R)
    if k.shape != (B, n * L, Hkv, D) or v.shape != k.shape or k.dtype != q_loc.dtype or v.dtype != q_loc.dtype:
        raise ValueError("q_loc/k/v shapes or dtypes disagree")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty(q_loc.shape, dtype=out_dtype or q_loc.dtype, device=q_loc.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, Hq, PL), dtype=torch.float32, device=q_loc.device)
    elif lse is False:
        lse = None
    _check("hd_attn_fwd_shard", lib().hd_attn_fwd_shard(
        _ptr(q_loc), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, L, n, R, r, Hq, Hkv, D, int(window), float(scale),
        _dt(q_loc), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


HD_MAX_RANKS = 8
HD_IPC_HANDLE_BYTES = 64


def _shard_list(parts, R: int, name: str, shape=None, dtype=None, allow_addr: bool = False):
    """R shard addresses from a list (tensors, or device addresses if
    allow_addr) or from one tensor [R, ...]; checks the tensors' shape/dtype."""
    if isinstance(parts, torch.Tensor):
        _need(parts, name)
        if parts.shape[0] != R:
            raise ValueError(f"{name} must hold R = {R} shards")
        parts = [parts[i] for i in range(R)]
    parts = list(parts)
    if len(parts) != R:
        raise ValueError(f"{name} must hold R = {R} shards")
    addrs = []
    for i, t in enumerate(parts):
        if isinstance(t, torch.Tensor):
            _need(t, f"{name}[{i}]")
            if shape is not None and (tuple(t.shape) != tuple(shape) or t.dtype != dtype):
                raise ValueError(f"{name}[{i}] must be {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")
            addrs.append(t.data_ptr())
        elif allow_addr and isinstance(t, int):
            addrs.append(t)
        elif allow_addr and t is None:
            addrs.append(0)
        else:
            raise TypeError(f"{name}[{i}] must be a CUDA tensor" + (" or a device address" if allow_addr else ""))
    return (ctypes.c_void_p * R)(*[a or None for a in addrs])


def _parts_common(q_loc, n, R, Hkv, scale, out, out_dtype, lse):
    _need(q_loc, "q_loc")
    B, PL, Hq, D = q_loc.shape
    if R < 1 or n % R or PL % (n // R):
        raise ValueError("shard shapes do not match n")
    L = PL // (n // R)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty(q_loc.shape, dtype=out_dtype or q_loc.dtype, device=q_loc.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, Hq, PL), dtype=torch.float32, device=q_loc.device)
    elif lse is False:
        lse = None
    return B, L, Hq, D, (B, (n // R) * L, Hkv, D), scale, out, lse, want_lse


def hd_attn_fwd_parts(q_loc: torch.Tensor, k_parts, v_parts, n: int, R: int, r: int, window: int = 0,
                      scale: float | None = None, out: torch.Tensor | None = None, out_dtype=None,
                      lse: torch.Tensor | bool | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """Cross-stream attention of rank r's queries q_loc [B, (n/R)*L, Hq, D]
    against the R ranks' shards (a list of R tensors [B, (n/R)*L, Hkv, D], or
    one tensor [R, B, (n/R)*L, Hkv, D] such as an all-gather output), read in
    place."""
    first = k_parts[0]
    Hkv = first.shape[-2]
    B, L, Hq, D, sh, scale, out, lse, want_lse = _parts_common(q_loc, n, R, Hkv, scale, out, out_dtype, lse)
    ka = _shard_list(k_parts, R, "k_parts", sh, q_loc.dtype)
    va = _shard_list(v_parts, R, "v_parts", sh, q_loc.dtype)
    _check("hd_attn_fwd_parts", lib().hd_attn_fwd_parts(
        _ptr(q_loc), ka, va, _ptr(out), _ptr(lse), B, L, n, R, r, Hq, Hkv, D, int(window), float(scale),
        _dt(q_loc), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_combine_streams(o_parts, lse_parts, n: int, R: int, r: int, out: torch.Tensor | None = None,
                            out_dtype=None, lse: torch.Tensor | bool | None = None, like: torch.Tensor | None = None,
                            stream=None):
    """Merge the R ranks' cross-stream decode partials for rank r's own
    stream queries.  o_parts / lse_parts: R tensors [B, n, Hq, D] / [B, n, Hq]
    (or a stacked tensor), or device addresses of peers' buffers; ``like``
    (or the first tensor among the parts) gives B, Hq, D and the dtype."""
    ref = like
    if ref is None:
        ref = next((t for t in o_parts if isinstance(t, torch.Tensor)), None)
    if ref is None:
        raise TypeError("give `like` when every part is a device address")
    B, nn, Hq, D = ref.shape
    if nn != n or R < 1 or n % R:
        raise ValueError("partials must be [B, n, Hq, D] with R dividing n")
    oa = _shard_list(o_parts, R, "o_parts", ref.shape, ref.dtype, allow_addr=True)
    la = _shard_list(lse_parts, R, "lse_parts", (B, n, Hq), torch.float32, allow_addr=True)
    if out is None:
        out = torch.empty((B, n // R, Hq, D), dtype=out_dtype or ref.dtype, device=ref.device)
    _need(out, "out")
    want_lse = lse is True or isinstance(lse, torch.Tensor)
    if lse is True:
        lse = torch.empty((B, n // R, Hq), dtype=torch.float32, device=ref.device)
    elif lse is False:
        lse = None
    _check("hd_attn_combine_streams", lib().hd_attn_combine_streams(
        oa, la, _ptr(out), _ptr(lse), B, n, Hq, D, R, r, _dt(ref), _dt(out), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_attn_peer_flags_bytes(B: int, L: int, n: int) -> int:
    return int(lib().hd_attn_peer_flags_bytes(B, L, n))


def hd_attn_fwd_peer_gather(q_loc: torch.Tensor, k_src, v_src, k_dst, v_dst, n: int, R: int, r: int,
                            flags: torch.Tensor | None = None, window: int = 0, scale: float | None = None,
                            out: torch.Tensor | None = None, out_dtype=None, lse: torch.Tensor | bool | None = None,
                            dev_status: torch.Tensor | None = None, stream=None):
    """hd_attn_fwd_parts with the exchange inside the kernel: k_src/v_src are
    R shards (entry r a local tensor; the others tensors or peer device
    addresses from :func:`hd_ipc_open`), copied once into the local k_dst/
    v_dst shards while the attention runs.  Entry r of k_dst/v_dst may be
    None (this rank's shard is then read in place) or a slot (the shard is
    copied too; when all R slots lie at one stride, as the slots of one
    [R, ...] tensor do, a key tile is one TMA box per 64 features)."""
    if not isinstance(k_src[r], torch.Tensor) or not isinstance(v_src[r], torch.Tensor):
        raise TypeError("k_src[r] and v_src[r] must be this rank's local shard tensors")
    Hkv = k_src[r].shape[-2]
    B, L, Hq, D, sh, scale, out, lse, want_lse = _parts_common(q_loc, n, R, Hkv, scale, out, out_dtype, lse)
    ks = _shard_list(k_src, R, "k_src", sh, q_loc.dtype, allow_addr=True)
    vs = _shard_list(v_src, R, "v_src", sh, q_loc.dtype, allow_addr=True)
    kd = _shard_list(k_dst, R, "k_dst", sh, q_loc.dtype, allow_addr=True)
    vd = _shard_list(v_dst, R, "v_dst", sh, q_loc.dtype, allow_addr=True)
    nb = hd_attn_peer_flags_bytes(B, L, n)
    if flags is None:
        flags = torch.empty(max(1, nb // 8), dtype=torch.int64, device=q_loc.device)
    _need(flags, "flags")
    _check("hd_attn_fwd_peer_gather", lib().hd_attn_fwd_peer_gather(
        _ptr(q_loc), ks, vs, kd, vd, _ptr(flags), flags.numel() * flags.element_size(), _ptr(out), _ptr(lse), B, L,
        n, R, r, Hq, Hkv, D, int(window), float(scale), _dt(q_loc), _dt(out), _ptr(dev_status), _stream(stream)))
    return (out, lse) if want_lse else out


def hd_ipc_export(t: torch.Tensor):
    """(handle bytes, byte offset) of the device allocation holding t."""
    _need(t, "t")
    h = ctypes.create_string_buffer(HD_IPC_HANDLE_BYTES)
    off = ctypes.c_size_t(0)
    _check("hd_ipc_export", lib().hd_ipc_export(_ptr(t), h, ctypes.byref(off)))
    return h.raw, int(off.value)


def hd_ipc_open(handle: bytes) -> int:
    """Map another process's allocation; returns its base device address."""
    if len(handle) != HD_IPC_HANDLE_BYTES:
        raise ValueError("bad IPC handle")
    base = ctypes.c_void_p(0)
    _check("hd_ipc_open", lib().hd_ipc_open(ctypes.create_string_buffer(handle, HD_IPC_HANDLE_BYTES),
                                            ctypes.byref(base)))
    return int(base.value)


def hd_ipc_close(base: int) -> None:
    _check("hd_ipc_close", lib().hd_ipc_close(ctypes.c_void_p(base)))


def hd_attn_decode_shard(q: torch.Tensor, k_cache_loc: torch.Tensor, v_cache_loc: torch.Tensor,
                         ctx_len: torch.Tensor, R: int, r: int, window: int = 0, scale: float | None = None,
                         out: torch.Tensor | None = None, out_dtype=torch.float32, lse: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None, stream=None):
    """Cross-stream decode of all n stream queries q [B, n, Hq, D] against
    rank r's cache streams [B, n/R, Lmax, Hkv, D]: returns the partial
    (O, lse) to be merged with :func:`hd_attn_combine`."""
    for t, nm in ((q, "q"), (k_cache_loc, "k_cache_loc"), (v_cache_loc, "v_cache_loc"), (ctx_len, "ctx_len")):
        _need(t, nm)
    B, n, Hq, D = q.shape
    _, nl, Lmax, Hkv, _ = k_cache_loc.shape
    if n % R or nl != n // R or v_cache_loc.shape != k_cache_loc.shape:
        raise ValueError("cache shard shapes do not match n / R")
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((B, n, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, n, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out")
    _need(lse, "lse")
    if workspace is None:
        workspace = torch.empty(max(hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, "cross"), 1),
                                dtype=torch.uint8, device=q.device)
    _check("hd_attn_decode_shard", lib().hd_attn_decode_shard(
        _ptr(q), _ptr(k_cache_loc), _ptr(v_cache_loc), _ptr(ctx_len), _ptr(out), _ptr(lse), B, n, R, r, Lmax, Hq,
        Hkv, D, int(window), float(scale), _dt(q), _dt(out), _ptr(workspace), workspace.numel(), _ptr(dev_status),
        _stream(stream)))
    return out, lse
