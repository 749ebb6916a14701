"""Stream parallelism: the intra-stream KV sharded across ranks by stream.

("Hidden Decoding at Scale", "Persistent KV and the KV-mirror Saving": by
introducing stream parallelism the intra-stream KV is sharded across
ranks.)  With R ranks (R divides n) rank r holds streams r, r + R, ..., in
the expanded order of its own n/R streams: local row i*(n/R) + l is token i
of global stream r + R*l.  Per layer:

* intra-stream attention and decode touch only a rank's own streams: the
  library's regular calls on the local tensors with n/R streams, no exchange;
* a cross-stream prefill layer all-gathers K and V (NCCL into local HBM),
  restores the expanded order with ``hd_stream_interleave`` and runs
  ``hd_attn_fwd_shard`` for the local queries;
* cross-stream decode all-gathers the n stream queries of the new token,
  runs ``hd_attn_decode_shard`` (every query against the local cache
  streams), all-gathers the partial (O, lse) and merges them with
  ``hd_attn_combine``.

Every rank takes the same collective steps in the same order.  This module
is host-side plumbing: the arithmetic runs in the library's kernels and the
exchange in ``torch.distributed`` (NCCL on GPUs).
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import hd


def local_streams(n: int, R: int, r: int) -> list[int]:
    """Global streams held by rank r of R: r, r + R, ..."""
    if R < 1 or n % R or not 0 <= r < R:
        raise ValueError(f"stream parallelism needs R | n and 0 <= r < R (n={n}, R={R}, r={r})")
    return list(range(r, n, R))


def all_gather_shards(x: torch.Tensor, group=None) -> torch.Tensor:
    """[R, *x.shape]: every rank's x, in rank order."""
    R = dist.get_world_size(group)
    x = x.contiguous()
    out = torch.empty((R,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    if x.is_cuda:
        dist.all_gather_into_tensor(out, x, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), x, group=group)
    return out


class StreamParallel:
    """One rank's view of an n-stream expansion sharded over a process group."""

    def __init__(self, n: int, group=None):
        self.n = n
        self.group = group
        self.R = dist.get_world_size(group)
        self.r = dist.get_rank(group)
        self.streams = local_streams(n, self.R, self.r)
        self.n_loc = n // self.R

    # ------------------------------------------------------------- prefill

    def intra_attention(self, q_loc, k_loc, v_loc, window: int = 0, scale=None, **kw):
        """Intra-stream layer on the local streams: no exchange."""
        return hd.hd_attn_fwd(q_loc, k_loc, v_loc, self.n_loc, "intra", window, scale, **kw)

    def gather_kv(self, k_loc: torch.Tensor, v_loc: torch.Tensor):
        """Every stream's K and V in the expanded order [B, n*L, Hkv, D]."""
        k = hd.hd_stream_interleave(all_gather_shards(k_loc, self.group), self.n)
        v = hd.hd_stream_interleave(all_gather_shards(v_loc, self.group), self.n)
        return k, v

    def cross_attention(self, q_loc, k_loc, v_loc, window: int = 0, scale=None, **kw):
        """Cross-stream layer: all-gather K/V, then the local queries' rows."""
        k, v = self.gather_kv(k_loc, v_loc)
        return hd.hd_attn_fwd_shard(q_loc, k, v, self.n, self.R, self.r, window, scale, **kw)

    # -------------------------------------------------------------- decode

    def intra_decode(self, q_loc, kc_loc, vc_loc, ctx_len, window: int = 0, scale=None, **kw):
        """Intra-stream decode of the local streams: no exchange."""
        return hd.hd_attn_decode(q_loc, kc_loc, vc_loc, ctx_len, "intra", window, scale, **kw)

    def cross_decode(self, q_loc, kc_loc, vc_loc, ctx_len, window: int = 0, scale=None, workspace=None):
        """Cross-stream decode of the local stream queries q_loc [B, n/R, Hq, D]
        against every rank's cache streams.  Returns O [B, n/R, Hq, D]."""
        q = hd.hd_stream_interleave(all_gather_shards(q_loc, self.group), self.n)  # [B, n, Hq, D]
        o_part, lse_part = hd.hd_attn_decode_shard(q, kc_loc, vc_loc, ctx_len, self.R, self.r, window, scale,
                                                   workspace=workspace)
        o_all = all_gather_shards(o_part, self.group)
        lse_all = all_gather_shards(lse_part, self.group)
        o = hd.hd_attn_combine(o_all, lse_all, out_dtype=q_loc.dtype)  # [B, n, Hq, D]
        return o[:, self.r::self.R].contiguous()
