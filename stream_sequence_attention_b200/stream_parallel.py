"""Stream parallelism: the intra-stream KV sharded across ranks by stream.

("Hidden Decoding at Scale", "Persistent KV and the KV-mirror Saving": by
introducing stream parallelism the intra-stream KV is sharded across
ranks.)  With R ranks (R divides n) rank r holds streams r, r + R, ..., in
the expanded order of its own n/R streams: local row i*(n/R) + l is token i
of global stream r + R*l.  Per layer:

* intra-stream attention and decode touch only a rank's own streams: the
  library's regular calls on the local tensors with n/R streams, no exchange;
* a cross-stream prefill layer all-gathers K and V (NCCL into local HBM)
  and runs ``hd_attn_fwd_parts`` for the local queries, which reads the
  gathered shards where they lie (a key tile is 128/R rows of every shard);
  ``hd_stream_interleave`` + ``hd_attn_fwd_shard`` cover the shapes that call
  does not take (float32, n not dividing 128, more than 8 ranks);
* or, with :class:`PeerShards`, the exchange runs inside the attention
  kernel: each rank exports its K/V shard buffers by CUDA IPC, and
  ``hd_attn_fwd_peer_gather`` copies the peers' shards into local memory
  tile by tile while it computes;
* cross-stream decode all-gathers the n stream queries of the new token,
  runs ``hd_attn_decode_shard`` (every query against the local cache
  streams), all-gathers the partial (O, lse) and merges them with
  ``hd_attn_combine``; or, with :class:`PeerDecode`, each rank merges its own
  stream rows straight from the ranks' exported partials
  (``hd_attn_combine_streams``).

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

    def parts_supported(self, dtype) -> bool:
        """Whether hd_attn_fwd_parts takes this layer (else the re-interleave path)."""
        return dtype == torch.bfloat16 and 128 % self.n == 0 and self.R <= hd.HD_MAX_RANKS

    def cross_attention(self, q_loc, k_loc, v_loc, window: int = 0, scale=None, **kw):
        """Cross-stream layer: all-gather K/V, then the local queries' rows."""
        if self.parts_supported(q_loc.dtype):
            kp = all_gather_shards(k_loc, self.group)
            vp = all_gather_shards(v_loc, self.group)
            return hd.hd_attn_fwd_parts(q_loc, kp, vp, self.n, self.R, self.r, window, scale, **kw)
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


class PeerShards:
    """K/V shard buffers of one cross-stream prefill layer shape, shared
    between the ranks of ``view`` by CUDA IPC, for ``hd_attn_fwd_peer_gather``.

    Each rank owns ``buffers`` pairs (K, V) of [B, (n/R)*L, Hkv, D] that the
    other ranks map; a layer writes its shard into the next pair (``stage``),
    all ranks pass a barrier (``fence``), and the kernel pulls the peers'
    shards over NVLink into local slots while it computes (``attend``); its
    own shard is copied into its slot too, so that the R local slots (one
    [R, ...] tensor) are read with one TMA box per 64 features.  With
    two pairs used in turn, one barrier per layer also keeps a rank from
    overwriting a pair before the peers' kernels that read it have finished:
    a rank passes the next barrier only after its previous kernel.

    ``fence`` is a device-side barrier on the current stream for NCCL groups
    (a one-element all-reduce); for other backends it synchronises the device
    and calls ``dist.barrier``.  Call ``close`` on every rank before the
    buffers go away.
    """

    def __init__(self, view: StreamParallel, B: int, L: int, Hkv: int, D: int, dtype=torch.bfloat16,
                 buffers: int = 2, device=None):
        if not view.parts_supported(dtype):
            raise ValueError("PeerShards needs bf16, n dividing 128 and at most HD_MAX_RANKS ranks")
        self.view = view
        self.shape = (B, view.n_loc * L, Hkv, D)
        self.dtype = dtype
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.own = [(torch.empty(self.shape, dtype=dtype, device=dev), torch.empty(self.shape, dtype=dtype, device=dev))
                    for _ in range(buffers)]
        self._peers = _PeerMap(view, [t for pair in self.own for t in pair])
        # src[i][rho] = (k, v) of rank rho's pair i: this rank's tensors, or peer addresses
        self.src = [[(self._peers.ref(rho, 2 * i, self.own[i][0]), self._peers.ref(rho, 2 * i + 1, self.own[i][1]))
                     for rho in range(view.R)] for i in range(buffers)]
        self.k_dst = torch.empty((view.R,) + self.shape, dtype=dtype, device=dev)
        self.v_dst = torch.empty_like(self.k_dst)
        nb = hd.hd_attn_peer_flags_bytes(B, L, view.n)
        self.flags = torch.empty(max(1, nb // 8), dtype=torch.int64, device=dev)
        self._tok = torch.zeros(1, dtype=torch.float32, device=dev)
        self.turn = 0
        self.staged = None

    def fence(self):
        _fence(self.view, self._tok)

    def stage(self, k_loc: torch.Tensor | None = None, v_loc: torch.Tensor | None = None) -> int:
        """Take the next buffer pair, copy k_loc/v_loc into it (None: the caller
        wrote ``own[i]`` directly) and return its index."""
        i = self.turn
        self.turn = (self.turn + 1) % len(self.own)
        if k_loc is not None:
            self.own[i][0].copy_(k_loc)
        if v_loc is not None:
            self.own[i][1].copy_(v_loc)
        self.staged = i
        return i

    def attend(self, q_loc, window: int = 0, scale=None, **kw):
        """The fused gather + attention of the local queries on the staged pair."""
        if self.staged is None:
            raise RuntimeError("stage() a buffer pair first")
        row = self.src[self.staged]
        ks = [row[rho][0] for rho in range(self.view.R)]
        vs = [row[rho][1] for rho in range(self.view.R)]
        return hd.hd_attn_fwd_peer_gather(q_loc, ks, vs, self.k_dst, self.v_dst, self.view.n, self.view.R,
                                          self.view.r, flags=self.flags, window=window, scale=scale, **kw)

    def cross_attention(self, q_loc, k_loc, v_loc, window: int = 0, scale=None, **kw):
        """stage + fence + attend."""
        self.stage(k_loc, v_loc)
        self.fence()
        return self.attend(q_loc, window, scale, **kw)

    def close(self):
        """Unmap the peers' buffers (after a barrier, so no rank still reads)."""
        self.fence()
        torch.cuda.synchronize()
        self._peers.close()


class PeerDecode:
    """Stream-parallel cross-stream decode with the partials' exchange fused
    into the merge: each rank writes its partial (O, lse) for all n stream
    queries into buffers the other ranks map by CUDA IPC, all ranks pass a
    barrier, and ``hd_attn_combine_streams`` reads the R partials of this
    rank's own stream rows where they lie.  Two buffer sets are used in turn,
    so one barrier per step also keeps a rank from overwriting a set that a
    peer still reads.  The n stream queries themselves are still gathered
    with a collective (``cross_decode``), or passed in whole (``partial``)."""

    def __init__(self, view: StreamParallel, B: int, Hq: int, D: int, buffers: int = 2, device=None):
        if view.R > hd.HD_MAX_RANKS:
            raise ValueError("PeerDecode supports at most HD_MAX_RANKS ranks")
        self.view = view
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        n = view.n
        self.own = [(torch.empty((B, n, Hq, D), dtype=torch.float32, device=dev),
                     torch.empty((B, n, Hq), dtype=torch.float32, device=dev)) for _ in range(buffers)]
        self._peers = _PeerMap(view, [t for pair in self.own for t in pair])
        self.src = [[(self._peers.ref(rho, 2 * i, self.own[i][0]), self._peers.ref(rho, 2 * i + 1, self.own[i][1]))
                     for rho in range(view.R)] for i in range(buffers)]
        self._tok = torch.zeros(1, dtype=torch.float32, device=dev)
        self.turn = 0
        self.staged = None

    def fence(self):
        _fence(self.view, self._tok)

    def partial(self, q, kc_loc, vc_loc, ctx_len, window: int = 0, scale=None, workspace=None, dev_status=None):
        """This rank's partial for all n stream queries q [B, n, Hq, D] against
        its cache streams, written into the next buffer set."""
        i = self.turn
        self.turn = (self.turn + 1) % len(self.own)
        o, lse = self.own[i]
        hd.hd_attn_decode_shard(q, kc_loc, vc_loc, ctx_len, self.view.R, self.view.r, window, scale, out=o, lse=lse,
                                workspace=workspace, dev_status=dev_status)
        self.staged = i
        return i

    def merge(self, out_dtype=torch.bfloat16, out=None):
        """O [B, n/R, Hq, D] of this rank's stream queries from the R partials."""
        if self.staged is None:
            raise RuntimeError("partial() first")
        row = self.src[self.staged]
        return hd.hd_attn_combine_streams([row[rho][0] for rho in range(self.view.R)],
                                          [row[rho][1] for rho in range(self.view.R)], self.view.n, self.view.R,
                                          self.view.r, out=out, out_dtype=out_dtype, like=self.own[self.staged][0])

    def cross_decode(self, q_loc, kc_loc, vc_loc, ctx_len, window: int = 0, scale=None, workspace=None):
        """All-gather the stream queries, partial, barrier, fused merge."""
        q = hd.hd_stream_interleave(all_gather_shards(q_loc, self.view.group), self.view.n)
        self.partial(q, kc_loc, vc_loc, ctx_len, window, scale, workspace)
        self.fence()
        return self.merge(out_dtype=q_loc.dtype)

    def close(self):
        self.fence()
        torch.cuda.synchronize()
        self._peers.close()


def _fence(view: StreamParallel, tok: torch.Tensor):
    """Barrier of the view's ranks on the current stream (NCCL: a one-element
    all-reduce; other backends: synchronise the device, then dist.barrier)."""
    if dist.get_backend(view.group) == "nccl":
        dist.all_reduce(tok, group=view.group)
    else:
        torch.cuda.synchronize()
        dist.barrier(group=view.group)


class _PeerMap:
    """CUDA IPC mapping of every rank's copy of a list of device tensors.
    ``ref(rho, j, mine)`` is rank rho's tensor j: ``mine`` for this rank, else
    the device address of the peer's tensor in this process."""

    def __init__(self, view: StreamParallel, tensors):
        def export(t):
            handle, off = hd.hd_ipc_export(t)
            return handle, off, t.data_ptr() - off  # the exporter's allocation base identifies it

        mine = [export(t) for t in tensors]
        every = [None] * view.R
        dist.all_gather_object(every, mine, group=view.group)
        # Tensors may share one allocation (the caching allocator splits
        # segments): map each exported allocation once.
        self._bases = {}
        self.addr = []
        for rho in range(view.R):
            row = []
            for handle, off, owner_base in every[rho]:
                if rho == view.r:
                    row.append(None)
                    continue
                key = (rho, owner_base)
                if key not in self._bases:
                    self._bases[key] = hd.hd_ipc_open(handle)
                row.append(self._bases[key] + off)
            self.addr.append(row)
        self.r = view.r

    def ref(self, rho: int, j: int, mine):
        return mine if rho == self.r else self.addr[rho][j]

    def close(self):
        for base in self._bases.values():
            hd.hd_ipc_close(base)
        self._bases = {}
