"""CPU float64 oracle for the Hidden Decoding hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` may use it.  It shares no code,
constant or helper with the CUDA path.

Sources (page "Hidden Decoding at Scale", WeLM blog):
  * "Multi-Stream Expansion and Training Objective", eq. S_t = E_k(x_i) at
    t = (i-1)n + k, and the statement that only the final stream E_n feeds the
    LM head  ->  :func:`expand`, :func:`final_stream_gather`.
  * "Stream-Factorized Attention", eqs. i(t) = ceil(t/n), s(t) = (t-1) mod n + 1
    and Figure 2 masks (a) full cross-stream causal, (b) local cross-stream
    causal sliding window, (c) intra-stream causal  ->  :func:`visible`,
    :func:`attn`, :func:`attn_rows`.
  * "Computational Cost" (the layers are trained through): the gradient of
    the attention forward  ->  :func:`attn_bwd`.
  * "Persistent KV and the KV-mirror Saving" (only the final stream runs
    through the mirrored layers)  ->  :func:`attn_final_stream`.
  * "Multi-Stream Expansion and Training Objective" (the expanded sequence
    runs with contiguous RoPE positions)  ->  :func:`rope`.
  * "Persistent KV and the KV-mirror Saving" (stream parallelism: the
    intra-stream KV sharded across ranks by stream)  ->  :func:`shard_streams`,
    :func:`stream_interleave`, :func:`decode_rows_streams`,
    :func:`combine_partials`.
  * "Persistent KV and the KV-mirror Saving" (a KV cache kept for every
    stream) and "Inference Throughput" (the n streams of a token are processed
    together in one pass)  ->  :func:`decode`.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against library routines (SDPA, index_select), closed forms, invariants and a
pure-Python brute force written from the pages' 1-based formulas.  The pages
print no worked numeric example, so no value of theirs pins a number.
"""

from .hd_oracle import (  # noqa: F401
    token_index,
    stream_index,
    visible,
    visible_matrix,
    expand,
    final_stream_gather,
    attn,
    attn_rows,
    attn_rows_block,
    attn_bwd,
    attn_bwd_blocked,
    attn_bwd_final_stream,
    attn_bwd_dq_rows,
    attn_bwd_dkv_rows,
    attn_bwd_query_rows,
    attn_final_stream,
    decode,
    decode_rows,
    decode_rows_streams,
    shard_streams,
    stream_interleave,
    combine_partials,
    pair_count,
    rope,
    rope_angles,
)
