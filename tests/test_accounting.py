"""The bench's closed-form work counts against the oracle's mask enumeration."""

import numpy as np
import pytest

import oracle
from stream_sequence_attention_b200 import accounting as acc


@pytest.mark.parametrize("L,n", [(9, 1), (8, 2), (6, 4), (5, 3)])
@pytest.mark.parametrize("mode", ["intra", "cross"])
@pytest.mark.parametrize("W", [0, 1, 2, 5, 40])
def test_pairs_match_mask_enumeration(L, n, mode, W):
    assert acc.pairs_per_head(L, n, mode, W) == oracle.pair_count(L, n, mode, W)


@pytest.mark.parametrize("n,T", [(1, 5), (4, 7), (3, 1)])
def test_decode_flops_match_enumeration(n, T):
    for mode in ("intra", "cross"):
        pairs = 0
        for s in range(n):
            p = (T - 1) * n + s
            pairs += int(np.count_nonzero(oracle.visible(p, np.arange(T * n), n, mode)))
        assert acc.decode_flops(1, n, T, 1, 1, mode) == pairs * 4


def test_headline_workload_numbers():
    # n=4, L=4096, batch 2, 32 query heads, head_dim 128
    assert abs(acc.attn_flops(2, 4096, 4, 32, 128, "intra") / 1e12 - 1.0998) < 1e-4
    assert abs(acc.attn_flops(2, 4096, 4, 32, 128, "cross") / 1e12 - 4.3983) < 1e-4
    # long context: n=4, L=32768, 64 heads, W=4096
    assert abs(acc.attn_flops(1, 32768, 4, 64, 128, "intra", 4096) / 1e12 - 16.493) < 1e-3
    # decode: batch 64, n=4, 32768 tokens, 64/8 heads
    assert abs(acc.decode_bytes(64, 4, 32768, 64, 8, 128) / 1e9 - 34.37) < 0.01


@pytest.mark.parametrize("L,n", [(7, 1), (6, 2), (5, 4), (9, 3)])
@pytest.mark.parametrize("mode", ["intra", "cross"])
@pytest.mark.parametrize("W", [0, 1, 3, 50])
def test_final_stream_pairs_match_enumeration(L, n, mode, W):
    pk = np.arange(n * L)
    want = sum(int(np.count_nonzero(oracle.visible(i * n + n - 1, pk, n, mode, W))) for i in range(L))
    assert acc.pairs_final_stream(L, n, mode, W) == want


def test_cross_shard_pairs_sum_to_the_full_cross_layer():
    from stream_sequence_attention_b200 import accounting as acc
    for n, R, L, W in [(4, 2, 9, 0), (4, 4, 7, 5), (6, 3, 5, 0), (2, 1, 11, 3)]:
        parts = [acc.pairs_cross_shard(L, n, R, r, W) for r in range(R)]
        assert sum(parts) == acc.pairs_per_head(L, n, "cross", W)
