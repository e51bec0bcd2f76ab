"""Property tests of the host-only layout calls over random tensor lists:
the padded layout, the server chunks (against the oracle's chunk rule) and
the shard ranges of the split step."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from error_compensated_bit_adam_b200 import _binding as B

sizes = st.lists(st.one_of(st.integers(0, 300), st.integers(0, 1 << 22)), min_size=1, max_size=12)
workers = st.integers(1, 64)


@settings(max_examples=150, deadline=None)
@given(n=st.integers(0, 1 << 34), W=workers)
def test_chunks_match_the_oracle_and_tile_the_tensor(n, W):
    o = oracle.default()
    ranges = [B.ob_chunk_range(n, W, j) for j in range(W)]
    assert ranges == [o.chunk_range(n, W, j) for j in range(W)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n
    for (b0, e0), (b1, e1) in zip(ranges, ranges[1:]):
        assert b0 <= e0 == b1 <= e1                     # contiguous, in order
    for b, e in ranges:
        assert b % 128 == 0 or b == n                   # word- and 16-byte-aligned starts


@settings(max_examples=150, deadline=None)
@given(numel=sizes, W=workers)
def test_layout_pads_and_orders_tensors(numel, W):
    offsets, n_pad = B.ob_layout(numel)
    ends = [o + -(-n // 128) * 128 for o, n in zip(offsets, numel)]
    assert offsets[0] == 0 and all(o % 128 == 0 for o in offsets)
    assert offsets[1:] == ends[:-1] and n_pad == ends[-1]


@settings(max_examples=150, deadline=None)
@given(numel=sizes, W=st.integers(1, 16), G=st.integers(1, 9))
def test_shards_partition_chunks_and_words(numel, W, G):
    offsets, n_pad = B.ob_layout(numel)
    C = len(numel) * W
    shards = [B.ob_server_shard_range(numel, W, G, r) for r in range(G)]
    assert shards[0][0] == 0 and shards[-1][1] == C
    assert shards[0][2] == 0 and shards[-1][3] == n_pad // 32
    for a, b in zip(shards, shards[1:]):
        assert a[1] == b[0] and a[3] == b[2]
    owner = np.full(n_pad // 32, -1)
    for r, (cb, ce, wb, we) in enumerate(shards):
        owner[wb:we] = r
        for c in range(cb, ce):                         # a chunk's words lie in its shard's range
            t, j = divmod(c, W)
            b, e = B.ob_chunk_range(numel[t], W, j)
            if e > b:
                assert wb <= (offsets[t] + b) // 32 and (offsets[t] + e + 31) // 32 <= we
    assert (owner >= 0).all()                           # every word has exactly one shard
