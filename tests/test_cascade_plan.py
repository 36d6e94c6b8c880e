"""The host-side cascade planner (workload.plan_cascade) on hand-built block tables:
sharing groups by first physical block, the common prefix capped at the shortest member,
chunk width and padding, and sequences that share nothing. CPU only."""
from __future__ import annotations

import numpy as np

from paged_kv_cache_348_b200 import workload as wl


def _tables(rows, width=6):
    t = np.full((len(rows), width), 999, dtype=np.int32)          # junk past the used entries
    for i, r in enumerate(rows):
        t[i, :len(r)] = r
    return t


def test_groups_prefix_and_chunks():
    bs = 4
    rows = [
        [7, 8, 9, 20],      # group A: shares 7, 8, 9 with the next two
        [7, 8, 9, 21, 22],
        [7, 8, 9],          # shortest member of A: 10 tokens (2.5 blocks)
        [3, 4],             # alone: no chunk
        [5, 6, 30],         # group B: shares 5, 6
        [5, 6, 31],
    ]
    ctx = np.array([16, 20, 10, 8, 12, 9], dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, bs, group=8)
    # group A: 3 common entries = 12 tokens, capped at the shortest member's 10 tokens
    # group B: 2 common entries = 8 tokens (both members are longer)
    assert prefix.tolist() == [10, 10, 10, 0, 8, 8]
    # width 16 // 8 = 2 members per chunk: group A splits into [0, 1] and [2, pad]
    assert members.tolist() == [[0, 1], [2, -1], [4, 5]]
    assert plens.tolist() == [10, 10, 8]


def test_chunk_width_and_padding_are_exact():
    bs = 16
    rows = [[1, 2, 3]] * 5 + [[9]]
    ctx = np.array([40, 41, 42, 43, 44, 5], dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, bs, group=4)
    # width 16 // 4 = 4: members 0..3 then 4 with padding; common prefix 3 blocks = 48
    # tokens, capped at the shortest member's 40
    assert members.tolist() == [[0, 1, 2, 3], [4, -1, -1, -1]]
    assert plens.tolist() == [40, 40]
    assert prefix.tolist() == [40, 40, 40, 40, 40, 0]
    prefix2, members2, plens2 = wl.plan_cascade(_tables(rows), ctx, bs, group=4, width=2)
    assert members2.tolist() == [[0, 1], [2, 3], [4, -1]] and plens2.tolist() == [40] * 3
    assert np.array_equal(prefix2, prefix)


def test_no_sharing_and_empty_sequences_give_no_chunks():
    rows = [[1, 2], [3, 4], [1, 2]]
    ctx = np.array([20, 20, 0], dtype=np.int32)     # the third shares block 1 but is empty
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, 16, group=8)
    assert prefix.tolist() == [0, 0, 0]
    assert members.shape == (0, 2) and plens.shape == (0,)


def test_divergence_inside_the_first_block_shares_nothing_beyond_it():
    # same first block, different second block: the prefix is exactly one block
    rows = [[5, 6, 7], [5, 8, 9]]
    ctx = np.array([40, 40], dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, 16, group=8)
    assert prefix.tolist() == [16, 16] and members.tolist() == [[0, 1]]
