"""The cascade planner.  The oracle's planner (oracle/cascade_plan.py) is pinned on
hand-built block tables: sharing groups by first physical block, the common prefix
capped at the shortest member, chunk width and padding, sequences that share nothing.
The library's planners (pa_plan_cascade on tables, pa_bm_plan_cascade on a block
manager's state) must then give the oracle's result exactly on random batches.
CPU only."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import cascade_plan as wl
from oracle.cow import RefBlockManager
from paged_kv_cache_348_b200 import block_manager as nbm


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
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, bs, group=8, width=2)
    # group A: 3 common entries = 12 tokens, capped at the shortest member's 10 tokens
    # group B: 2 common entries = 8 tokens (both members are longer)
    assert prefix.tolist() == [10, 10, 10, 0, 8, 8]
    # 2 members per chunk: group A splits into [0, 1] and [2, pad]
    assert members.tolist() == [[0, 1], [2, -1], [4, 5]]
    assert plens.tolist() == [10, 10, 8]


def test_chunk_width_and_padding_are_exact():
    bs = 16
    rows = [[1, 2, 3]] * 5 + [[9]]
    ctx = np.array([40, 41, 42, 43, 44, 5], dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, bs, group=4, width=4)
    # width 4: members 0..3 then 4 with padding; common prefix 3 blocks = 48 tokens,
    # capped at the shortest member's 40
    assert members.tolist() == [[0, 1, 2, 3], [4, -1, -1, -1]]
    assert plens.tolist() == [40, 40]
    assert prefix.tolist() == [40, 40, 40, 40, 40, 0]
    prefix2, members2, plens2 = wl.plan_cascade(_tables(rows), ctx, bs, group=4, width=2)
    assert members2.tolist() == [[0, 1], [2, 3], [4, -1]] and plens2.tolist() == [40] * 3
    assert np.array_equal(prefix2, prefix)
    # default width: fitted to the sharing group, 5 members fit one chunk of <= 16
    prefix3, members3, plens3 = wl.plan_cascade(_tables(rows), ctx, bs, group=4)
    assert members3.tolist() == [[0, 1, 2, 3, 4]] and plens3.tolist() == [40]
    assert np.array_equal(prefix3, prefix)


def test_default_width_spreads_a_large_group_evenly():
    # group 4: at most 16 members a chunk.  20 sharers need 2 chunks, so 10 each; a second
    # group of 3 is padded to that width; a group of 40 would need 3 chunks of 14.
    bs = 8
    rows = [[7, 8]] * 20 + [[3, 4]] * 3
    ctx = np.array([16] * 23, dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, bs, group=4)
    assert members.tolist() == [list(range(10)), list(range(10, 20)),
                                [20, 21, 22] + [-1] * 7]
    assert plens.tolist() == [16, 16, 16] and prefix.tolist() == [16] * 23
    rows40 = [[7, 8]] * 40
    _, m40, _ = wl.plan_cascade(_tables(rows40), np.full(40, 16, np.int32), bs, group=4)
    assert m40.shape == (3, 14) and m40[2].tolist() == list(range(28, 40)) + [-1, -1]
    # an explicit width is kept as given
    _, m2, _ = wl.plan_cascade(_tables(rows), ctx, bs, group=4, width=16)
    assert m2.shape == (3, 16)


def test_no_sharing_and_empty_sequences_give_no_chunks():
    rows = [[1, 2], [3, 4], [1, 2]]
    ctx = np.array([20, 20, 0], dtype=np.int32)     # the third shares block 1 but is empty
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, 16, group=8)
    assert prefix.tolist() == [0, 0, 0]
    assert members.shape == (0, 8) and plens.shape == (0,)


def test_divergence_inside_the_first_block_shares_nothing_beyond_it():
    # same first block, different second block: the prefix is exactly one block
    rows = [[5, 6, 7], [5, 8, 9]]
    ctx = np.array([40, 40], dtype=np.int32)
    prefix, members, plens = wl.plan_cascade(_tables(rows), ctx, 16, group=8)
    assert prefix.tolist() == [16, 16] and members.tolist() == [[0, 1]]


def _random_sharing_batch(rng, bs):
    """Roots with random lengths, forks, and random appends (copy on write), through the
    oracle's reference block manager; returns (tables, ctx) of the live sequences."""
    N = 400
    bm = RefBlockManager(N, bs, list(rng.permutation(N)))
    sids = []
    for _ in range(int(rng.integers(1, 6))):
        root = bm.new_seq(int(rng.integers(0, 6 * bs)))
        fam = [root] + [bm.fork(root) for _ in range(int(rng.integers(0, 12)))]
        for s in fam:
            for _ in range(int(rng.integers(0, 3 * bs))):
                bm.append_slot(s)
        sids += fam
    rng.shuffle(sids)
    M = max(1, max(len(bm.tables[s]) for s in sids))
    tables = np.full((len(sids), M), 77, dtype=np.int32)
    for i, s in enumerate(sids):
        tables[i, :len(bm.tables[s])] = bm.tables[s]
    return tables, np.array([bm.ctx[s] for s in sids], dtype=np.int32)


@pytest.mark.parametrize("bs", [1, 4, 16])
def test_library_planner_equals_oracle_on_random_batches(bs):
    rng = np.random.default_rng(500 + bs)
    for _ in range(40):
        tables, ctx = _random_sharing_batch(rng, bs)
        for group, width in [(4, None), (8, None), (1, 3), (16, 4), (2, 1)]:
            want = wl.plan_cascade(tables, ctx, bs, group, width)
            got = nbm.plan_cascade_tables(tables, ctx, bs, group, width)
            for a, b in zip(got, want):
                assert a.dtype == b.dtype and np.array_equal(a, b)


def test_block_manager_planner_equals_oracle_on_its_own_tables():
    rng = np.random.default_rng(520)
    for trial in range(20):
        bs = int(rng.choice([1, 8, 16]))
        N = 300
        bm = nbm.BlockManager(N, bs, rng.permutation(N))
        sids = []
        for _ in range(int(rng.integers(1, 5))):
            root = bm.allocate(int(rng.integers(1, 5 * bs)))
            fam = [root] + [bm.fork(root) for _ in range(int(rng.integers(0, 9)))]
            for s in fam:
                for _ in range(int(rng.integers(0, 2 * bs))):
                    bm.append_token(s)
            sids += fam
        order = list(rng.permutation(len(sids)))
        batch = [sids[i] for i in order]
        tables, ctx = bm.block_tables(batch), bm.context_lens(batch)
        for group in (4, 8):
            want = wl.plan_cascade(tables, ctx, bs, group)
            got = bm.plan_cascade(batch, group)
            for a, b in zip(got, want):
                assert np.array_equal(a, b)


def test_library_planner_limits():
    t = np.array([[1, 2], [1, 2]], dtype=np.int32)
    c = np.array([20, 20], dtype=np.int32)
    with pytest.raises(ValueError):
        nbm.plan_cascade_tables(t, c, 16, group=8, width=9)       # 72 query rows > 64
    with pytest.raises(ValueError):
        nbm.plan_cascade_tables(t, np.array([20, 40], np.int32), 16, group=8)   # 3 blocks > 2
    p, m, l = nbm.plan_cascade_tables(t[:0], c[:0], 16, group=8)
    assert p.shape == (0,) and m.shape == (0, 8) and l.shape == (0,)
