"""Host block manager (product) against the oracle's reference planner, plus the
workload generators' shapes.  CPU only."""
from __future__ import annotations

import numpy as np
import pytest

from oracle.cow import RefBlockManager
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200.block_manager import BlockManager, PoolExhausted


def _scenario(mgr_cls, order):
    m = mgr_cls(200, 8, order)
    out = []
    new = (lambda n: m.allocate(n)) if mgr_cls is BlockManager else (lambda n: m.new_seq(n))
    app = (lambda s: m.append_token(s)) if mgr_cls is BlockManager else (lambda s: m.append_slot(s))
    a = new(21)
    b = m.fork(a)
    c = m.fork(a)
    for sid in (a, b, c, b, c, a):
        out.append(app(sid))
    d = new(8)
    e = m.fork(d)
    out.append(app(e))                       # full shared block: fresh block, no copy
    tables = (m.table if mgr_cls is BlockManager else (lambda s: m.tables[s]))
    return out, [list(tables(s)) for s in (a, b, c, d, e)]


def test_matches_reference_planner_exactly():
    order = inputs.pool_order(200, 9)
    assert _scenario(BlockManager, order) == _scenario(RefBlockManager, order)


def test_cow_fork_phase_pairs_and_slots():
    bs = 16
    m = BlockManager(1000, bs, inputs.pool_order(1000, 3))
    root = m.allocate(2048 + 7)
    kids = [root] + [m.fork(root) for _ in range(7)]
    shared = m.table(root)[-1]
    res = [m.append_token(s) for s in kids]
    pairs = [c for _, c in res if c]
    assert len(pairs) == 7 and {p[0] for p in pairs} == {shared}
    assert m.refcount(shared) == 1
    assert all(slot % bs == 7 for slot, _ in res)
    assert len({slot // bs for slot, _ in res}) == 8


def test_release_returns_blocks_and_exhaustion_raises():
    m = BlockManager(10, 4)
    a = m.allocate(16)
    b = m.fork(a)
    assert m.free_blocks == 6
    m.release(a)
    assert m.free_blocks == 6                # still held by b
    m.release(b)
    assert m.free_blocks == 10
    m.allocate(40)
    with pytest.raises(PoolExhausted):
        m.allocate(1)


def test_tail_waste_counts_only_last_block_tails():
    m = BlockManager(100, 16)
    lens = [1, 16, 17, 40, 5]
    sids = [m.allocate(n) for n in lens]
    held = sum(-(-n // 16) * 16 for n in lens)
    unused = 0
    for s, n in zip(sids, lens):              # brute force: count empty slots per block
        for i, _ in enumerate(m.table(s)):
            unused += sum(1 for o in range(16) if i * 16 + o >= n)
    assert m.tail_waste(sids) == pytest.approx(unused / held)


def test_slot_of_matches_table():
    m = BlockManager(50, 8, inputs.pool_order(50, 1))
    s = m.allocate(30)
    t = m.table(s)
    for pos in range(30):
        assert m.slot_of(s, pos) == t[pos // 8] * 8 + pos % 8


def test_workload_generators():
    assert list(inputs.context_lens(inputs.TINY)) == [5, 16, 17, 40]
    c1 = inputs.context_lens(inputs.LLAMA8B)
    assert len(c1) == 64 and c1.min() >= 128 and c1.max() <= 2048
    c2 = inputs.context_lens(inputs.LLAMA70B)
    assert len(c2) == 32 and c2.min() >= 1000 and c2.max() <= 8000
    c4 = inputs.context_lens(inputs.HEAVYTAIL)
    assert len(c4) == 256 and c4.min() >= 16 and c4.max() <= 32768
    assert 300 < np.median(c4) < 800
    c3 = inputs.context_lens(inputs.PREFIX)
    assert len(c3) == 128 and c3.min() >= 2048 and c3.max() <= 2048 + 512
    t = inputs.prefix_fork_tails()
    assert t.min() >= 1 and t.max() <= 15
    assert np.array_equal(inputs.context_lens(inputs.LLAMA8B), c1)        # seeded
    p = inputs.pool_order(64, 0)
    assert sorted(p) == list(range(64)) and not np.array_equal(p, np.arange(64))
