"""Host block manager (product: the native pa_bm_* calls of libpagedkv, through its
Python wrapper) against the oracle's reference planner, plus the workload generators'
shapes.  CPU only: the manager never touches a GPU."""
from __future__ import annotations

import numpy as np
import pytest

from oracle.cow import RefBlockManager
from paged_kv_cache_348_b200 import build as pbuild
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200.block_manager import BlockManager, PoolExhausted


@pytest.fixture(scope="module", autouse=True)
def _library():
    pbuild.build()


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


def test_random_operations_match_reference_planner():
    """Differential run: the same random stream of prefills, forks, single and batched
    appends and releases on the native manager and on the reference planner."""
    rng = np.random.default_rng(123)
    for trial in range(20):
        N, bs = int(rng.integers(20, 120)), int(rng.choice([1, 4, 8, 16]))
        order = rng.permutation(N).astype(np.int32)
        m, r = BlockManager(N, bs, order), RefBlockManager(N, bs, order)
        live = []
        for _ in range(150):
            op = rng.integers(0, 10)
            if op < 2 or not live:
                n = int(rng.integers(0, 3 * bs + 2))
                try:
                    sid = m.allocate(n)
                except PoolExhausted:
                    assert len(r.free) < -(-n // bs)     # the reference could not either
                    continue
                assert r.new_seq(n) == sid
                live.append(sid)
            elif op < 4:
                p = int(rng.choice(live))
                c = m.fork(p)
                assert r.fork(p) == c
                live.append(c)
            elif op < 8:
                batch = [int(x) for x in rng.choice(live, size=int(rng.integers(1, 5)))]
                free0 = m.free_blocks
                tables0 = {s: m.table(s) for s in live}
                try:
                    slots, pairs = m.append_tokens(batch)
                except PoolExhausted:
                    # nothing changed
                    assert m.free_blocks == free0
                    assert {s: m.table(s) for s in live} == tables0
                    continue
                ref_slots, ref_pairs = [], []
                for sid in batch:
                    sl, cow = r.append_slot(sid)
                    ref_slots.append(sl)
                    if cow:
                        ref_pairs.append(cow)
                assert list(slots) == ref_slots
                assert [tuple(p) for p in pairs.tolist()] == ref_pairs
            else:
                sid = int(rng.choice(live))
                m.release(sid)
                r.release(sid)
                live.remove(sid)
            assert m.free_blocks == len(r.free)
            for sid in live:
                assert m.table(sid) == r.tables[sid]
                assert m.context_len(sid) == r.ctx[sid]
            for b in range(N):
                assert m.refcount(b) == r.ref[b]


def test_batch_append_that_does_not_fit_changes_nothing():
    m = BlockManager(6, 4)
    a = m.allocate(6)                      # 2 blocks, the second holds 2 of 4 tokens
    kids = [m.fork(a) for _ in range(3)]   # all four share both blocks
    assert m.free_blocks == 4
    free0, t0 = m.free_blocks, {s: m.table(s) for s in [a] + kids}
    # 3 copies of the shared partial block, then a and kids[0] each cross into a new
    # block: 5 fresh blocks needed, 4 free
    with pytest.raises(PoolExhausted):
        m.append_tokens([a] + kids + [a, a, kids[0], kids[0]])
    assert m.free_blocks == free0 and {s: m.table(s) for s in [a] + kids} == t0
    assert [m.refcount(b) for b in t0[a]] == [4, 4]
    slots, pairs = m.append_tokens([a] + kids)   # the last writer keeps the original
    shared = t0[a][1]
    assert [p[0] for p in pairs.tolist()] == [shared] * 3 and m.free_blocks == 1
    assert m.table(kids[-1])[1] == shared and m.refcount(shared) == 1
    assert slots[-1] == shared * 4 + 2


def test_native_manager_rejects_bad_arguments():
    with pytest.raises(ValueError):
        BlockManager(4, 4, [0, 1, 1, 3])
    m = BlockManager(8, 4)
    with pytest.raises(ValueError):
        m.fork(7)
    with pytest.raises(ValueError):
        m.release(3)
    s = m.allocate(5)
    with pytest.raises(ValueError):
        m.slot_of(s, 5)
    with pytest.raises(ValueError):
        m.block_tables([s], width=1)
    assert m.block_tables([s], width=3, fill=-1).tolist() == [[0, 1, -1]]


def test_random_operations_with_preemption_match_reference_planner():
    """Differential run as above with swap-outs and swap-ins mixed in: returned blocks,
    tables, lengths, free and reference counts agree after every operation, and a
    swapped-out sequence is refused by the calls that need its table."""
    rng = np.random.default_rng(321)
    for trial in range(20):
        N, bs = int(rng.integers(20, 100)), int(rng.choice([1, 4, 8, 16]))
        order = rng.permutation(N).astype(np.int32)
        m, r = BlockManager(N, bs, order), RefBlockManager(N, bs, order)
        live, out = [], []
        for _ in range(200):
            op = rng.integers(0, 12)
            if op < 2 or not (live or out):
                n = int(rng.integers(0, 3 * bs + 2))
                try:
                    sid = m.allocate(n)
                except PoolExhausted:
                    continue
                assert r.new_seq(n) == sid
                live.append(sid)
            elif op < 3 and live:
                p = int(rng.choice(live))
                c = m.fork(p)
                assert r.fork(p) == c
                live.append(c)
            elif op < 6 and live:
                sid = int(rng.choice(live))
                try:
                    slot, cow = m.append_token(sid)
                except PoolExhausted:
                    continue
                assert (slot, cow) == r.append_slot(sid)
            elif op < 8 and live:
                sid = live.pop(int(rng.integers(len(live))))
                got = m.swap_out(sid)
                assert got.tolist() == r.swap_out(sid)
                out.append(sid)
                with pytest.raises(ValueError):
                    m.append_token(sid)
                with pytest.raises(ValueError):
                    m.fork(sid)
                assert m.context_len(sid) == r.ctx[sid]
            elif op < 10 and out:
                sid = int(rng.choice(out))
                try:
                    got = m.swap_in(sid)
                except PoolExhausted:
                    with pytest.raises(MemoryError):
                        r.swap_in(sid)
                    continue
                assert got.tolist() == r.swap_in(sid)
                out.remove(sid)
                live.append(sid)
            else:
                pool = live + out
                if not pool:
                    continue
                sid = int(rng.choice(pool))
                m.release(sid)
                r.release(sid)
                (live if sid in live else out).remove(sid)
            assert m.free_blocks == len(r.free)
            for sid in live:
                assert m.table(sid) == r.tables[sid] and m.context_len(sid) == r.ctx[sid]
            for b in range(N):
                assert m.refcount(b) == r.ref[b]
