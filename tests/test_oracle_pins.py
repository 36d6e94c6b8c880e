"""Pins for the CPU oracle: each test checks it against something other than itself
(the pages' worked numbers, closed forms, a library routine, exact brute force,
invariants).  CPU only."""
from __future__ import annotations

import json
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
from oracle.cow import RefBlockManager
from tests.helpers import NAN_BITS, bits_to_f64, make_case

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- sizing identity
def test_sizing_identity_matches_pages():
    g = _gold("p1_kv_sizing.json")
    per_tok = oracle.kv_bytes_per_token(g["layers"], g["kv_heads"], g["head_dim"], g["elem_bytes"])
    assert per_tok == g["bytes_per_token"] == 327_680
    assert round(128_000 * per_tok / 2**30, 2) == g["gib_at_128000_tokens_2dp"]
    assert round(g["prompt_tokens_read_as"] * per_tok / 1e9, 2) == g["gb_for_prompt_2dp"]
    # 4,000 tokens would not give the printed figure: the reading in the fixture is needed
    assert round(4000 * per_tok / 1e9, 2) != g["gb_for_prompt_2dp"]


# ---------------------------------------------------------------- the worked block table
def test_core_principle_worked_block_table():
    g = _gold("p2_core_principle_block_table.json")
    bs, n = g["block_size"], g["num_tokens"]
    N, Hkv, D = 64, 1, 2
    # every slot holds a marker (block, offset) in its two dims, as exact fp16 integers
    cache = np.zeros((N, Hkv, bs, D), dtype=np.float16)
    for b in range(N):
        for o in range(bs):
            cache[b, 0, o] = (b, o)
    table = np.array(g["block_table"], dtype=np.int32)
    got = oracle.gather(cache.view(np.uint16), "f16", table, n, 0)
    assert got.shape == (n, D)
    assert [tuple(int(x) for x in r) for r in got] == [tuple(e) for e in
                                                      g["expected_physical_location_per_token"]]


# ---------------------------------------------------------------- conversions
def test_f16_decode_all_patterns():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.to_f64(int(p), "f16") for p in pats])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_bf16_decode_all_patterns():
    pats = np.arange(65536, dtype=np.uint32)
    ref = (pats << 16).view(np.float32).astype(np.float64)
    got = np.array([oracle.to_f64(int(p), "bf16") for p in pats])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def _sample_doubles(n, seed):
    r = np.random.default_rng(seed)
    mags = 2.0 ** r.uniform(-30, 20, size=n)
    x = mags * r.choice([-1.0, 1.0], size=n)
    return np.concatenate([x, [0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 6.0e-8, 2.98e-8,
                               2.0**-24, 2.0**-25, 3 * 2.0**-26, 1 + 2.0**-11, 1 + 3 * 2.0**-11]])


def test_f64_to_f16_rne_matches_numpy():
    for x in _sample_doubles(20000, 5):
        ref = np.array([x]).astype(np.float16).view(np.uint16)[0]
        assert oracle.from_f64(float(x), "f16") == ref, x


def test_f64_to_bf16_rne_brute_force_grid():
    # every finite bf16 value, decoded by numpy; nearest neighbour, ties to even pattern
    pats = np.arange(0, 0x7F80, dtype=np.uint32)            # +0 .. max finite
    vals = (pats << 16).view(np.float32).astype(np.float64)
    for x in np.concatenate([_sample_doubles(20000, 6), [1 + 2.0**-8, 1 + 3 * 2.0**-8, 0.1]]):
        ax = abs(x)
        i = int(np.searchsorted(vals, ax))
        if i == 0:
            p = 0
        else:
            lo, hi = i - 1, min(i, len(vals) - 1)
            dlo, dhi = ax - vals[lo], vals[hi] - ax
            p = lo if (dlo < dhi or (dlo == dhi and lo % 2 == 0)) else hi
        exp = p | (0x8000 if np.signbit(x) else 0)
        assert oracle.from_f64(float(x), "bf16") == exp, x
    assert oracle.from_f64(0.1, "bf16") == 0x3DCD          # 0x3DCCCCCD rounded up
    assert oracle.from_f64(1 + 2.0**-8, "bf16") == 0x3F80   # tie -> even
    assert oracle.from_f64(1 + 3 * 2.0**-8, "bf16") == 0x3F82
    assert oracle.from_f64(3.5e38, "bf16") == 0x7F80        # overflow -> inf


# ---------------------------------------------------------------- brute force (mpmath)
def _mp_decode(case, s, h):
    """softmax(scale q.k) V with 50 significant digits, no max shift, dims outermost."""
    mpmath.mp.dps = 50
    g = case["Hq"] // case["Hkv"]
    kvh = h // g
    ctx, bs, D = int(case["ctx"][s]), case["bs"], case["D"]
    qf = bits_to_f64(case["q"][s, h], case["dtype"])
    rows = [(int(case["tables"][s, t // bs]), t % bs) for t in range(ctx)]
    kf = [bits_to_f64(case["k"][b, kvh, o], case["dtype"]) for b, o in rows]
    vf = [bits_to_f64(case["v"][b, kvh, o], case["dtype"]) for b, o in rows]
    sc = mpmath.mpf(case["scale"])
    w = [mpmath.exp(sc * mpmath.fsum(mpmath.mpf(qf[d]) * mpmath.mpf(kf[t][d]) for d in range(D)))
         for t in range(ctx)]
    den = mpmath.fsum(w)
    return [float(mpmath.fsum(w[t] * mpmath.mpf(vf[t][d]) for t in range(ctx)) / den)
            for d in range(D)]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_brute_force_tiny(dtype):
    case = make_case(4, 4, 2, 8, 2, [1, 2, 3, 7], dtype=dtype, seed=11)
    out64, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                             case["scale"], dtype)
    for s in range(4):
        for h in range(4):
            ref = np.array(_mp_decode(case, s, h))
            np.testing.assert_allclose(out64[s, h], ref, rtol=1e-12, atol=1e-14)


def test_brute_force_tiny_workload_shape():
    # the 4-sequence, head_dim 64, block_size 16 shape with context lens {5,16,17,40}
    case = make_case(4, 4, 4, 64, 16, [5, 16, 17, 40], dtype="f16", seed=0, pool_blocks=64)
    out64, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                             case["scale"], "f16")
    for s, h in [(0, 0), (1, 3), (2, 1), (3, 2)]:
        np.testing.assert_allclose(out64[s, h], _mp_decode(case, s, h), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- library special case
@pytest.mark.parametrize("Hq,Hkv,D,bs", [(8, 2, 16, 4), (6, 6, 32, 16), (8, 1, 8, 1)])
def test_contiguous_case_equals_torch_sdpa(Hq, Hkv, D, bs):
    ctx = [1, 5, 13, 24]
    case = make_case(4, Hq, Hkv, D, bs, ctx, dtype="f16", seed=3, shuffle=False, poison=False)
    out64, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                             case["scale"], "f16")
    k = torch.from_numpy(bits_to_f64(case["k"], "f16"))
    v = torch.from_numpy(bits_to_f64(case["v"], "f16"))
    q = torch.from_numpy(bits_to_f64(case["q"], "f16"))
    start = 0
    for s, c in enumerate(ctx):
        nb = -(-c // bs)
        assert list(case["tables"][s, :nb]) == list(range(start, start + nb))  # contiguous
        Ks = k[start:start + nb].permute(1, 0, 2, 3).reshape(Hkv, nb * bs, D)[:, :c]
        Vs = v[start:start + nb].permute(1, 0, 2, 3).reshape(Hkv, nb * bs, D)[:, :c]
        Ks = Ks.repeat_interleave(Hq // Hkv, dim=0)
        Vs = Vs.repeat_interleave(Hq // Hkv, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[s].unsqueeze(1), Ks, Vs, scale=case["scale"]).squeeze(1)
        np.testing.assert_allclose(out64[s], ref.numpy(), rtol=1e-12, atol=1e-13)
        start += nb


# ---------------------------------------------------------------- closed forms
def test_identical_keys_give_mean_of_values():
    case = make_case(2, 4, 2, 16, 4, [9, 30], seed=4, poison=False)
    k = case["k"]
    for s in range(2):
        for t in range(int(case["ctx"][s])):
            b = case["tables"][s, t // 4]
            k[b, :, t % 4] = k[case["tables"][s, 0], :, 0]
    out64, _ = oracle.decode(case["q"], k, case["v"], case["tables"], case["ctx"], case["scale"],
                             "f16")
    for s in range(2):
        for h in range(4):
            rows = [bits_to_f64(case["v"][case["tables"][s, t // 4], h // 2, t % 4], "f16")
                    for t in range(int(case["ctx"][s]))]
            np.testing.assert_allclose(out64[s, h], np.mean(rows, axis=0), rtol=1e-14, atol=1e-15)


def test_dominant_key_returns_its_value_row():
    D, bs, ctx, j = 16, 4, 11, 6
    case = make_case(1, 1, 1, D, bs, [ctx], seed=5, poison=False)
    q = np.zeros((1, 1, D), dtype=np.float16)
    q[0, 0, 0] = 16.0
    k = bits_to_f64(case["k"], "f16").astype(np.float16)
    for t in range(ctx):
        k[case["tables"][0, t // bs], 0, t % bs, 0] = 16.0 if t == j else 0.0
    out64, _ = oracle.decode(q.view(np.uint16), k.view(np.uint16), case["v"], case["tables"],
                             case["ctx"], 1.0, "f16")
    vj = bits_to_f64(case["v"][case["tables"][0, j // bs], 0, j % bs], "f16")
    np.testing.assert_allclose(out64[0, 0], vj, rtol=1e-15, atol=1e-100)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_token_returns_v0_and_empty_returns_zero(dtype):
    case = make_case(2, 2, 1, 32, 8, [1, 0], dtype=dtype, seed=6)
    out64, out16 = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                                 case["scale"], dtype)
    v0 = case["v"][case["tables"][0, 0], 0, 0]
    assert np.array_equal(out16[0, 0], v0) and np.array_equal(out16[0, 1], v0)
    assert np.array_equal(out64[0, 0], bits_to_f64(v0, dtype))
    assert not out64[1].any() and not out16[1].any()


# ---------------------------------------------------------------- invariants
def test_physical_permutation_is_bit_invariant():
    case = make_case(3, 8, 2, 32, 4, [7, 19, 33], seed=7)
    ref, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], "f16")
    perm = np.random.default_rng(1).permutation(case["N"])
    k2, v2 = np.empty_like(case["k"]), np.empty_like(case["v"])
    k2[perm], v2[perm] = case["k"], case["v"]
    t2 = np.where(case["tables"] >= 0, perm[np.clip(case["tables"], 0, None)], case["tables"])
    got, _ = oracle.decode(case["q"], k2, v2, t2.astype(np.int32), case["ctx"], case["scale"], "f16")
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_shared_prefix_blocks_equal_private_copies():
    bs, D = 4, 16
    shared = make_case(2, 4, 2, D, bs, [13, 13], seed=8, poison=False)
    t = shared["tables"].copy()
    t[1, :3] = t[0, :3]                 # seq 1 reuses seq 0's first 3 blocks (12 tokens)
    for lb in range(3):                 # ...whose private copies hold the same bytes
        shared["k"][shared["tables"][1, lb]] = shared["k"][t[0, lb]]
        shared["v"][shared["tables"][1, lb]] = shared["v"][t[0, lb]]
    a, _ = oracle.decode(shared["q"], shared["k"], shared["v"], t, shared["ctx"], shared["scale"],
                         "f16")
    b, _ = oracle.decode(shared["q"], shared["k"], shared["v"], shared["tables"], shared["ctx"],
                         shared["scale"], "f16")
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_poisoned_free_blocks_and_tails_change_nothing(dtype):
    clean = make_case(3, 4, 1, 16, 8, [3, 8, 21], dtype=dtype, seed=9, poison=False)
    dirty = make_case(3, 4, 1, 16, 8, [3, 8, 21], dtype=dtype, seed=9, poison=True)
    assert (dirty["k"] == NAN_BITS[dtype]).any()
    a, _ = oracle.decode(clean["q"], clean["k"], clean["v"], clean["tables"], clean["ctx"],
                         clean["scale"], dtype)
    b, _ = oracle.decode(dirty["q"], dirty["k"], dirty["v"], dirty["tables"], dirty["ctx"],
                         dirty["scale"], dtype)
    assert np.isfinite(b).all() and np.array_equal(a.view(np.uint64), b.view(np.uint64))


def test_threads_and_item_subset_do_not_change_bits():
    case = make_case(5, 8, 2, 32, 16, [40, 1, 77, 16, 3], seed=10)
    a, a16 = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], "f16", nthreads=1)
    b, b16 = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], "f16", nthreads=4)
    c, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                         case["scale"], "f16", items=[2, 4])
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64)) and np.array_equal(a16, b16)
    assert np.array_equal(c[[2, 4]].view(np.uint64), a[[2, 4]].view(np.uint64))
    assert not c[[0, 1, 3]].any()


def test_bad_block_id_is_reported():
    case = make_case(1, 2, 1, 16, 4, [9], seed=12)
    case["tables"][0, 1] = case["N"]
    with pytest.raises(ValueError):
        oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"], 1.0, "f16")


# ---------------------------------------------------------------- append / copy / COW
def test_append_round_trip_and_nothing_else_changes():
    N, Hkv, bs, D, T = 10, 3, 4, 16, 9
    r = np.random.default_rng(13)
    k = r.integers(0, 0x7C00, size=(N, Hkv, bs, D), dtype=np.uint16)
    v = r.integers(0, 0x7C00, size=(N, Hkv, bs, D), dtype=np.uint16)
    knew = r.integers(0, 0x7C00, size=(T, Hkv, D), dtype=np.uint16)
    vnew = r.integers(0, 0x7C00, size=(T, Hkv, D), dtype=np.uint16)
    slots = r.choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[3] = -1                                       # padding token
    k0, v0 = k.copy(), v.copy()
    oracle.cache_append(k, v, knew, vnew, slots)
    touched = np.zeros((N, bs), dtype=bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        b, o = divmod(int(s), bs)
        touched[b, o] = True
        assert np.array_equal(k[b, :, o], knew[i]) and np.array_equal(v[b, :, o], vnew[i])
    keep = ~touched
    assert np.array_equal(k.transpose(0, 2, 1, 3)[keep], k0.transpose(0, 2, 1, 3)[keep])
    assert np.array_equal(v.transpose(0, 2, 1, 3)[keep], v0.transpose(0, 2, 1, 3)[keep])
    with pytest.raises(ValueError):
        oracle.cache_append(k, v, knew[:1], vnew[:1], np.array([N * bs], dtype=np.int64))


def test_copy_blocks_all_layers():
    L, N = 3, 12
    r = np.random.default_rng(14)
    ks = [r.integers(0, 65535, size=(N, 2, 4, 8), dtype=np.uint16) for _ in range(L)]
    vs = [r.integers(0, 65535, size=(N, 2, 4, 8), dtype=np.uint16) for _ in range(L)]
    k0, v0 = [a.copy() for a in ks], [a.copy() for a in vs]
    pairs = np.array([[1, 5], [7, 2], [1, 11]], dtype=np.int32)
    oracle.copy_blocks(ks, vs, pairs)
    for l in range(L):
        exp_k, exp_v = k0[l].copy(), v0[l].copy()
        for s, d in pairs:
            exp_k[d], exp_v[d] = k0[l][s], v0[l][s]
        assert np.array_equal(ks[l], exp_k) and np.array_equal(vs[l], exp_v)


def test_cow_fork_phase_copies_the_shared_partial_block():
    bs, samples, tail = 16, 8, 5
    bm = RefBlockManager(400, bs)
    root = bm.new_seq(2048 + tail)                      # 129 blocks, the last one partial
    kids = [root] + [bm.fork(root) for _ in range(samples - 1)]
    partial = bm.tables[root][-1]
    assert bm.ref[partial] == samples
    pairs, slots = [], []
    for sid in kids:
        slot, cow = bm.append_slot(sid)
        slots.append(slot)
        if cow:
            pairs.append(cow)
    # every sample but the last one to write diverges from the shared partial block
    assert len(pairs) == samples - 1 and all(src == partial for src, _ in pairs)
    assert len({d for _, d in pairs}) == samples - 1
    assert bm.ref[partial] == 1 and bm.tables[kids[-1]][-1] == partial
    assert len(set(slots)) == samples and all(s % bs == tail for s in slots)
    # a full shared block is never copied: appending past it allocates a fresh block
    bm2 = RefBlockManager(20, bs)
    a = bm2.new_seq(32)
    b = bm2.fork(a)
    s1, c1 = bm2.append_slot(b)
    assert c1 is None and s1 % bs == 0 and bm2.tables[b][:2] == bm2.tables[a][:2]


# ---- RefBlockManager.release, pinned on its own: "PagedAttention in Production",
# "Core Principle" (a finished request's blocks go back to the pool) and "Paged Attention
# and Memory Efficiency in Production LLM Serving", "How PagedAttention borrows OS
# paging" (shared blocks stay while any sharer holds them).

def test_release_of_a_fork_keeps_the_shared_blocks():
    bm = RefBlockManager(10, 4)
    a = bm.new_seq(10)                                   # 3 blocks: 0, 1, 2
    b = bm.fork(a)
    assert [bm.ref[x] for x in bm.tables[a]] == [2, 2, 2]
    free_before = list(bm.free)
    bm.release(b)
    # every block is still held by `a`: count down to 1, nothing returns to the pool
    assert [bm.ref[x] for x in bm.tables[a]] == [1, 1, 1]
    assert bm.free == free_before and b not in bm.tables and b not in bm.ctx
    assert bm.tables[a] == [0, 1, 2] and bm.ctx[a] == 10


def test_release_of_the_last_holder_frees_in_table_order_at_the_back():
    order = [5, 2, 7, 0, 3, 1, 6, 4]
    bm = RefBlockManager(8, 4, order)
    a = bm.new_seq(9)                                     # takes 5, 2, 7
    b = bm.new_seq(4)                                     # takes 0
    assert bm.tables[a] == [5, 2, 7] and bm.tables[b] == [0] and bm.free == [3, 1, 6, 4]
    bm.release(a)
    assert bm.free == [3, 1, 6, 4, 5, 2, 7]               # back of the queue, table order
    assert [bm.ref[x] for x in (5, 2, 7)] == [0, 0, 0] and bm.ref[0] == 1
    # the released blocks are handed out again, after the older free ones
    c = bm.new_seq(4 * 6)
    assert bm.tables[c] == [3, 1, 6, 4, 5, 2]
    assert bm.free == [7]


def test_release_of_a_diverged_sample_returns_only_its_private_copy():
    bm = RefBlockManager(12, 4)
    root = bm.new_seq(6)                                   # blocks 0 (full), 1 (partial)
    kid = bm.fork(root)
    slot, cow = bm.append_slot(kid)                        # kid copies the partial block
    assert cow == (1, 2) and bm.tables[kid] == [0, 2] and slot == 2 * 4 + 2
    bm.release(kid)
    assert bm.ref[0] == 1 and bm.ref[1] == 1 and bm.ref[2] == 0
    assert bm.free[-1] == 2 and 0 not in bm.free and 1 not in bm.free


def test_release_conserves_the_pool_under_random_forks_and_appends():
    rng = np.random.default_rng(21)
    for trial in range(20):
        N, bs = 64, int(rng.choice([1, 2, 4, 8]))
        bm = RefBlockManager(N, bs, list(rng.permutation(N)))
        live = []
        for _ in range(120):
            op = rng.integers(0, 4)
            try:
                if op == 0 or not live:
                    live.append(bm.new_seq(int(rng.integers(0, 3 * bs + 1))))
                elif op == 1:
                    live.append(bm.fork(live[int(rng.integers(len(live)))]))
                elif op == 2:
                    bm.append_slot(live[int(rng.integers(len(live)))])
                else:
                    bm.release(live.pop(int(rng.integers(len(live)))))
            except MemoryError:
                pass
            # recount from the tables alone: a block's count is the number of table
            # entries naming it, and a block is free exactly when nothing names it
            held = {}
            for t in bm.tables.values():
                for x in t:
                    held[x] = held.get(x, 0) + 1
            assert all(bm.ref[x] == held.get(x, 0) for x in range(N))
            assert sorted(bm.free + list(held)) == list(range(N))
        for s in live:
            bm.release(s)
        assert sorted(bm.free) == list(range(N)) and not any(bm.ref) and not bm.tables


# ---- RefBlockManager.swap_out / swap_in (preemption): "Paged Attention and Memory
# Efficiency in Production LLM Serving", "Why KV cache memory was the bottleneck"
# (requests are preempted when the cache runs out), with the release rule of
# "PagedAttention in Production", "Core Principle".

def test_swap_out_releases_like_release_and_keeps_the_length():
    bm = RefBlockManager(10, 4, [9, 8, 7, 6, 5, 4, 3, 2, 1, 0])
    a = bm.new_seq(9)                                      # 9, 8, 7
    b = bm.fork(a)
    bm.append_slot(b)                                      # b copies partial block 7 -> 6
    assert bm.tables[b] == [9, 8, 6] and bm.free == [5, 4, 3, 2, 1, 0]
    out = bm.swap_out(b)
    assert out == [9, 8, 6]                                 # table order, to be saved
    assert bm.ref[9] == 1 and bm.ref[8] == 1 and bm.ref[6] == 0   # shared ones stay with a
    assert bm.free == [5, 4, 3, 2, 1, 0, 6] and bm.ctx[b] == 10 and bm.tables[b] == []
    assert bm.tables[a] == [9, 8, 7] and bm.ctx[a] == 9


def test_swap_in_takes_fresh_blocks_from_the_front():
    bm = RefBlockManager(8, 4, [3, 1, 4, 0, 5, 2, 6, 7])
    a = bm.new_seq(10)                                     # 3, 1, 4
    out = bm.swap_out(a)
    assert out == [3, 1, 4] and bm.free == [0, 5, 2, 6, 7, 3, 1, 4]
    c = bm.new_seq(20)                                     # 0, 5, 2, 6, 7: reuses nothing yet
    assert bm.tables[c] == [0, 5, 2, 6, 7]
    back = bm.swap_in(a)
    assert back == [3, 1, 4] and bm.tables[a] == [3, 1, 4] and bm.free == []
    assert all(bm.ref[x] == 1 for x in back) and a not in bm.swapped and bm.ctx[a] == 10


def test_swap_in_that_does_not_fit_changes_nothing():
    bm = RefBlockManager(4, 4)
    a = bm.new_seq(12)                                     # 0, 1, 2
    bm.swap_out(a)
    c = bm.new_seq(8)                                      # 3, 0
    free0, ref0 = list(bm.free), list(bm.ref)
    with pytest.raises(MemoryError):
        bm.swap_in(a)                                      # needs 3, 2 free
    assert bm.free == free0 and bm.ref == ref0 and a in bm.swapped and bm.tables[a] == []
    bm.release(c)
    assert len(bm.swap_in(a)) == 3
