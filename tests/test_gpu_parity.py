"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Attention: |gpu - oracle| <= 2e-3 + 1e-2*|oracle| per element (fp64 oracle before
its own rounding).  Append, copy and gather: bit-exact.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200 import pagedkv as pk
from paged_kv_cache_348_b200 import workload as wl
from tests.conftest import record_parity
from tests.helpers import NAN_BITS, bits, from_bits, make_case

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2
NTHREADS = 8


def assert_attn_close(got: torch.Tensor, ref64: np.ndarray, rows=None, what=""):
    """|gpu - oracle| <= 2e-3 + 1e-2 |oracle| per element.  Records, per case, the max
    abs error, the max rel error over |oracle| >= 1e-3, and the worst err / bound ratio
    (the margin to the bound), which tests/conftest.py writes out at the end of the run."""
    g = got.detach().float().cpu().double().numpy()
    if rows is not None:
        g, ref64 = g[rows], ref64[rows]
    assert np.isfinite(g).all(), what + ": non-finite output"
    err = np.abs(g - ref64)
    bound = ATOL + RTOL * np.abs(ref64)
    bad = err > bound
    big = np.abs(ref64) >= 1e-3
    rel = (err[big] / np.abs(ref64[big])).max() if big.any() else 0.0
    record_parity(what, float(err.max()), float(rel), float((err / bound).max()), err.size)
    assert not bad.any(), "%s: %d/%d elements out of tolerance; max abs %.3g, max rel %.3g" % (
        what, int(bad.sum()), bad.size, err.max(), rel)
    return float(err.max()), float(rel)


def _dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def run_case(case, device="cuda"):
    """Upload an oracle-side case (uint16 bits) and run pa_decode; returns out tensor."""
    dt = case["dtype"]
    q = from_bits(case["q"], dt).to(device)
    k = from_bits(case["k"], dt).to(device)
    v = from_bits(case["v"], dt).to(device)
    tables = _dev(case["tables"])
    ctx = _dev(case["ctx"])
    out = torch.full_like(q, float("nan"))
    ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)                               # workspace content on entry must not matter
    st = pk.new_status()
    pk.pa_decode(out, q, k, v, tables, ctx, case["scale"], ws, st)
    torch.cuda.synchronize()
    return out, int(st.item())


def oracle_of(case, items=None):
    return oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                         case["scale"], case["dtype"], items=items, nthreads=NTHREADS)


# ------------------------------------------------------------------ shape sweep
CTX_MIX = [0, 1, 2, 15, 16, 17, 31, 63, 64, 65, 100, 129, 255, 300, 511, 1000]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 4), (12, 1), (32, 2)])
def test_decode_shape_sweep(dtype, D, bs, Hq, Hkv):
    case = make_case(len(CTX_MIX), Hq, Hkv, D, bs, CTX_MIX, dtype=dtype,
                     seed=100 + D + bs + Hq)
    out, st = run_case(case)
    assert st == 0
    ref, _ = oracle_of(case)
    assert_attn_close(out, ref, what="sweep %s D%d bs%d %d/%d" % (dtype, D, bs, Hq, Hkv))
    assert not out[0].float().abs().max().item()          # empty context -> zeros


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_single_token_context_returns_v0_bits(dtype):
    case = make_case(3, 8, 1, 128, 16, [1, 1, 1], dtype=dtype, seed=7)
    out, st = run_case(case)
    assert st == 0
    got = bits(out)
    for s in range(3):
        v0 = case["v"][case["tables"][s, 0], 0, 0]
        assert np.array_equal(got[s], np.broadcast_to(v0, got[s].shape))


# ------------------------------------------------------------------ invariants (bit-exact)
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_physical_permutation_and_identity_table_are_bit_identical(bs):
    ctx = [700, 33, 1, 2048, 129, 0, 64]
    a = make_case(len(ctx), 32, 8, 128, bs, ctx, dtype="bf16", seed=21, shuffle=True)
    out_a, _ = run_case(a)
    perm = np.random.default_rng(5).permutation(a["N"])
    b = dict(a)
    b["k"], b["v"] = np.empty_like(a["k"]), np.empty_like(a["v"])
    b["k"][perm], b["v"][perm] = a["k"], a["v"]
    b["tables"] = np.where(a["tables"] >= 0, perm[np.clip(a["tables"], 0, None)],
                           a["tables"]).astype(np.int32)
    out_b, _ = run_case(b)
    assert torch.equal(bits_t(out_a), bits_t(out_b))
    # contiguous placement (identity table) of the same logical data
    c = make_case(len(ctx), 32, 8, 128, bs, ctx, dtype="bf16", seed=21, shuffle=False)
    for s in range(len(ctx)):
        for lb in range(-(-ctx[s] // bs)):
            c["k"][c["tables"][s, lb]] = a["k"][a["tables"][s, lb]]
            c["v"][c["tables"][s, lb]] = a["v"][a["tables"][s, lb]]
    c["q"] = a["q"]
    out_c, _ = run_case(c)
    assert torch.equal(bits_t(out_a), bits_t(out_c))


def bits_t(t):
    return t.contiguous().view(torch.int16)


def test_nan_poisoned_free_blocks_and_tails_change_no_bit():
    ctx = [5, 16, 17, 40, 333]
    clean = make_case(5, 16, 4, 128, 16, ctx, dtype="f16", seed=9, poison=False)
    dirty = make_case(5, 16, 4, 128, 16, ctx, dtype="f16", seed=9, poison=True)
    assert (dirty["k"] == NAN_BITS["f16"]).any()
    a, _ = run_case(clean)
    b, _ = run_case(dirty)
    assert torch.equal(bits_t(a), bits_t(b))


def test_shared_prefix_blocks_equal_private_copies():
    bs, ctx = 16, [300, 300, 300]
    priv = make_case(3, 32, 8, 128, bs, ctx, dtype="f16", seed=31, poison=False)
    shared = dict(priv)
    shared["tables"] = priv["tables"].copy()
    shared["k"], shared["v"] = priv["k"].copy(), priv["v"].copy()
    for s in (1, 2):                                   # first 10 blocks shared with seq 0
        for lb in range(10):
            shared["k"][priv["tables"][s, lb]] = priv["k"][priv["tables"][0, lb]]
            shared["v"][priv["tables"][s, lb]] = priv["v"][priv["tables"][0, lb]]
    a, _ = run_case(shared)
    shared["tables"][1:, :10] = priv["tables"][0, :10]
    b, _ = run_case(shared)
    assert torch.equal(bits_t(a), bits_t(b))


def test_repeat_runs_are_deterministic():
    case = make_case(9, 64, 8, 128, 16, [4000, 17, 2500, 9000, 1, 64, 333, 7777, 128],
                     dtype="bf16", seed=41)
    a, _ = run_case(case)
    b, _ = run_case(case)
    assert torch.equal(bits_t(a), bits_t(b))


# ------------------------------------------------------------------ device error reporting
def test_bad_block_id_sets_status_and_does_not_fault():
    case = make_case(3, 8, 2, 128, 16, [40, 50, 60], dtype="f16", seed=51)
    case["tables"][1, 2] = case["N"] + 5
    out, st = run_case(case)
    assert st & pk.DEV_BAD_BLOCK_ID
    ref, _ = oracle_of(case, items=[0, 2])
    assert_attn_close(out, ref, rows=[0, 2], what="rows without the bad id")


def test_context_len_over_capacity_is_flagged_and_clamped():
    case = make_case(2, 8, 2, 64, 16, [40, 50], dtype="f16", seed=52)
    case["ctx"] = case["ctx"].copy()
    case["ctx"][1] = case["tables"].shape[1] * 16 + 100
    out, st = run_case(case)
    assert st & pk.DEV_BAD_CONTEXT_LEN


def test_host_validation_errors():
    case = make_case(2, 8, 2, 128, 16, [40, 50], dtype="f16", seed=53)
    q = from_bits(case["q"], "f16").cuda()
    k = from_bits(case["k"], "f16").cuda()
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(pk.PagedKVError, match="invalid"):
        pk.pa_decode(torch.empty_like(q), q, k, k, _dev(case["tables"]), _dev(case["ctx"]), 0.1,
                     small)


# ------------------------------------------------------------------ append / copy (bit-exact)
def test_append_bit_exact_and_bad_slot_flag():
    N, Hkv, bs, D, T = 50, 8, 16, 128, 37
    k = inputs.randn((N, Hkv, bs, D), "bf16", 60, "cuda", 1)
    v = inputs.randn((N, Hkv, bs, D), "bf16", 60, "cuda", 2)
    kn = inputs.randn((T, Hkv, D), "bf16", 60, "cuda", 3)
    vn = inputs.randn((T, Hkv, D), "bf16", 60, "cuda", 4)
    slots = np.random.default_rng(6).choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1
    hk, hv = bits(k), bits(v)
    oracle.cache_append(hk, hv, bits(kn), bits(vn), slots)
    st = pk.new_status()
    pk.pa_cache_append(k, v, kn, vn, _dev(slots), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(bits(k), hk) and np.array_equal(bits(v), hv)
    bad = torch.tensor([N * bs + 3], dtype=torch.int64, device="cuda")
    pk.pa_cache_append(k, v, kn[:1], vn[:1], bad, st)
    torch.cuda.synchronize()
    assert int(st.item()) & pk.DEV_BAD_SLOT
    assert np.array_equal(bits(k), hk)


def test_copy_blocks_bit_exact_all_layers_and_bad_pair_flag():
    L, N, Hkv, bs, D = 5, 40, 8, 16, 128
    ks = [inputs.randn((N, Hkv, bs, D), "f16", 70, "cuda", 2 * l) for l in range(L)]
    vs = [inputs.randn((N, Hkv, bs, D), "f16", 70, "cuda", 2 * l + 1) for l in range(L)]
    hks, hvs = [bits(t) for t in ks], [bits(t) for t in vs]
    pairs = np.array([[1, 30], [7, 2], [1, 31], [39, 0]], dtype=np.int32)
    oracle.copy_blocks(hks, hvs, pairs)
    st = pk.new_status()
    pk.pa_copy_blocks(ks, vs, _dev(pairs), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for l in range(L):
        assert np.array_equal(bits(ks[l]), hks[l]) and np.array_equal(bits(vs[l]), hvs[l])
    pk.pa_copy_blocks(ks, vs, _dev(np.array([[0, N]], dtype=np.int32)), st)
    torch.cuda.synchronize()
    assert int(st.item()) & pk.DEV_BAD_PAIR


# ------------------------------------------------------------------ the measured workloads
def _host(b, layer):
    return (bits(b.q[layer]), bits(b.k_caches[layer]), bits(b.v_caches[layer]),
            b.block_tables.cpu().numpy(), b.context_lens.cpu().numpy())


def _step_and_check(b, layers, items=None, check_append=True):
    """Run one full step; check append bit-exact and decode against the oracle for the
    listed layers (items: sampled sequences, None = all)."""
    pre = {l: (bits(b.k_caches[l]), bits(b.v_caches[l])) for l in layers} if check_append else {}
    wl.run_step(b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    res = []
    for l in layers:
        q, k, v, t, c = _host(b, l)
        if check_append:
            hk, hv = pre[l]
            if b.cow_pairs is not None:
                oracle.copy_blocks([hk], [hv], b.cow_pairs.cpu().numpy())
            oracle.cache_append(hk, hv, bits(b.k_new[l]), bits(b.v_new[l]),
                                b.slot_mapping.cpu().numpy())
            assert np.array_equal(k, hk) and np.array_equal(v, hv), "append/copy mismatch"
        ref, _ = oracle.decode(q, k, v, t, c, b.scale, b.w.dtype, items=items, nthreads=NTHREADS)
        rows = items if items is not None else slice(None)
        res.append(assert_attn_close(b.out[l], ref, rows=rows, what="%s layer %d" % (b.w.name, l)))
    return res


def test_workload_tiny():
    b = wl.build(inputs.TINY)
    # poison every slot no sequence holds, then check nothing changes
    used = torch.zeros((b.num_blocks, b.block_size), dtype=torch.bool)
    for s in b.sids:
        for t in range(b.bm.context_len(s)):
            used[b.bm.table(s)[t // b.block_size], t % b.block_size] = True
    free = (~used).nonzero()
    for kc in b.k_caches + b.v_caches:
        kc[free[:, 0].cuda(), :, free[:, 1].cuda()] = float("nan")
    _step_and_check(b, [0])


def test_workload_llama8b_full():
    _step_and_check(wl.build(inputs.LLAMA8B), [0])


def test_workload_llama70b_two_layers_full_size():
    b = wl.build(inputs.LLAMA70B, layers=2)
    assert b.w.num_q_heads == 64 and b.w.dtype == "bf16"
    _step_and_check(b, [0, 1])


def test_workload_prefix_fork_cow():
    b = wl.build_prefix_fork()
    assert b.cow_pairs.shape[0] == inputs.PREFIX_PROMPTS * (inputs.PREFIX_SAMPLES - 1)
    items = list(range(0, 128, 5)) + [127]
    _step_and_check(b, [0], items=items)


def test_workload_prefix_decode_sampled():
    b = wl.build_prefix_decode()
    assert b.unique_kv_bytes_per_step() < b.kv_bytes_per_step() / 3
    items = list(range(0, 128, 9)) + [127]
    _step_and_check(b, [0], items=items)


@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_workload_heavytail_sampled(bs):
    b = wl.build(inputs.HEAVYTAIL, block_size=bs)
    ctx = b.context_lens.cpu().numpy()
    longest = list(np.argsort(ctx)[-6:])
    items = sorted(set(longest + list(range(0, 256, 17))))
    _step_and_check(b, [0], items=[int(i) for i in items])


def test_bounded_waits_give_up_and_the_gpu_stays_usable():
    """The wait helpers every decode pipeline uses give up after their limit when nothing
    completes the barrier or raises the count (the kernels then set PA_DEV_TIMEOUT and
    leave), and the device stays usable: a decode right after matches the oracle."""
    res = pk.pa_check_bounded_waits(20000)             # 20 ms limit
    assert res[0] == 1 and res[1] == 1, res
    assert 20000 <= res[2] < 1000000 and 20000 <= res[3] < 1000000, res
    case = make_case(3, 8, 2, 128, 16, [5, 40, 100], dtype="f16", seed=610)
    out, status = run_case(case)
    assert status == 0
    ref, _ = oracle_of(case)
    assert_attn_close(out, ref, what="decode after the wait check")
