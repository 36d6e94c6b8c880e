"""GPU parity of the 8-bit E4M3 KV cache with per-(block, kv head) scales, through the C
ABI: pa_cache_append_e4m3_bs bit-exact (codes and scales) against the oracle's quantising
append, pa_decode_e4m3_bs (one or several new tokens) within |gpu - oracle| <= 2e-3 +
1e-2*|oracle| of the oracle's fp64 decode over the same codes and scales, block-permutation
invariance, and a full-size 70B-shape layer whose pools were filled by the append."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200 import pagedkv as pk
from paged_kv_cache_348_b200 import workload as wl
from tests.helpers import bits, from_bits, make_case
from tests.test_gpu_parity import assert_attn_close

pytestmark = pytest.mark.gpu

NTHREADS = 8
NAN8 = 0x7F


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bs_case(ctx, Hq, Hkv, bs, dtype, seed, q_len=1, skip_last=False, D=128):
    """8-bit pools filled the way a server fills them: every cached token appended in
    position order through the oracle's block-scaled append (so each block's scale is the
    one its first token fixed); free blocks and tails hold NaN codes, blocks without a
    token NaN scales.  skip_last: each sequence's newest token (position ctx-1) is left
    out, for the fused append to write."""
    case = make_case(len(ctx), Hq, Hkv, D, bs, ctx, dtype=dtype, seed=seed, poison=False)
    N = case["N"]
    k8 = np.full((N, Hkv, bs, D), NAN8, np.uint8)
    v8 = np.full((N, Hkv, bs, D), NAN8, np.uint8)
    ks = np.full((N, Hkv), np.nan, np.float32)
    vs = np.full((N, Hkv), np.nan, np.float32)
    slots = []
    for i, s in enumerate(case["sids"]):
        t = case["bm"].tables[s]
        n = int(ctx[i]) - (1 if skip_last and ctx[i] > 0 else 0)
        slots += [t[p // bs] * bs + p % bs for p in range(n)]
    slots = np.array(slots, np.int64)
    T = max(1, len(slots))
    rng_k = bits(inputs.randn((T, Hkv, D), dtype, seed, stream=41))
    rng_v = bits(inputs.randn((T, Hkv, D), dtype, seed, stream=42))
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, rng_k[:len(slots)], rng_v[:len(slots)], slots,
                                dtype)
    case.update(k8=k8, v8=v8, ks=ks, vs=vs)
    if q_len > 1:
        case["q"] = bits(inputs.randn((len(ctx), q_len, Hq, D), dtype, seed, stream=43))
    return case


def run_bs(case):
    q = from_bits(case["q"], case["dtype"]).cuda()
    out = torch.full_like(q, float("nan"))
    ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)
    st = pk.new_status()
    pk.pa_decode_e4m3_bs(out, q, _dev(case["k8"]), _dev(case["v8"]), _dev(case["ks"]),
                         _dev(case["vs"]), _dev(case["tables"]), _dev(case["ctx"]), case["scale"],
                         ws, st)
    torch.cuda.synchronize()
    return out, int(st.item())


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_block_scaled_append_is_bit_exact(dtype, bs):
    N, Hkv, D = 40, 4, 128
    rng = np.random.default_rng(700 + bs)
    k8 = rng.integers(0, 256, size=(N, Hkv, bs, D), dtype=np.uint8)
    v8 = rng.integers(0, 256, size=(N, Hkv, bs, D), dtype=np.uint8)
    ks = rng.uniform(0.1, 1.0, size=(N, Hkv)).astype(np.float32)
    vs = rng.uniform(0.1, 1.0, size=(N, Hkv)).astype(np.float32)
    # offsets 0 and later of several blocks, the offset-0 token after a later one, padding
    blocks = rng.permutation(N)[:12]
    slots = []
    for b in blocks[:8]:
        offs = rng.permutation(bs)[:min(bs, 3)].tolist()
        if 0 not in offs and rng.random() < 0.6:
            offs.append(0)
        slots += [int(b) * bs + o for o in offs]
    slots += [-1, int(blocks[9]) * bs + bs - 1]
    slots = np.array(rng.permutation(slots), np.int64)
    T = len(slots)
    k = bits(inputs.randn((T, Hkv, D), dtype, 70, stream=1) * 3)
    v = bits(inputs.randn((T, Hkv, D), dtype, 70, stream=2) * 0.05)
    dk8, dv8, dks, dvs = _dev(k8), _dev(v8), _dev(ks), _dev(vs)
    st = pk.new_status()
    pk.pa_cache_append_e4m3_bs(dk8, dv8, dks, dvs, from_bits(k, dtype).cuda(),
                               from_bits(v, dtype).cuda(), _dev(slots), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, k, v, slots, dtype)
    assert np.array_equal(dks.cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(dvs.cpu().numpy().view(np.uint32), vs.view(np.uint32))
    assert np.array_equal(dk8.cpu().numpy(), k8) and np.array_equal(dv8.cpu().numpy(), v8)


CTX_MIX = [0, 1, 2, 15, 16, 17, 31, 63, 64, 65, 100, 129, 255, 300, 511, 1000, 2047]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv,q_len,D", [(4, 4, 1, 128), (32, 8, 1, 128), (64, 8, 1, 128),
                                            (16, 1, 1, 128), (32, 8, 4, 128), (64, 8, 2, 128),
                                            (8, 8, 3, 128), (4, 4, 1, 64), (32, 8, 1, 64),
                                            (16, 1, 1, 64), (8, 2, 4, 64)])
def test_block_scaled_decode_matches_oracle(dtype, bs, Hq, Hkv, q_len, D):
    case = bs_case(CTX_MIX, Hq, Hkv, bs, dtype, seed=710 + bs + Hq + q_len + D, q_len=q_len, D=D)
    out, st = run_bs(case)
    assert st == 0
    ref, _ = oracle.decode_e4m3_bs(case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                   case["tables"], case["ctx"], case["scale"], dtype,
                                   nthreads=NTHREADS)
    assert_attn_close(out, ref, what="e4m3 block scales %s D%d bs%d %d/%d q_len %d" % (
        dtype, D, bs, Hq, Hkv, q_len))
    assert not out[0].float().abs().max().item()


def test_block_scaled_decode_is_permutation_invariant_and_repeatable():
    ctx = [700, 33, 1, 2048, 129, 0, 64, 4097]
    a = bs_case(ctx, 32, 8, 16, "bf16", seed=730)
    o1, _ = run_bs(a)
    o2, _ = run_bs(a)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    perm = np.random.default_rng(5).permutation(a["N"])
    b = dict(a)
    for key in ("k8", "v8", "ks", "vs"):
        b[key] = np.empty_like(a[key])
        b[key][perm] = a[key]
    b["tables"] = np.where(a["tables"] >= 0, perm[np.clip(a["tables"], 0, None)],
                           a["tables"]).astype(np.int32)
    o3, _ = run_bs(b)
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_block_scaled_llama70b_layer_full_size():
    """A full-size 70B-shape layer (32 seqs, 64/8 heads, ctx U[1000,8000], bf16) whose 8-bit
    pools were filled by pa_cache_append_e4m3_bs over every cached token; sequences
    sampled against the oracle."""
    b = wl.build(inputs.LLAMA70B, layers=1, kv8="block")
    out = torch.empty_like(b.q[0])
    pk.pa_decode_e4m3_bs(out, b.q[0], b.k_caches[0], b.v_caches[0], b.kv_bscales[0][0],
                         b.kv_bscales[0][1], b.block_tables, b.context_lens, b.scale, b.workspace,
                         b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    items = [0, 9, 17, 31]
    ref, _ = oracle.decode_e4m3_bs(bits(b.q[0]), b.k_caches[0].cpu().numpy(),
                                   b.v_caches[0].cpu().numpy(), b.kv_bscales[0][0].cpu().numpy(),
                                   b.kv_bscales[0][1].cpu().numpy(), b.block_tables.cpu().numpy(),
                                   b.context_lens.cpu().numpy(), b.scale, "bf16", items=items,
                                   nthreads=NTHREADS)
    assert_attn_close(out, ref, rows=items, what="70B e4m3 block scales")


# ---- the fused append over block-scaled pools

CTX_APPEND = [0, 1, 2, 9, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 129, 255, 300, 511, 1000]


def _newest_slots(case):
    bs = case["bs"]
    return np.array([case["tables"][s, (c - 1) // bs] * bs + (c - 1) % bs if c > 0 else -1
                     for s, c in enumerate(case["ctx"])], dtype=np.int64)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 128), (32, 8, 128), (64, 8, 128), (16, 1, 128),
                                      (32, 8, 64), (16, 1, 64)])
def test_block_scaled_fused_append_equals_append_then_decode(dtype, bs, Hq, Hkv, D):
    """pa_decode_append_e4m3_bs: the same codes, scales and output bits as
    pa_cache_append_e4m3_bs of the newest tokens followed by pa_decode_e4m3_bs; codes and
    scales bit-exact against the oracle's append, the output within tolerance of its
    decode.  The mix has newest tokens at offset 0 of a fresh block (NaN scale before the
    call) and later offsets."""
    seed = 760 + bs + Hq + D
    case = bs_case(CTX_APPEND, Hq, Hkv, bs, dtype, seed=seed, skip_last=True, D=D)
    B = case["B"]
    kn = inputs.randn((B, Hkv, D), dtype, seed, "cuda", stream=21) * 2
    vn = inputs.randn((B, Hkv, D), dtype, seed, "cuda", stream=22) * 0.1
    q = from_bits(case["q"], dtype).cuda()
    tables, ctx = _dev(case["tables"]), _dev(case["ctx"])
    ws = pk.new_workspace(B, Hq, Hkv, D)
    pools = lambda: [_dev(case[x]) for x in ("k8", "v8", "ks", "vs")]
    k1, v1, ks1, vs1 = pools()
    st1 = pk.new_status()
    pk.pa_cache_append_e4m3_bs(k1, v1, ks1, vs1, kn, vn, _dev(_newest_slots(case)), st1)
    o1 = torch.empty_like(q)
    pk.pa_decode_e4m3_bs(o1, q, k1, v1, ks1, vs1, tables, ctx, case["scale"], ws, st1)
    k2, v2, ks2, vs2 = pools()
    st2 = pk.new_status()
    o2 = torch.full_like(q, float("nan"))
    pk.pa_decode_append_e4m3_bs(o2, q, k2, v2, ks2, vs2, kn, vn, tables, ctx, case["scale"], ws,
                                st2)
    torch.cuda.synchronize()
    assert int(st1.item()) == 0 and int(st2.item()) == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    assert torch.equal(ks1.view(torch.int32), ks2.view(torch.int32))
    assert torch.equal(vs1.view(torch.int32), vs2.view(torch.int32))
    k8, v8, ks, vs = (case[x].copy() for x in ("k8", "v8", "ks", "vs"))
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, bits(kn), bits(vn), _newest_slots(case), dtype)
    assert np.array_equal(k2.cpu().numpy(), k8) and np.array_equal(v2.cpu().numpy(), v8)
    assert np.array_equal(ks2.cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(vs2.cpu().numpy().view(np.uint32), vs.view(np.uint32))
    ref, _ = oracle.decode_e4m3_bs(case["q"], k8, v8, ks, vs, case["tables"], case["ctx"],
                                   case["scale"], dtype, nthreads=NTHREADS)
    assert_attn_close(o2, ref, what="e4m3 block-scaled fused append %s D%d bs%d %d/%d" % (
        dtype, D, bs, Hq, Hkv))


def test_block_scaled_fused_append_llama70b_layer_full_size():
    """A full-size 70B-shape layer over block-scaled 8-bit pools: the fused append of every
    sequence's newest token against the oracle's append (codes and scales bit-exact) and
    decode (sampled sequences)."""
    b = wl.build(inputs.LLAMA70B, layers=1, kv8="block")
    k8, v8 = b.k_caches[0].cpu().numpy(), b.v_caches[0].cpu().numpy()
    ks, vs = (x.cpu().numpy() for x in b.kv_bscales[0])
    pk.pa_decode_append_e4m3_bs(b.out[0], b.q[0], b.k_caches[0], b.v_caches[0],
                                b.kv_bscales[0][0], b.kv_bscales[0][1], b.k_new[0], b.v_new[0],
                                b.block_tables, b.context_lens, b.scale, b.workspace, b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, bits(b.k_new[0]), bits(b.v_new[0]),
                                b.slot_mapping.cpu().numpy(), "bf16")
    assert np.array_equal(b.k_caches[0].cpu().numpy(), k8)
    assert np.array_equal(b.v_caches[0].cpu().numpy(), v8)
    assert np.array_equal(b.kv_bscales[0][0].cpu().numpy().view(np.uint32), ks.view(np.uint32))
    assert np.array_equal(b.kv_bscales[0][1].cpu().numpy().view(np.uint32), vs.view(np.uint32))
    items = [0, 13, 31]
    ref, _ = oracle.decode_e4m3_bs(bits(b.q[0]), k8, v8, ks, vs, b.block_tables.cpu().numpy(),
                                   b.context_lens.cpu().numpy(), b.scale, "bf16", items=items,
                                   nthreads=NTHREADS)
    assert_attn_close(b.out[0], ref, rows=items, what="70B e4m3 block-scaled fused append")


# ---- the cascade over block-scaled pools

def shared_bs_case(groups, Hq, Hkv, bs, dtype, seed, D=128):
    """test_gpu_cascade's forked sequences, their 8-bit pools filled through the oracle's
    block-scaled append: every physical slot some sequence uses is appended once (a
    shared block's tokens once for all its sharers)."""
    from tests.test_gpu_cascade import shared_case
    case = shared_case(groups, Hq, Hkv, D, bs, dtype, seed, poison=False)
    N = case["N"]
    used = sorted({int(case["tables"][i, p // bs]) * bs + p % bs
                   for i in range(case["B"]) for p in range(int(case["ctx"][i]))})
    slots = np.array(used, np.int64)
    blk, off = slots // bs, slots % bs
    rows_k = case["k"][blk, :, off, :]                     # [T, Hkv, D]
    rows_v = case["v"][blk, :, off, :]
    k8 = np.full((N, Hkv, bs, D), NAN8, np.uint8)
    v8 = np.full((N, Hkv, bs, D), NAN8, np.uint8)
    ks = np.full((N, Hkv), np.nan, np.float32)
    vs = np.full((N, Hkv), np.nan, np.float32)
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, np.ascontiguousarray(rows_k),
                                np.ascontiguousarray(rows_v), slots, dtype)
    case.update(k8=k8, v8=v8, ks=ks, vs=vs)
    return case


def run_cascade_bs(case, plan):
    q = from_bits(case["q"], case["dtype"]).cuda()
    prefix, members, plens = plan
    out = torch.full_like(q, float("nan"))
    ws = pk.new_cascade_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)
    st = pk.new_status()
    pk.pa_decode_cascade_e4m3_bs(out, q, _dev(case["k8"]), _dev(case["v8"]), _dev(case["ks"]),
                                 _dev(case["vs"]), _dev(case["tables"]), _dev(case["ctx"]),
                                 _dev(prefix), _dev(members), _dev(plens), case["scale"], ws, st)
    torch.cuda.synchronize()
    return out, int(st.item())


CASCADE_GROUPS = [(40, [3, 0, 17, 1]), (0, [5]), (33, [0, 0]),
                  (64, [1, 2, 3, 4, 5, 6, 7, 8, 9]), (200, [30]), (16, [100, 1, 16]),
                  (1, [0, 2])]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv,width,D", [(8, 2, 2, 128), (8, 2, 4, 128), (32, 8, 2, 128),
                                            (4, 4, 8, 128), (4, 4, 16, 128), (16, 1, 1, 128),
                                            (8, 2, 4, 64), (4, 4, 16, 64)])
def test_block_scaled_cascade_matches_oracle(dtype, bs, Hq, Hkv, width, D):
    case = shared_bs_case(CASCADE_GROUPS, Hq, Hkv, bs, dtype, seed=780 + bs + Hq + width + D, D=D)
    plan = wl.plan_cascade(case["tables"], case["ctx"], bs, Hq // Hkv, width)
    out, st = run_cascade_bs(case, plan)
    assert st == 0
    assert len(plan[2]) > 0 and (plan[0] > 0).sum() > 8      # sharing actually exercised
    ref, _ = oracle.decode_e4m3_bs(case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                   case["tables"], case["ctx"], case["scale"], dtype,
                                   nthreads=NTHREADS)
    assert_attn_close(out, ref, what="e4m3 block-scaled cascade %s D%d bs%d %d/%d w%d" % (
        dtype, D, bs, Hq, Hkv, width))


def test_block_scaled_cascade_without_chunks_is_decode_and_repeats_bit_identical():
    case = shared_bs_case(CASCADE_GROUPS, 32, 8, 16, "bf16", seed=790)
    B = case["B"]
    none = (np.zeros(B, np.int32), np.zeros((0, 2), np.int32), np.zeros(0, np.int32))
    a, st = run_cascade_bs(case, none)
    assert st == 0
    ref, _ = run_bs(case)
    assert torch.equal(a.view(torch.int16), ref.view(torch.int16))   # suffix pass == decode
    plan = wl.plan_cascade(case["tables"], case["ctx"], 16, 4, 4)
    b1, _ = run_cascade_bs(case, plan)
    b2, _ = run_cascade_bs(case, plan)
    assert torch.equal(b1.view(torch.int16), b2.view(torch.int16))


def test_block_scaled_cascade_rejects_chunks_over_16_rows():
    case = shared_bs_case(CASCADE_GROUPS[:1], 8, 2, 16, "f16", seed=795)
    plan = wl.plan_cascade(case["tables"], case["ctx"], 16, 4, 8)      # 32 query rows
    with pytest.raises(pk.PagedKVError):
        run_cascade_bs(case, plan)
