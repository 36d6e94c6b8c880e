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


def bs_case(ctx, Hq, Hkv, bs, dtype, seed, q_len=1):
    """8-bit pools filled the way a server fills them: every cached token appended in
    position order through the oracle's block-scaled append (so each block's scale is the
    one its first token fixed); free blocks and tails hold NaN codes."""
    case = make_case(len(ctx), Hq, Hkv, 128, bs, ctx, dtype=dtype, seed=seed, poison=False)
    N = case["N"]
    k8 = np.full((N, Hkv, bs, 128), NAN8, np.uint8)
    v8 = np.full((N, Hkv, bs, 128), NAN8, np.uint8)
    ks = np.full((N, Hkv), np.nan, np.float32)
    vs = np.full((N, Hkv), np.nan, np.float32)
    slots = []
    for i, s in enumerate(case["sids"]):
        t = case["bm"].tables[s]
        slots += [t[p // bs] * bs + p % bs for p in range(int(ctx[i]))]
    slots = np.array(slots, np.int64)
    T = len(slots)
    rng_k = bits(inputs.randn((T, Hkv, 128), dtype, seed, stream=41))
    rng_v = bits(inputs.randn((T, Hkv, 128), dtype, seed, stream=42))
    oracle.cache_append_e4m3_bs(k8, v8, ks, vs, rng_k, rng_v, slots, dtype)
    case.update(k8=k8, v8=v8, ks=ks, vs=vs)
    if q_len > 1:
        case["q"] = bits(inputs.randn((len(ctx), q_len, Hq, 128), dtype, seed, stream=43))
    return case


def run_bs(case):
    q = from_bits(case["q"], case["dtype"]).cuda()
    out = torch.full_like(q, float("nan"))
    ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], 128)
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
@pytest.mark.parametrize("Hq,Hkv,q_len", [(4, 4, 1), (32, 8, 1), (64, 8, 1), (16, 1, 1),
                                          (32, 8, 4), (64, 8, 2), (8, 8, 3)])
def test_block_scaled_decode_matches_oracle(dtype, bs, Hq, Hkv, q_len):
    case = bs_case(CTX_MIX, Hq, Hkv, bs, dtype, seed=710 + bs + Hq + q_len, q_len=q_len)
    out, st = run_bs(case)
    assert st == 0
    ref, _ = oracle.decode_e4m3_bs(case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                   case["tables"], case["ctx"], case["scale"], dtype,
                                   nthreads=NTHREADS)
    assert_attn_close(out, ref, what="e4m3 block scales %s bs%d %d/%d q_len %d" % (
        dtype, bs, Hq, Hkv, q_len))
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
