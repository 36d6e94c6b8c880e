"""GPU parity of pa_decode_append (the newest token's cache append fused into decode)
through the C ABI: the same output bits and the same cache bytes as pa_cache_append of
the newest tokens followed by pa_decode, and the cache bit-exact against the oracle's
append, the output within tolerance of the oracle's decode."""
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

CTX_MIX = [0, 1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 129, 255, 300, 511, 1000]


def _newest_slots(case):
    bs = case["bs"]
    return np.array([case["tables"][s, (c - 1) // bs] * bs + (c - 1) % bs if c > 0 else -1
                     for s, c in enumerate(case["ctx"])], dtype=np.int64)


def _run_both(case, seed):
    dt, B, Hkv, D = case["dtype"], case["B"], case["Hkv"], case["D"]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    kn = inputs.randn((B, Hkv, D), dt, seed, "cuda", stream=21)
    vn = inputs.randn((B, Hkv, D), dt, seed, "cuda", stream=22)
    q = from_bits(case["q"], dt).cuda()
    tables, ctx = dev(case["tables"]), dev(case["ctx"])
    ws = pk.new_workspace(B, case["Hq"], Hkv, D)
    # separate calls
    k1, v1 = from_bits(case["k"], dt).cuda(), from_bits(case["v"], dt).cuda()
    st1 = pk.new_status()
    pk.pa_cache_append(k1, v1, kn, vn, dev(_newest_slots(case)), st1)
    o1 = torch.empty_like(q)
    pk.pa_decode(o1, q, k1, v1, tables, ctx, case["scale"], ws, st1)
    # fused
    k2, v2 = from_bits(case["k"], dt).cuda(), from_bits(case["v"], dt).cuda()
    st2 = pk.new_status()
    o2 = torch.full_like(q, float("nan"))
    pk.pa_decode_append(o2, q, k2, v2, kn, vn, tables, ctx, case["scale"], ws, st2)
    torch.cuda.synchronize()
    return (o1, k1, v1, int(st1.item())), (o2, k2, v2, int(st2.item())), (kn, vn)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (32, 8), (64, 8), (16, 1),
                                    # 9+ query rows a kv head: the tcgen05 kernel, which
                                    # writes the new rows before reading their tile
                                    (12, 1), (32, 1), (64, 1)])
def test_fused_append_equals_append_then_decode(dtype, D, bs, Hq, Hkv):
    case = make_case(len(CTX_MIX), Hq, Hkv, D, bs, CTX_MIX, dtype=dtype,
                     seed=500 + D + bs + Hq)
    sep, fused, (kn, vn) = _run_both(case, 500 + bs)
    assert sep[3] == 0 and fused[3] == 0
    assert torch.equal(sep[0].view(torch.int16), fused[0].view(torch.int16))   # output bits
    assert torch.equal(sep[1].view(torch.int16), fused[1].view(torch.int16))   # K cache
    assert torch.equal(sep[2].view(torch.int16), fused[2].view(torch.int16))   # V cache
    # and against the oracle
    hk, hv = case["k"].copy(), case["v"].copy()
    oracle.cache_append(hk, hv, bits(kn), bits(vn), _newest_slots(case))
    assert np.array_equal(bits(fused[1]), hk) and np.array_equal(bits(fused[2]), hv)
    ref, _ = oracle.decode(case["q"], hk, hv, case["tables"], case["ctx"], case["scale"], dtype,
                           nthreads=8)
    assert_attn_close(fused[0], ref, what="fused append %s D%d bs%d %d/%d" % (dtype, D, bs, Hq,
                                                                              Hkv))


def test_fused_append_llama70b_two_layers_full_size():
    b = wl.build(inputs.LLAMA70B, layers=2)
    pre = [(bits(b.k_caches[l]), bits(b.v_caches[l])) for l in range(2)]
    for l in range(2):
        pk.pa_decode_append(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], b.k_new[l],
                            b.v_new[l], b.block_tables, b.context_lens, b.scale, b.workspace,
                            b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    for l in range(2):
        hk, hv = pre[l]
        oracle.cache_append(hk, hv, bits(b.k_new[l]), bits(b.v_new[l]),
                            b.slot_mapping.cpu().numpy())
        assert np.array_equal(bits(b.k_caches[l]), hk) and np.array_equal(bits(b.v_caches[l]), hv)
        ref, _ = oracle.decode(bits(b.q[l]), hk, hv, b.block_tables.cpu().numpy(),
                               b.context_lens.cpu().numpy(), b.scale, "bf16", nthreads=8)
        assert_attn_close(b.out[l], ref, what="70B fused layer %d" % l)


def test_fused_append_bad_block_id_is_flagged_and_not_written():
    case = make_case(3, 8, 2, 128, 16, [40, 50, 60], dtype="f16", seed=520)
    case["tables"][1, 3] = case["N"] + 9                  # block of position 49
    sep, fused, _ = _run_both(case, 520)
    assert fused[3] & pk.DEV_BAD_BLOCK_ID
    assert sep[3] & pk.DEV_BAD_SLOT                        # the separate append skips it too
    assert torch.equal(sep[1].view(torch.int16), fused[1].view(torch.int16))
    assert torch.equal(sep[2].view(torch.int16), fused[2].view(torch.int16))
    assert torch.equal(sep[0][[0, 2]].view(torch.int16), fused[0][[0, 2]].view(torch.int16))


def test_fused_append_group16_llama70b_shape_full_size():
    """pa_decode_append with 16 query rows per kv head (128 q / 8 kv heads) at full size:
    both warps of the newest token's unit patch their tile, one writes the cache."""
    import dataclasses
    w = dataclasses.replace(inputs.LLAMA70B, num_q_heads=128)
    b = wl.build(w, layers=1)
    hk, hv = bits(b.k_caches[0]), bits(b.v_caches[0])
    pk.pa_decode_append(b.out[0], b.q[0], b.k_caches[0], b.v_caches[0], b.k_new[0], b.v_new[0],
                        b.block_tables, b.context_lens, b.scale, b.workspace, b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    oracle.cache_append(hk, hv, bits(b.k_new[0]), bits(b.v_new[0]), b.slot_mapping.cpu().numpy())
    assert np.array_equal(bits(b.k_caches[0]), hk) and np.array_equal(bits(b.v_caches[0]), hv)
    ref, _ = oracle.decode(bits(b.q[0]), hk, hv, b.block_tables.cpu().numpy(),
                           b.context_lens.cpu().numpy(), b.scale, "bf16", nthreads=8)
    assert_attn_close(b.out[0], ref, what="70B-shape group 16 fused append")
