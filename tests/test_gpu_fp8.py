"""GPU parity of the 8-bit E4M3 KV cache through the C ABI: pa_cache_append_e4m3 bit-exact
against the oracle's quantising append, pa_decode_e4m3 within |gpu - oracle| <= 2e-3 +
1e-2*|oracle| of the oracle's fp64 decode over the same codes, block-permutation
invariance and NaN-coded free slots that change no output bit."""
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


def e4m3_case(ctx, Hq, Hkv, bs, dtype, seed, ks=0.02, vs=0.03, shuffle=True, poison=True, D=128):
    case = make_case(len(ctx), Hq, Hkv, D, bs, ctx, dtype=dtype, seed=seed, shuffle=shuffle,
                     poison=False)
    shape = case["k"].shape
    case["k8"] = inputs.randn_e4m3(shape, ks, seed, stream=31).numpy()
    case["v8"] = inputs.randn_e4m3(shape, vs, seed, stream=32).numpy()
    case["ks"], case["vs"] = ks, vs
    if poison:
        used = np.zeros((case["N"], bs), dtype=bool)
        for i, s in enumerate(case["sids"]):
            for t in range(int(case["ctx"][i])):
                used[case["bm"].tables[s][t // bs], t % bs] = True
        case["k8"].transpose(0, 2, 1, 3)[~used] = NAN8
        case["v8"].transpose(0, 2, 1, 3)[~used] = NAN8
    return case


def run_e4m3(case):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q = from_bits(case["q"], case["dtype"]).cuda()
    out = torch.full_like(q, float("nan"))
    ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)
    st = pk.new_status()
    pk.pa_decode_e4m3(out, q, dev(case["k8"]), dev(case["v8"]), case["ks"], case["vs"],
                      dev(case["tables"]), dev(case["ctx"]), case["scale"], ws, st)
    torch.cuda.synchronize()
    return out, int(st.item())


CTX_MIX = [0, 1, 2, 15, 16, 17, 31, 63, 64, 65, 100, 129, 255, 300, 511, 1000, 2047]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (32, 8), (64, 8), (16, 1)])
def test_e4m3_decode_matches_oracle(dtype, D, bs, Hq, Hkv):
    case = e4m3_case(CTX_MIX, Hq, Hkv, bs, dtype, seed=600 + bs + Hq + D, D=D)
    out, st = run_e4m3(case)
    assert st == 0
    ref, _ = oracle.decode_e4m3(case["q"], case["k8"], case["v8"], case["ks"], case["vs"],
                                case["tables"], case["ctx"], case["scale"], dtype,
                                nthreads=NTHREADS)
    assert_attn_close(out, ref, what="e4m3 %s D%d bs%d %d/%d" % (dtype, D, bs, Hq, Hkv))
    assert not out[0].float().abs().max().item()


def test_e4m3_decode_is_block_permutation_and_poison_invariant():
    ctx = [700, 33, 1, 2048, 129, 0, 64]
    a = e4m3_case(ctx, 32, 8, 16, "bf16", seed=610, poison=True)
    out_a, _ = run_e4m3(a)
    clean = e4m3_case(ctx, 32, 8, 16, "bf16", seed=610, poison=False)
    out_c, _ = run_e4m3(clean)
    assert torch.equal(out_a.view(torch.int16), out_c.view(torch.int16))
    perm = np.random.default_rng(11).permutation(a["N"])
    b = dict(a)
    b["k8"], b["v8"] = np.empty_like(a["k8"]), np.empty_like(a["v8"])
    b["k8"][perm], b["v8"][perm] = a["k8"], a["v8"]
    b["tables"] = np.where(a["tables"] >= 0, perm[np.clip(a["tables"], 0, None)],
                           a["tables"]).astype(np.int32)
    out_b, _ = run_e4m3(b)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("scales", [(0.02, 0.03), (1.0 / 64, 0.5), (0.001, 0.001)])
def test_e4m3_append_bit_exact(dtype, scales):
    N, Hkv, bs, D, T = 40, 8, 16, 128, 37
    ks, vs = scales
    k8 = inputs.randn_e4m3((N, Hkv, bs, D), 0.05, 62, "cuda", 1)
    v8 = inputs.randn_e4m3((N, Hkv, bs, D), 0.05, 62, "cuda", 2)
    kn = inputs.randn((T, Hkv, D), dtype, 62, "cuda", 3) * 3       # some codes saturate
    vn = inputs.randn((T, Hkv, D), dtype, 62, "cuda", 4)
    slots = np.random.default_rng(7).choice(N * bs, size=T, replace=False).astype(np.int64)
    slots[[2, 9]] = -1
    hk, hv = k8.cpu().numpy().copy(), v8.cpu().numpy().copy()
    oracle.cache_append_e4m3(hk, hv, bits(kn), bits(vn), slots, dtype, ks, vs)
    st = pk.new_status()
    pk.pa_cache_append_e4m3(k8, v8, kn, vn, torch.from_numpy(slots).cuda(), ks, vs, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert np.array_equal(k8.cpu().numpy(), hk) and np.array_equal(v8.cpu().numpy(), hv)


def test_e4m3_unsupported_head_dim_is_rejected():
    q = torch.zeros((2, 4, 96), dtype=torch.float16, device="cuda")
    k8 = torch.zeros((4, 4, 16, 96), dtype=torch.uint8, device="cuda")
    t = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    c = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedKVError, match="unsupported"):
        pk.pa_decode_e4m3(torch.empty_like(q), q, k8, k8, 0.1, 0.1, t, c, 0.125,
                          pk.new_workspace(2, 4, 4, 96))


def test_e4m3_llama70b_shape_step_full_size():
    """The 70B-shape batch with 8-bit pools: per layer the quantising append of the
    newest tokens then decode; 2 full-size layers, every sequence checked."""
    b = wl.build(inputs.LLAMA70B, layers=2, kv8=True)
    pre = [(b.k_caches[l].cpu().numpy().copy(), b.v_caches[l].cpu().numpy().copy())
           for l in range(2)]
    wl.run_step(b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ks, vs = b.kv_scales
    for l in range(2):
        hk, hv = pre[l]
        oracle.cache_append_e4m3(hk, hv, bits(b.k_new[l]), bits(b.v_new[l]),
                                 b.slot_mapping.cpu().numpy(), "bf16", ks, vs)
        assert np.array_equal(b.k_caches[l].cpu().numpy(), hk)
        assert np.array_equal(b.v_caches[l].cpu().numpy(), hv)
        ref, _ = oracle.decode_e4m3(bits(b.q[l]), hk, hv, ks, vs, b.block_tables.cpu().numpy(),
                                    b.context_lens.cpu().numpy(), b.scale, "bf16",
                                    nthreads=NTHREADS)
        assert_attn_close(b.out[l], ref, what="70B e4m3 layer %d" % l)


def test_e4m3_group16_llama70b_shape_full_size():
    """16 query rows per kv head with 8-bit pools at full size (128 q / 8 kv heads, the
    70B-shape lengths): the warp pairs' split columns and the end-of-portion merge of
    every ring slot, every sequence checked."""
    import dataclasses
    w = dataclasses.replace(inputs.LLAMA70B, num_q_heads=128)
    b = wl.build(w, layers=1, kv8=True)
    wl.decode_layer(b, 0)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ks, vs = b.kv_scales
    ref, _ = oracle.decode_e4m3(bits(b.q[0]), b.k_caches[0].cpu().numpy(),
                                b.v_caches[0].cpu().numpy(), ks, vs,
                                b.block_tables.cpu().numpy(), b.context_lens.cpu().numpy(),
                                b.scale, "bf16", nthreads=NTHREADS)
    assert_attn_close(b.out[0], ref, what="70B-shape group 16 e4m3")


@pytest.mark.parametrize("bs", [1, 16])
def test_e4m3_heavytail_sampled(bs):
    """The heavy-tailed batch with 8-bit pools at full size (256 sequences, lognormal
    lengths up to the clip): the quantising append then decode, sequences sampled."""
    b = wl.build(inputs.HEAVYTAIL, block_size=bs, kv8=True)
    hk, hv = b.k_caches[0].cpu().numpy().copy(), b.v_caches[0].cpu().numpy().copy()
    wl.run_step(b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ks, vs = b.kv_scales
    oracle.cache_append_e4m3(hk, hv, bits(b.k_new[0]), bits(b.v_new[0]),
                             b.slot_mapping.cpu().numpy(), "f16", ks, vs)
    assert np.array_equal(b.k_caches[0].cpu().numpy(), hk)
    assert np.array_equal(b.v_caches[0].cpu().numpy(), hv)
    ctx = b.context_lens.cpu().numpy()
    items = sorted(set([int(i) for i in np.argsort(ctx)[-4:]] + list(range(0, 256, 23))))
    ref, _ = oracle.decode_e4m3(bits(b.q[0]), hk, hv, ks, vs, b.block_tables.cpu().numpy(), ctx,
                                b.scale, "f16", items=items, nthreads=NTHREADS)
    assert_attn_close(b.out[0], ref, rows=items, what="heavytail e4m3 bs%d" % bs)
