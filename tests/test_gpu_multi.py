"""GPU parity of pa_decode_multi (q_len new tokens per sequence, causal among them)
against the CPU oracle, through the C ABI.

Attention: |gpu - oracle| <= 2e-3 + 1e-2*|oracle| per element; invariants bit-exact.
"""
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


def _multi_q(case, q_len, seed):
    return bits(inputs.randn((case["B"], q_len, case["Hq"], case["D"]), case["dtype"], seed,
                             stream=11))


def run_multi(case, q, device="cuda"):
    dt = case["dtype"]
    qd = from_bits(q, dt).to(device)
    k = from_bits(case["k"], dt).to(device)
    v = from_bits(case["v"], dt).to(device)
    tables = torch.from_numpy(np.ascontiguousarray(case["tables"])).to(device)
    ctx = torch.from_numpy(np.ascontiguousarray(case["ctx"])).to(device)
    out = torch.full_like(qd, float("nan"))
    ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)
    st = pk.new_status()
    pk.pa_decode_multi(out, qd, k, v, tables, ctx, case["scale"], ws, st)
    torch.cuda.synchronize()
    return out, int(st.item())


CTX_MIX = [0, 1, 2, 3, 15, 16, 17, 63, 64, 65, 200, 513, 1000, 2047]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv,q_len", [(8, 2, 2), (8, 2, 4), (32, 8, 3), (64, 8, 2),
                                          (16, 16, 8), (4, 1, 3), (2, 2, 16),
                                          # 17..64 query rows per kv head: the tcgen05 kernel
                                          (64, 8, 4), (64, 8, 8), (32, 8, 16), (24, 8, 6)])
def test_multi_shape_sweep(dtype, D, bs, Hq, Hkv, q_len):
    case = make_case(len(CTX_MIX), Hq, Hkv, D, bs, CTX_MIX, dtype=dtype,
                     seed=300 + D + bs + Hq + q_len)
    q = _multi_q(case, q_len, 300 + q_len)
    out, st = run_multi(case, q)
    assert st == 0
    ref, _ = oracle.decode_multi(q, case["k"], case["v"], case["tables"], case["ctx"],
                                 case["scale"], dtype, nthreads=NTHREADS)
    assert_attn_close(out, ref, what="multi %s D%d bs%d %d/%d q_len %d" % (dtype, D, bs, Hq, Hkv,
                                                                           q_len))
    got = out.float().cpu()
    assert not got[0].abs().max().item()                   # ctx 0: all rows zero
    assert not got[1, :q_len - 1].abs().max().item()       # ctx 1: only the last token sees one


def test_multi_q_len_1_gives_the_bits_of_pa_decode():
    ctx = [700, 33, 1, 2048, 129, 0, 64, 4097]
    case = make_case(len(ctx), 32, 8, 128, 16, ctx, dtype="bf16", seed=310)
    q = _multi_q(case, 1, 310)
    out, _ = run_multi(case, q)
    qd = from_bits(q[:, 0], "bf16").cuda()
    k = from_bits(case["k"], "bf16").cuda()
    v = from_bits(case["v"], "bf16").cuda()
    ref = torch.empty_like(qd)
    ws = pk.new_workspace(case["B"], 32, 8, 128)
    pk.pa_decode(ref, qd, k, v, torch.from_numpy(case["tables"]).cuda(),
                 torch.from_numpy(case["ctx"]).cuda(), case["scale"], ws)
    torch.cuda.synchronize()
    assert torch.equal(out[:, 0].contiguous().view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("bs", [8, 16])
def test_multi_physical_permutation_is_bit_identical(bs):
    ctx = [700, 33, 3, 2048, 129, 0, 64]
    a = make_case(len(ctx), 16, 4, 128, bs, ctx, dtype="f16", seed=320)
    q = _multi_q(case=a, q_len=4, seed=320)
    out_a, _ = run_multi(a, q)
    perm = np.random.default_rng(9).permutation(a["N"])
    b = dict(a)
    b["k"], b["v"] = np.empty_like(a["k"]), np.empty_like(a["v"])
    b["k"][perm], b["v"][perm] = a["k"], a["v"]
    b["tables"] = np.where(a["tables"] >= 0, perm[np.clip(a["tables"], 0, None)],
                           a["tables"]).astype(np.int32)
    out_b, _ = run_multi(b, q)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))


def test_multi_rejects_more_than_64_query_rows_per_kv_head():
    case = make_case(2, 32, 8, 128, 16, [40, 50], dtype="f16", seed=330)
    q = _multi_q(case, 17, 330)                            # group 4 x 17 tokens = 68 rows
    with pytest.raises(pk.PagedKVError, match="unsupported"):
        run_multi(case, q)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_wide_group_single_token(dtype):
    """One new token per sequence with 32 q heads per kv head (more than the mma.sync
    kernel's 16 columns): pa_decode runs on the tcgen05 kernel."""
    ctx = [0, 1, 17, 700, 2048, 129, 4097, 64, 3, 1500]
    case = make_case(len(ctx), 64, 2, 128, 16, ctx, dtype=dtype, seed=335)
    qd = from_bits(case["q"], dtype).cuda()
    out = torch.full_like(qd, float("nan"))
    st = pk.new_status()
    pk.pa_decode(out, qd, from_bits(case["k"], dtype).cuda(), from_bits(case["v"], dtype).cuda(),
                 torch.from_numpy(case["tables"]).cuda(), torch.from_numpy(case["ctx"]).cuda(),
                 case["scale"], pk.new_workspace(case["B"], 64, 2, 128), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], dtype, nthreads=NTHREADS)
    assert_attn_close(out, ref, what="group 32 %s" % dtype)


def test_wide_repeat_runs_are_bit_identical_and_permutation_invariant():
    ctx = [900, 33, 3, 4100, 129, 0, 64, 2500]
    a = make_case(len(ctx), 64, 8, 128, 16, ctx, dtype="bf16", seed=336)
    q = _multi_q(a, 8, 336)
    o1, st1 = run_multi(a, q)
    o2, st2 = run_multi(a, q)
    assert st1 == 0 and st2 == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    perm = np.random.default_rng(11).permutation(a["N"])
    b = dict(a)
    b["k"], b["v"] = np.empty_like(a["k"]), np.empty_like(a["v"])
    b["k"][perm], b["v"][perm] = a["k"], a["v"]
    b["tables"] = np.where(a["tables"] >= 0, perm[np.clip(a["tables"], 0, None)],
                           a["tables"]).astype(np.int32)
    o3, _ = run_multi(b, q)
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))


def test_multi_llama8b_shape_four_new_tokens_full_size():
    """The 8B-shape batch (64 seqs, 32/8 heads, d128, fp16, ctx U[128,2048]) with 4 new
    tokens per sequence: 16 query rows per kv head, every sequence checked."""
    b = wl.build(inputs.LLAMA8B)
    q_len = 4
    q = inputs.randn((64, q_len, 32, 128), "f16", 1, "cuda", stream=77)
    out = torch.empty_like(q)
    pk.pa_decode_multi(out, q, b.k_caches[0], b.v_caches[0], b.block_tables, b.context_lens,
                       b.scale, b.workspace, b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    ref, _ = oracle.decode_multi(bits(q), bits(b.k_caches[0]), bits(b.v_caches[0]),
                                 b.block_tables.cpu().numpy(), b.context_lens.cpu().numpy(),
                                 b.scale, "f16", nthreads=NTHREADS)
    assert_attn_close(out, ref, what="llama8b q_len 4")


def test_multi_llama70b_shape_two_new_tokens_two_layers_sampled():
    """The bench's q_len-2 step at full size (70B shape, 16 query rows per kv head, warp
    pairs splitting the columns): 2 layers through run_step, sequences sampled."""
    b = wl.build(inputs.LLAMA70B, layers=2, q_len=2)
    pre = [(bits(b.k_caches[l]), bits(b.v_caches[l])) for l in range(2)]
    wl.run_step(b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    items = [0, 5, 11, 17, 23, 31]
    for l in range(2):
        hk, hv = pre[l]
        oracle.cache_append(hk, hv, bits(b.k_new[l]), bits(b.v_new[l]),
                            b.slot_mapping.cpu().numpy())
        assert np.array_equal(bits(b.k_caches[l]), hk) and np.array_equal(bits(b.v_caches[l]), hv)
        ref, _ = oracle.decode_multi(bits(b.q[l]), hk, hv, b.block_tables.cpu().numpy(),
                                     b.context_lens.cpu().numpy(), b.scale, "bf16", items=items,
                                     nthreads=NTHREADS)
        assert_attn_close(b.out[l], ref, rows=items, what="70B q_len 2 layer %d" % l)


@pytest.mark.parametrize("q_len", [4, 8])
def test_multi_llama70b_shape_wide_two_layers_sampled(q_len):
    """The 70B shape with 4 and 8 new tokens per sequence (32 and 64 query rows per kv
    head, the tcgen05 kernel) at full size: 2 layers through run_step, sequences sampled."""
    b = wl.build(inputs.LLAMA70B, layers=2, q_len=q_len)
    pre = [(bits(b.k_caches[l]), bits(b.v_caches[l])) for l in range(2)]
    wl.run_step(b)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    items = [0, 7, 13, 22, 31]
    for l in range(2):
        hk, hv = pre[l]
        oracle.cache_append(hk, hv, bits(b.k_new[l]), bits(b.v_new[l]),
                            b.slot_mapping.cpu().numpy())
        ref, _ = oracle.decode_multi(bits(b.q[l]), hk, hv, b.block_tables.cpu().numpy(),
                                     b.context_lens.cpu().numpy(), b.scale, "bf16", items=items,
                                     nthreads=NTHREADS)
        assert_attn_close(b.out[l], ref, rows=items, what="70B q_len %d layer %d" % (q_len, l))
