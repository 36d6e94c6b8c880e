"""GPU parity of pa_decode_cascade (sequences that share a KV prefix decoded with the
shared part read once per chunk of sharers) against the CPU oracle, through the C ABI.

The oracle is plain decode over each sequence's whole context: splitting the softmax at
the prefix boundary and recombining is exact algebra, so the cascade must meet the
same tolerance, |gpu - oracle| <= 2e-3 + 1e-2*|oracle|, and be deterministic.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle.cow import RefBlockManager
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200 import pagedkv as pk
from paged_kv_cache_348_b200 import workload as wl
from tests.helpers import NAN_BITS, bits, from_bits
from tests.test_gpu_parity import assert_attn_close

pytestmark = pytest.mark.gpu

NTHREADS = 8


def shared_case(groups, Hq, Hkv, D, bs, dtype, seed, poison=True):
    """groups: list of (prefix_tokens, [private tokens of each member]).  Members of a
    group fork one root holding the prefix, then append their private tokens (copy on
    write of a shared partial block, as the block manager does)."""
    rng = np.random.default_rng(seed)
    need = sum(-(-p // bs) + sum(-(-(p % bs + x) // bs) + 1 for x in priv) for p, priv in groups)
    N = need + 8
    bm = RefBlockManager(N, bs, inputs.pool_order(N, seed))
    sids = []
    for p, priv in groups:
        root = bm.new_seq(p)
        kids = [root] + [bm.fork(root) for _ in range(len(priv) - 1)]
        for sid, x in zip(kids, priv):
            for _ in range(x):
                bm.append_slot(sid)
            sids.append(sid)
    B = len(sids)
    ctx = np.array([bm.ctx[s] for s in sids], dtype=np.int32)
    M = max(1, max(len(bm.tables[s]) for s in sids))
    tables = np.full((B, M), -5, dtype=np.int32)
    for i, s in enumerate(sids):
        tables[i, :len(bm.tables[s])] = bm.tables[s]
    q = bits(inputs.randn((B, Hq, D), dtype, seed, stream=1))
    k = bits(inputs.randn((N, Hkv, bs, D), dtype, seed, stream=2))
    v = bits(inputs.randn((N, Hkv, bs, D), dtype, seed, stream=3))
    if poison:
        used = np.zeros((N, bs), dtype=bool)
        for i, s in enumerate(sids):
            for t in range(int(ctx[i])):
                used[bm.tables[s][t // bs], t % bs] = True
        k.transpose(0, 2, 1, 3)[~used] = NAN_BITS[dtype]
        v.transpose(0, 2, 1, 3)[~used] = NAN_BITS[dtype]
    _ = rng
    return dict(q=q, k=k, v=v, tables=tables, ctx=ctx, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs,
                dtype=dtype, N=N, scale=1.0 / np.sqrt(D))


def run_cascade(case, plan=None):
    dt = case["dtype"]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q = from_bits(case["q"], dt).cuda()
    k = from_bits(case["k"], dt).cuda()
    v = from_bits(case["v"], dt).cuda()
    if plan is None:
        plan = wl.plan_cascade(case["tables"], case["ctx"], case["bs"], case["Hq"] // case["Hkv"])
    prefix, members, plens = plan
    out = torch.full_like(q, float("nan"))
    ws = pk.new_cascade_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
    ws.fill_(0xFF)
    st = pk.new_status()
    pk.pa_decode_cascade(out, q, k, v, dev(case["tables"]), dev(case["ctx"]), dev(prefix),
                         dev(members), dev(plens), case["scale"], ws, st)
    torch.cuda.synchronize()
    return out, int(st.item()), plan


GROUPS = [(40, [3, 0, 17, 1]), (0, [5]), (33, [0, 0]), (64, [1, 2, 3, 4, 5, 6, 7, 8, 9]),
          (200, [30]), (16, [100, 1, 16]), (1, [0, 2])]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 8, 16, 32])
@pytest.mark.parametrize("Hq,Hkv,width", [(8, 2, 2), (8, 2, 4), (32, 8, 2), (4, 4, 8), (4, 4, 16),
                                          (16, 1, 1),
                                          # chunks wider than 16 query rows: tcgen05 prefix pass
                                          (32, 8, 8), (8, 2, 16), (16, 1, 4)])
def test_cascade_matches_oracle(dtype, D, bs, Hq, Hkv, width):
    case = shared_case(GROUPS, Hq, Hkv, D, bs, dtype, seed=400 + D + bs + Hq)
    plan = wl.plan_cascade(case["tables"], case["ctx"], bs, Hq // Hkv, width)
    out, st, plan = run_cascade(case, plan)
    assert st == 0
    assert len(plan[2]) > 0 and (plan[0] > 0).sum() > 8      # sharing actually exercised
    ref, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], dtype, nthreads=NTHREADS)
    assert_attn_close(out, ref, what="cascade %s D%d bs%d %d/%d" % (dtype, D, bs, Hq, Hkv))


def test_cascade_without_chunks_is_plain_decode_and_runs_repeat_bit_identical():
    case = shared_case(GROUPS, 32, 8, 128, 16, "bf16", seed=450)
    B = case["B"]
    none = (np.zeros(B, np.int32), np.zeros((0, 2), np.int32), np.zeros(0, np.int32))
    a, st, _ = run_cascade(case, none)
    assert st == 0
    ref = torch.empty_like(a)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pk.pa_decode(ref, from_bits(case["q"], "bf16").cuda(), from_bits(case["k"], "bf16").cuda(),
                 from_bits(case["v"], "bf16").cuda(), dev(case["tables"]), dev(case["ctx"]),
                 case["scale"], pk.new_workspace(B, 32, 8, 128))
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), ref.view(torch.int16))   # suffix pass == decode
    b1, _, _ = run_cascade(case)
    b2, _, _ = run_cascade(case)
    assert torch.equal(b1.view(torch.int16), b2.view(torch.int16))


def test_cascade_shared_prefix_workload_full_size():
    """The shared-prefix workload: 16 prompts x 8 samples, 2048 shared tokens each, 0..512
    private tokens, 32 q / 8 kv heads, d128, fp16."""
    b = wl.build_prefix_decode()
    tables, ctx = b.block_tables.cpu().numpy(), b.context_lens.cpu().numpy()
    prefix, members, plens = wl.plan_cascade(tables, ctx, b.block_size, 4)
    assert (prefix == inputs.PREFIX_LEN).all() and len(plens) == 16       # 1 chunk a prompt
    out = torch.empty_like(b.q[0])
    ws = pk.new_cascade_workspace(128, 32, 8, 128)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    pk.pa_decode_cascade(out, b.q[0], b.k_caches[0], b.v_caches[0], b.block_tables,
                         b.context_lens, dev(prefix), dev(members), dev(plens), b.scale, ws,
                         b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    items = list(range(0, 128, 3)) + [127]
    ref, _ = oracle.decode(bits(b.q[0]), bits(b.k_caches[0]), bits(b.v_caches[0]), tables, ctx,
                           b.scale, "f16", items=items, nthreads=NTHREADS)
    assert_attn_close(out, ref, rows=items, what="prefix workload cascade")


def test_cascade_padding_and_invalid_members_are_ignored():
    case = shared_case([(48, [2, 5, 0])], 8, 2, 64, 16, "f16", seed=460)
    prefix, members, plens = wl.plan_cascade(case["tables"], case["ctx"], 16, 4, width=4)
    assert members.shape == (1, 4) and members[0, 3] == -1
    members = members.copy()
    members[0, 3] = 1000                                  # out of range: a padding slot
    out, st, _ = run_cascade(case, (prefix, members, plens))
    assert st == 0
    ref, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                           case["scale"], "f16")
    assert_attn_close(out, ref, what="padding slots")
