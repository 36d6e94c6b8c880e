"""Preemption through the C ABI: a sequence's blocks saved to page-locked host memory
(pa_bm_swap_out + pa_swap_out_blocks), the pool reused and scribbled over, then the
sequence restored into fresh blocks (pa_bm_swap_in + pa_swap_in_blocks).

The saved bytes must equal the pool blocks exactly (numpy gather of the pool), and
decode after the round trip must give the bits decode gave before it: the placement of
blocks never changes a result ("Paged Attention and Memory Efficiency in Production LLM
Serving", "How PagedAttention borrows OS paging").
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200 import pagedkv as pk
from paged_kv_cache_348_b200.block_manager import BlockManager
from tests.helpers import bits

pytestmark = pytest.mark.gpu


def _decode(k, v, q, bm, sids, scale, ws):
    tables = torch.from_numpy(bm.block_tables(sids, fill=-3)).cuda()
    ctx = torch.from_numpy(bm.context_lens(sids)).cuda()
    outs = []
    st = pk.new_status()
    for l in range(len(k)):
        o = torch.empty_like(q[l])
        pk.pa_decode(o, q[l], k[l], v[l], tables, ctx, scale, ws, st)
        outs.append(o)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return outs


@pytest.mark.parametrize("dtype,bs", [("bf16", 16), ("f16", 8), ("f16", 1)])
def test_swap_round_trip_restores_decode_bits(dtype, bs):
    L, Hq, Hkv, D = 2, 32, 8, 128
    ctx = [700, 33, 2048, 1, 129, 500]
    N = sum(-(-c // bs) for c in ctx) * 2 + 64
    bm = BlockManager(N, bs, inputs.pool_order(N, 91))
    sids = [bm.allocate(c) for c in ctx]
    child = bm.fork(sids[0])                               # shares seq 0's blocks
    for _ in range(20):
        bm.append_token(child)                             # copy on write of the partial block
    sids.append(child)
    shape = (N, Hkv, bs, D)
    k = [inputs.randn(shape, dtype, 91, "cuda", stream=10 + 2 * l) for l in range(L)]
    v = [inputs.randn(shape, dtype, 91, "cuda", stream=11 + 2 * l) for l in range(L)]
    q = [inputs.randn((len(sids), Hq, D), dtype, 91, "cuda", stream=30 + l) for l in range(L)]
    ws = pk.new_workspace(len(sids), Hq, Hkv, D)
    scale = 1.0 / np.sqrt(D)
    before = _decode(k, v, q, bm, sids, scale, ws)

    victims = [sids[0], sids[2], child]                    # seq 0 shares blocks with child
    saved = {}
    for s in victims:
        blocks = bm.swap_out(s)
        dev_blocks = torch.from_numpy(blocks).cuda()
        buf = torch.empty(pk.swap_buffer_bytes(k, len(blocks)), dtype=torch.uint8,
                          pin_memory=True)
        pk.pa_swap_out_blocks(buf, k, v, dev_blocks)
        torch.cuda.synchronize()
        # the saved bytes: [layer][K, V][i][block] of exactly these pool blocks
        want = np.concatenate([bits(pool)[blocks].reshape(-1).view(np.uint8)
                               for l in range(L) for pool in (k[l], v[l])])
        assert np.array_equal(buf.numpy(), want)
        saved[s] = buf
    # the pool reuses the released blocks: a filler takes every free block, and every
    # block nobody holds now is scribbled over (NaN)
    filler = bm.allocate(bm.free_blocks * bs)
    held = set()
    for s in sids + [filler]:
        if s not in victims:
            held.update(bm.table(s))
    loose = torch.tensor(sorted(set(range(N)) - (held - set(bm.table(filler)))), device="cuda")
    for l in range(L):
        k[l][loose] = float("nan")
        v[l][loose] = float("nan")
    bm.release(filler)
    for s in victims:
        fresh = bm.swap_in(s)
        pk.pa_swap_in_blocks(k, v, torch.from_numpy(fresh).cuda(), saved[s])
    after = _decode(k, v, q, bm, sids, scale, ws)
    for l in range(L):
        assert torch.equal(before[l].view(torch.int16), after[l].view(torch.int16))


def test_swap_refuses_pageable_host_memory():
    k = [torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")]
    v = [torch.zeros_like(k[0])]
    blocks = torch.tensor([1, 2], dtype=torch.int32, device="cuda")
    pageable = torch.empty(pk.swap_buffer_bytes(k, 2), dtype=torch.uint8)
    with pytest.raises(pk.PagedKVError, match="invalid argument"):
        pk.pa_swap_out_blocks(pageable, k, v, blocks)
    dev = torch.empty(pk.swap_buffer_bytes(k, 2), dtype=torch.uint8, device="cuda")
    pk.pa_swap_out_blocks(dev, k, v, blocks)               # device memory is fine
    torch.cuda.synchronize()
