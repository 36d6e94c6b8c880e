"""Device-resident decode batches for the measured workloads.

Builds, from the seeded generators in ``inputs`` and the host ``BlockManager``:
per-layer K/V pools, one block table for all layers, context lengths, the newest
token's q / k / v per layer and its slot mapping, output buffers, the decode
workspace and a device status word.

A decode step (``run_step``) is, for every layer: pa_cache_append of the newest
token of every sequence, then pa_decode over all cached tokens (the newest one
included).  Copy-on-write pairs, when the block manager produced some, are copied
with one pa_copy_blocks call over all layers first.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

from . import inputs
from . import pagedkv as pk
from .block_manager import BlockManager


@dataclasses.dataclass
class DecodeBatch:
    w: inputs.Workload
    block_size: int
    bm: BlockManager
    sids: list
    num_blocks: int
    k_caches: list
    v_caches: list
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    slot_mapping: torch.Tensor
    q: list
    k_new: list
    v_new: list
    out: list
    workspace: torch.Tensor
    status: torch.Tensor
    cow_pairs: torch.Tensor | None
    scale: float
    q_len: int = 1
    cascade: tuple | None = None     # (prefix_lens, chunk_members, chunk_prefix_lens) on device
    kv_scales: tuple | None = None   # (k_scale, v_scale) of 8-bit E4M3 pools, else None
    kv_bscales: list | None = None   # per layer (k_scales, v_scales) [N, Hkv] of block-scaled pools

    @property
    def layers(self) -> int:
        return len(self.k_caches)

    def kv_bytes_per_step(self) -> int:
        """Algorithmic KV bytes one decode step reads: every cached token of every
        sequence, K and V, all kv heads, all layers."""
        w = self.w
        ctx = self.context_lens.cpu().numpy().astype(np.int64)
        elem = self.k_caches[0].element_size()
        return int(ctx.sum()) * w.num_kv_heads * w.head_dim * 2 * elem * self.layers

    def unique_kv_bytes_per_step(self) -> int:
        """KV bytes with every shared block counted once (blocks x fill)."""
        seen = {}
        for s in self.sids:
            n = self.bm.context_len(s)
            for i, b in enumerate(self.bm.table(s)):
                seen[b] = max(seen.get(b, 0), min(self.block_size, n - i * self.block_size))
        w = self.w
        elem = self.k_caches[0].element_size()
        return sum(seen.values()) * w.num_kv_heads * w.head_dim * 2 * elem * self.layers


def _pool_size(w: inputs.Workload, need: int) -> int:
    return w.pool_blocks if w.pool_blocks else int(math.ceil(w.pool_factor * need))


KV8_SCALE = 1.0 / 64.0               # per-tensor scale of the synthetic 8-bit pools


def _alloc_layers(w, N, bs, layers, device, seed, kv8=False):
    k, v = [], []
    shape = (N, w.num_kv_heads, bs, w.head_dim)
    for l in range(layers):
        if kv8:
            k.append(inputs.randn_e4m3(shape, KV8_SCALE, seed, device, stream=1000 + 2 * l))
            v.append(inputs.randn_e4m3(shape, KV8_SCALE, seed, device, stream=1001 + 2 * l))
        else:
            k.append(inputs.randn(shape, w.dtype, seed, device, stream=1000 + 2 * l))
            v.append(inputs.randn(shape, w.dtype, seed, device, stream=1001 + 2 * l))
    return k, v


def _fill_block_scaled(w, bs, bm, sids, N, layers, device, seed):
    """8-bit pools with per-(block, kv head) scales, filled the way a server fills them:
    every cached token's 16-bit K/V rows (N(0,1)) appended in position order with
    pa_cache_append_e4m3_bs, so each block's scale is the one its first token fixed."""
    import torch

    slots = torch.tensor([bm.slot_of(s, p) for s in sids for p in range(bm.context_len(s))],
                         dtype=torch.int64, device=device)
    T = slots.shape[0]
    k8, v8, sc = [], [], []
    for l in range(layers):
        kc = torch.zeros((N, w.num_kv_heads, bs, w.head_dim), dtype=torch.uint8, device=device)
        vc = torch.zeros_like(kc)
        ks = torch.ones((N, w.num_kv_heads), dtype=torch.float32, device=device)
        vs = torch.ones_like(ks)
        kr = inputs.randn((T, w.num_kv_heads, w.head_dim), w.dtype, seed, device, stream=1000 + 2 * l)
        vr = inputs.randn((T, w.num_kv_heads, w.head_dim), w.dtype, seed, device, stream=1001 + 2 * l)
        pk.pa_cache_append_e4m3_bs(kc, vc, ks, vs, kr, vr, slots)
        del kr, vr
        k8.append(kc)
        v8.append(vc)
        sc.append((ks, vs))
    return k8, v8, sc


def _finish(w, bs, bm, sids, N, layers, device, cow_pairs=None, q_len=1,
            kv8=False) -> DecodeBatch:
    B = len(sids)
    if kv8 == "block":
        k_caches, v_caches, bscales = _fill_block_scaled(w, bs, bm, sids, N, layers, device,
                                                         w.seed)
    else:
        k_caches, v_caches = _alloc_layers(w, N, bs, layers, device, w.seed, kv8)
        bscales = None
    tables = torch.from_numpy(bm.block_tables(sids)).to(device)
    ctx = torch.from_numpy(bm.context_lens(sids)).to(device)
    # the newest q_len tokens of every sequence are the ones appended and queried
    slots = torch.tensor([bm.slot_of(s, bm.context_len(s) - q_len + j) for s in sids
                          for j in range(q_len)], dtype=torch.int64, device=device)
    qshape = (B, w.num_q_heads, w.head_dim) if q_len == 1 else \
        (B, q_len, w.num_q_heads, w.head_dim)
    q, kn, vn, out = [], [], [], []
    for l in range(layers):
        q.append(inputs.randn(qshape, w.dtype, w.seed, device, stream=5000 + 3 * l))
        kn.append(inputs.randn((B * q_len, w.num_kv_heads, w.head_dim), w.dtype, w.seed, device,
                               stream=5001 + 3 * l))
        vn.append(inputs.randn((B * q_len, w.num_kv_heads, w.head_dim), w.dtype, w.seed, device,
                               stream=5002 + 3 * l))
        out.append(torch.empty(qshape, dtype=inputs.torch_dtype(w.dtype), device=device))
    ws = pk.new_workspace(B, w.num_q_heads, w.num_kv_heads, w.head_dim, device)
    st = pk.new_status(device)
    pairs = None
    if cow_pairs:
        pairs = torch.tensor(cow_pairs, dtype=torch.int32, device=device).reshape(-1, 2)
    return DecodeBatch(w, bs, bm, sids, N, k_caches, v_caches, tables, ctx, slots, q, kn, vn, out,
                       ws, st, pairs, 1.0 / math.sqrt(w.head_dim), q_len,
                       kv_scales=(KV8_SCALE, KV8_SCALE) if kv8 is True else None,
                       kv_bscales=bscales)


def build(w: inputs.Workload, device="cuda", block_size: int | None = None,
          layers: int | None = None, q_len: int = 1, kv8=False,
          contiguous: bool = False) -> DecodeBatch:
    """Independent sequences (every workload but the shared-prefix one).  With q_len > 1
    every sequence's newest q_len tokens are appended and queried each step.  kv8: False
    (16-bit pools), True (8-bit pools, one scale per pool) or "block" (8-bit pools with
    per-(block, kv head) scales, filled by the quantising append).  With
    contiguous=True the pool hands out blocks in id order, so every sequence's table is
    one run of consecutive blocks (the identity placement a contiguous cache would have)
    instead of the seeded fragmented one."""
    bs = block_size or w.block_size
    ctx = inputs.context_lens(w)
    need = int(sum(-(-int(c) // bs) for c in ctx))
    N = _pool_size(w, need)
    bm = BlockManager(N, bs, None if contiguous else inputs.pool_order(N, w.seed))
    sids = [bm.allocate(int(c)) for c in ctx]
    return _finish(w, bs, bm, sids, N, layers or w.layers, device, q_len=q_len, kv8=kv8)


def build_prefix_decode(w: inputs.Workload = inputs.PREFIX, device="cuda") -> DecodeBatch:
    """Shared-prefix parallel sampling, decode phase: per prompt a 2048-token prefix
    held once (refcount 8) and 0..512 private tokens per sample."""
    bs = w.block_size
    ctx = inputs.context_lens(w)                       # prefix + private, per sample
    need = inputs.PREFIX_PROMPTS * (inputs.PREFIX_LEN // bs) + int(
        sum(-(-int(c - inputs.PREFIX_LEN) // bs) for c in ctx))
    N = _pool_size(w, need)
    bm = BlockManager(N, bs, inputs.pool_order(N, w.seed))
    sids = []
    for p in range(inputs.PREFIX_PROMPTS):
        root = bm.allocate(inputs.PREFIX_LEN)
        kids = [root] + [bm.fork(root) for _ in range(inputs.PREFIX_SAMPLES - 1)]
        for j, sid in enumerate(kids):
            for _ in range(int(ctx[p * inputs.PREFIX_SAMPLES + j]) - inputs.PREFIX_LEN):
                slot, cow = bm.append_token(sid)
                assert cow is None                     # prefix is block aligned
            sids.append(sid)
    return _finish(w, bs, bm, sids, N, w.layers, device)


def build_prefix_fork(w: inputs.Workload = inputs.PREFIX, device="cuda") -> DecodeBatch:
    """Shared-prefix fork phase: each prompt's shared region is 2048 + t tokens
    (t in 1..15), so its last block is partial and shared by 8 samples; every sample
    then appends one token, and all but the last writer copy that block first."""
    bs = w.block_size
    tails = inputs.prefix_fork_tails(w)
    per_prompt = -(-(inputs.PREFIX_LEN + int(tails.max())) // bs) + inputs.PREFIX_SAMPLES
    N = _pool_size(w, inputs.PREFIX_PROMPTS * per_prompt)
    bm = BlockManager(N, bs, inputs.pool_order(N, w.seed))
    sids, pairs = [], []
    for p in range(inputs.PREFIX_PROMPTS):
        root = bm.allocate(inputs.PREFIX_LEN + int(tails[p]))
        kids = [root] + [bm.fork(root) for _ in range(inputs.PREFIX_SAMPLES - 1)]
        for sid in kids:
            _, cow = bm.append_token(sid)
            if cow:
                pairs.append(cow)
            sids.append(sid)
    return _finish(w, bs, bm, sids, N, w.layers, device, cow_pairs=pairs)


def run_step(b: DecodeBatch, stream=None, layers=None, fused: bool = False) -> None:
    """One decode step over all layers (see module docstring).  With fused=True each
    layer is one pa_decode_append (pa_decode_append_e4m3_bs over block-scaled 8-bit pools)
    call: the newest token's append fused into decode; one new token per sequence, no
    cascade."""
    if b.cow_pairs is not None and b.cow_pairs.shape[0]:
        pk.pa_copy_blocks(b.k_caches, b.v_caches, b.cow_pairs, b.status, stream)
    for l in range(layers if layers is not None else b.layers):
        if fused and b.kv_scales is None:
            append_decode_layer(b, l, stream)
            continue
        if b.kv_bscales is not None:
            pk.pa_cache_append_e4m3_bs(b.k_caches[l], b.v_caches[l], *b.kv_bscales[l], b.k_new[l],
                                       b.v_new[l], b.slot_mapping, b.status, stream)
        elif b.kv_scales is not None:
            pk.pa_cache_append_e4m3(b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                                    b.slot_mapping, *b.kv_scales, b.status, stream)
        else:
            pk.pa_cache_append(b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                               b.slot_mapping, b.status, stream)
        decode_layer(b, l, stream)


def append_decode_layer(b: DecodeBatch, l: int, stream=None, block_tables=None,
                        context_lens=None) -> None:
    """pa_decode_append of layer l: append the newest token of every sequence and decode."""
    assert b.q_len == 1 and b.cascade is None
    if b.kv_bscales is not None:
        pk.pa_decode_append_e4m3_bs(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l],
                                    *b.kv_bscales[l], b.k_new[l], b.v_new[l],
                                    b.block_tables if block_tables is None else block_tables,
                                    b.context_lens if context_lens is None else context_lens,
                                    b.scale, b.workspace, b.status, stream)
        return
    pk.pa_decode_append(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], b.k_new[l], b.v_new[l],
                        b.block_tables if block_tables is None else block_tables,
                        b.context_lens if context_lens is None else context_lens, b.scale,
                        b.workspace, b.status, stream)


def use_cascade(b: DecodeBatch, width: int | None = None) -> DecodeBatch:
    """Decode this batch with pa_decode_cascade (pa_decode_cascade_e4m3_bs over block-scaled
    8-bit pools, whose chunks hold up to 16 query rows): plan the shared-prefix chunks from
    its block tables (the workspace grows to the cascade size)."""
    w = b.w
    ctx = b.context_lens.cpu().numpy()
    if width is None and b.kv_bscales is not None:
        width = max(1, 16 // (w.num_q_heads // w.num_kv_heads))
    prefix, members, plens = b.bm.plan_cascade(b.sids, w.num_q_heads // w.num_kv_heads, width)
    dev = b.block_tables.device
    b.cascade = (torch.from_numpy(prefix).to(dev), torch.from_numpy(members).to(dev),
                 torch.from_numpy(plens).to(dev))
    b.workspace = pk.new_cascade_workspace(len(ctx), w.num_q_heads, w.num_kv_heads, w.head_dim,
                                           dev)
    return b


def decode_layer(b: DecodeBatch, l: int, stream=None) -> None:
    """pa_decode (one new token per sequence), pa_decode_multi (q_len > 1) or
    pa_decode_cascade (after use_cascade) of layer l."""
    if b.cascade is not None and b.kv_bscales is not None:
        pk.pa_decode_cascade_e4m3_bs(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l],
                                     *b.kv_bscales[l], b.block_tables, b.context_lens,
                                     *b.cascade, b.scale, b.workspace, b.status, stream)
        return
    if b.cascade is not None:
        pk.pa_decode_cascade(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], b.block_tables,
                             b.context_lens, *b.cascade, b.scale, b.workspace, b.status, stream)
        return
    if b.kv_bscales is not None:
        pk.pa_decode_e4m3_bs(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], *b.kv_bscales[l],
                             b.block_tables, b.context_lens, b.scale, b.workspace, b.status, stream)
        return
    if b.kv_scales is not None:
        pk.pa_decode_e4m3(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], *b.kv_scales,
                          b.block_tables, b.context_lens, b.scale, b.workspace, b.status, stream)
        return
    fn = pk.pa_decode if b.q_len == 1 else pk.pa_decode_multi
    fn(b.out[l], b.q[l], b.k_caches[l], b.v_caches[l], b.block_tables, b.context_lens, b.scale,
       b.workspace, b.status, stream)


def plan_cascade(tables: np.ndarray, ctx: np.ndarray, block_size: int, group: int,
                 width: int | None = None):
    """Chunks of sequences that share a prefix of their block tables, for
    pa_decode_cascade, planned by the library (pa_plan_cascade): sequences whose first
    block is the same physical block form a sharing group; its prefix is the leading
    table entries common to all members, capped at the shortest member's length; a
    chunk holds at most `width` members (by default fitted to the sharing groups: each
    in the fewest chunks of at most 64 // group members, spread evenly)."""
    from .block_manager import plan_cascade_tables

    return plan_cascade_tables(tables, ctx, block_size, group, width)
