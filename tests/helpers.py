"""Test-side helpers: build small paged caches from the seeded generators.

Tables come from the oracle's reference block manager so that oracle-only tests do
not depend on the product library.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle.cow import RefBlockManager
from paged_kv_cache_348_b200 import inputs

NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


def bits(t: torch.Tensor) -> np.ndarray:
    """16-bit tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(inputs.torch_dtype(dtype))


def bits_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening by numpy's own formats (independent of the oracle's decoder)."""
    a = np.asarray(a, dtype=np.uint16)
    if dtype == "f16":
        return a.view(np.float16).astype(np.float64)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def make_case(B, Hq, Hkv, D, bs, ctx, dtype="f16", seed=0, pool_blocks=None, shuffle=True,
              poison=True):
    """Random q / K / V pools with block tables for the given context lengths.

    Unused pool blocks and the unused tail slots of each last block are set to NaN
    when `poison` is true (they must never be read)."""
    ctx = np.asarray(ctx, dtype=np.int32)
    need = int(sum(-(-int(c) // bs) for c in ctx))
    N = pool_blocks if pool_blocks is not None else max(need + 3, int(np.ceil(need * 1.2)))
    order = inputs.pool_order(N, seed) if shuffle else np.arange(N, dtype=np.int32)
    bm = RefBlockManager(N, bs, order)
    sids = [bm.new_seq(int(c)) for c in ctx]
    M = max(1, max(len(bm.tables[s]) for s in sids))
    tables = np.full((B, M), -7, dtype=np.int32)    # entries past the last block: junk
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
        mask = ~used
        k.transpose(0, 2, 1, 3)[mask] = NAN_BITS[dtype]
        v.transpose(0, 2, 1, 3)[mask] = NAN_BITS[dtype]
    return dict(q=q, k=k, v=v, tables=tables, ctx=ctx, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs,
                dtype=dtype, N=N, scale=1.0 / np.sqrt(D), bm=bm, sids=sids)
