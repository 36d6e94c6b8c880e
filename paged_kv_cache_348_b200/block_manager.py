"""Host-side block manager for a paged KV cache.

Bookkeeping only (no value arithmetic): a pool of fixed-size physical blocks, one
block table per sequence, reference counts, on-demand allocation, copy-on-write
when a sequence writes into a block it shares, and release.

Follows "PagedAttention in Production: Boosting LLM Serving Throughput with Paged KV
Cache", section "Core Principle" (logical blocks map to physical blocks through a
block table; blocks are allocated on demand and returned to the pool), "Paged
Attention and Memory Efficiency in Production LLM Serving", section "How PagedAttention
borrows OS paging" (shared prefixes point at the same blocks; a new block is
allocated only on divergence -- copy-on-write), and "PagedAttention -- The KV Cache
Problem", section "How It Works".

It produces exactly what the CUDA calls consume: int32 block tables, int32 context
lengths, int64 slot mappings and int32 (src, dst) copy pairs.

The bookkeeping itself is native: this class is a ctypes wrapper over the pa_bm_*
calls of libpagedkv (include/pagedkv.h, csrc/block_manager.cpp).  It needs the
library but no GPU.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import pagedkv as pk


class PoolExhausted(MemoryError):
    pass


def _lib():
    L = pk.load()
    if not getattr(L, "_bm_ready", False):
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.pa_bm_create.argtypes = [i32, i32, P, ctypes.POINTER(P)]
        L.pa_bm_create.restype = i32
        L.pa_bm_destroy.argtypes = [P]
        L.pa_bm_destroy.restype = None
        L.pa_bm_free_blocks.argtypes = [P]
        L.pa_bm_free_blocks.restype = i32
        L.pa_bm_refcount.argtypes = [P, i32]
        L.pa_bm_refcount.restype = i32
        L.pa_bm_allocate.argtypes = [P, i32, P]
        L.pa_bm_allocate.restype = i32
        L.pa_bm_fork.argtypes = [P, i32, P]
        L.pa_bm_fork.restype = i32
        L.pa_bm_append_tokens.argtypes = [P, P, i32, P, P, P]
        L.pa_bm_append_tokens.restype = i32
        L.pa_bm_release.argtypes = [P, i32]
        L.pa_bm_release.restype = i32
        L.pa_bm_context_len.argtypes = [P, i32]
        L.pa_bm_context_len.restype = i64
        L.pa_bm_num_blocks_of.argtypes = [P, i32]
        L.pa_bm_num_blocks_of.restype = i32
        L.pa_bm_max_blocks.argtypes = [P, P, i32]
        L.pa_bm_max_blocks.restype = i32
        L.pa_bm_block_tables.argtypes = [P, P, i32, i32, i32, P, P]
        L.pa_bm_block_tables.restype = i32
        L.pa_bm_slot_of.argtypes = [P, i32, i64, P]
        L.pa_bm_slot_of.restype = i32
        L.pa_bm_plan_cascade.argtypes = [P, P, i32, i32, i32, P, P, P, P, P]
        L.pa_bm_plan_cascade.restype = i32
        L.pa_plan_cascade.argtypes = [P, i32, P, i32, i32, i32, i32, P, P, P, P, P]
        L.pa_plan_cascade.restype = i32
        L.pa_bm_swap_out.argtypes = [P, i32, P, P]
        L.pa_bm_swap_out.restype = i32
        L.pa_bm_swap_in.argtypes = [P, i32, P, P]
        L.pa_bm_swap_in.restype = i32
        L._bm_ready = True
    return L


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _cascade_width(group: int, width: int | None) -> int:
    return int(width) if width else max(1, 64 // int(group))


def plan_cascade_tables(tables: np.ndarray, ctx: np.ndarray, block_size: int, group: int,
                        width: int | None = None):
    """Shared-prefix chunks of a batch for pa_decode_cascade, from its block tables
    (pa_plan_cascade in include/pagedkv.h).  Returns (prefix_lens int32 [B],
    chunk_members int32 [C, W], chunk_prefix_lens int32 [C]); W = width, or by default
    fitted to the sharing groups (each in the fewest chunks of at most 64 // group
    members, spread evenly)."""
    t = np.ascontiguousarray(np.asarray(tables, dtype=np.int32))
    c = np.ascontiguousarray(np.asarray(ctx, dtype=np.int32))
    B = c.shape[0]
    W = _cascade_width(group, width)
    prefix = np.zeros(max(B, 1), dtype=np.int32)
    members = np.zeros((max(B, 1), W), dtype=np.int32)
    plens = np.zeros(max(B, 1), dtype=np.int32)
    nc, wo = ctypes.c_int(), ctypes.c_int()
    rc = _lib().pa_plan_cascade(_ptr(t), t.shape[1] if t.ndim == 2 else 0, _ptr(c), B,
                                int(block_size), int(group), int(width or 0), _ptr(prefix),
                                _ptr(members), _ptr(plens), ctypes.byref(nc), ctypes.byref(wo))
    if rc != pk.PA_OK:
        raise ValueError("pa_plan_cascade failed (%d)" % rc)
    return _unpack_plan(prefix, members, plens, B, nc.value, wo.value)


def _unpack_plan(prefix, members, plens, B, nc, w):
    m = members.reshape(-1)[:nc * w].reshape(nc, w)
    return prefix[:B].copy(), m.copy(), plens[:nc].copy()


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        L = _lib()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if order.shape != (num_blocks,):
                raise ValueError("free_order must be a permutation of the pool")
        h = ctypes.c_void_p()
        rc = L.pa_bm_create(num_blocks, block_size, None if order is None else _ptr(order),
                            ctypes.byref(h))
        if rc == pk.PA_ERR_INVALID:
            raise ValueError("free_order must be a permutation of the pool")
        if rc != pk.PA_OK:
            raise RuntimeError("pa_bm_create failed (%d)" % rc)
        self._h = h
        self._L = L

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._L.pa_bm_destroy(h)
            self._h = None

    def _check(self, rc: int, what: str):
        if rc == pk.PA_ERR_NO_BLOCKS:
            raise PoolExhausted("%s: not enough free KV blocks (%d free)" % (what, self.free_blocks))
        if rc != pk.PA_OK:
            raise ValueError("%s failed (%d)" % (what, rc))

    # ---------------------------------------------------------------- allocation
    @property
    def free_blocks(self) -> int:
        return int(self._L.pa_bm_free_blocks(self._h))

    def refcount(self, block: int) -> int:
        r = int(self._L.pa_bm_refcount(self._h, int(block)))
        if r < 0:
            raise IndexError(block)
        return r

    def allocate(self, n_tokens: int) -> int:
        """New sequence holding n_tokens cached tokens; returns its id."""
        sid = ctypes.c_int32()
        self._check(self._L.pa_bm_allocate(self._h, int(n_tokens), ctypes.byref(sid)), "allocate")
        return sid.value

    def fork(self, sid: int) -> int:
        """New sequence sharing every block of `sid` (parallel sampling / beams)."""
        child = ctypes.c_int32()
        self._check(self._L.pa_bm_fork(self._h, int(sid), ctypes.byref(child)), "fork")
        return child.value

    def append_tokens(self, sids):
        """Reserve the next slot of each listed sequence, in order.  Returns (slots
        int64 [n], copy-on-write pairs int32 [k, 2]) -- the pairs must be copied before
        the new tokens are written."""
        s = np.ascontiguousarray(np.asarray(sids, dtype=np.int32))
        n = s.shape[0]
        slots = np.zeros(n, dtype=np.int64)
        pairs = np.zeros((max(n, 1), 2), dtype=np.int32)
        nc = ctypes.c_int()
        self._check(self._L.pa_bm_append_tokens(self._h, _ptr(s), n, _ptr(slots), _ptr(pairs),
                                                ctypes.byref(nc)), "append")
        return slots, pairs[:nc.value].copy()

    def append_token(self, sid: int):
        """Reserve the slot of the next token of `sid`.

        Returns (slot, cow): slot = physical_block * block_size + offset, and cow is
        None or the (src, dst) block pair to copy before the new token is written."""
        slots, pairs = self.append_tokens([sid])
        cow = (int(pairs[0, 0]), int(pairs[0, 1])) if len(pairs) else None
        return int(slots[0]), cow

    def release(self, sid: int) -> None:
        self._check(self._L.pa_bm_release(self._h, int(sid)), "release")

    def swap_out(self, sid: int) -> np.ndarray:
        """Preempt `sid` (pa_bm_swap_out): returns its blocks in table order, whose
        contents must be saved (pa_swap_out_blocks) before the pool reuses them; the
        blocks go back to the pool as on release and `sid` keeps its length."""
        n = max(int(self._L.pa_bm_num_blocks_of(self._h, int(sid))), 1)
        out = np.zeros(n, dtype=np.int32)
        k = ctypes.c_int()
        self._check(self._L.pa_bm_swap_out(self._h, int(sid), _ptr(out), ctypes.byref(k)),
                    "swap_out")
        return out[:k.value].copy()

    def swap_in(self, sid: int) -> np.ndarray:
        """Resume a swapped-out `sid` (pa_bm_swap_in): fresh blocks in table order, into
        which the saved contents are restored (pa_swap_in_blocks)."""
        n = max(-(-self.context_len(sid) // self.block_size), 1)
        out = np.zeros(n, dtype=np.int32)
        k = ctypes.c_int()
        self._check(self._L.pa_bm_swap_in(self._h, int(sid), _ptr(out), ctypes.byref(k)),
                    "swap_in")
        return out[:k.value].copy()

    # ---------------------------------------------------------------- views
    def table(self, sid: int) -> list[int]:
        n = int(self._L.pa_bm_num_blocks_of(self._h, int(sid)))
        if n < 0:
            raise KeyError(sid)
        return [int(x) for x in self.block_tables([sid], width=max(n, 1))[0, :n]]

    def context_len(self, sid: int) -> int:
        n = int(self._L.pa_bm_context_len(self._h, int(sid)))
        if n < 0:
            raise KeyError(sid)
        return n

    def slot_of(self, sid: int, pos: int) -> int:
        """Flat slot of logical position `pos` of `sid`."""
        out = ctypes.c_int64()
        self._check(self._L.pa_bm_slot_of(self._h, int(sid), int(pos), ctypes.byref(out)),
                    "slot_of")
        return out.value

    def block_tables(self, sids, width: int | None = None, fill: int = 0) -> np.ndarray:
        return self._tables(sids, width, fill)[0]

    def _tables(self, sids, width, fill):
        s = np.ascontiguousarray(np.asarray(list(sids), dtype=np.int32))
        if width is None:
            width = max(int(self._L.pa_bm_max_blocks(self._h, _ptr(s), len(s))), 1)
        out = np.empty((len(s), width), dtype=np.int32)
        lens = np.empty(len(s), dtype=np.int32)
        rc = self._L.pa_bm_block_tables(self._h, _ptr(s), len(s), int(width), int(fill),
                                        _ptr(out), _ptr(lens))
        if rc != pk.PA_OK:
            raise ValueError("block table wider than width, or unknown sequence")
        return out, lens

    def context_lens(self, sids) -> np.ndarray:
        return self._tables(sids, None, 0)[1]

    def plan_cascade(self, sids, group: int, width: int | None = None):
        """Shared-prefix chunks of the batch sids (batch row i = sids[i]) from the
        manager's own tables (pa_bm_plan_cascade); same result as plan_cascade_tables."""
        s = np.ascontiguousarray(np.asarray(list(sids), dtype=np.int32))
        B = s.shape[0]
        W = _cascade_width(group, width)
        prefix = np.zeros(max(B, 1), dtype=np.int32)
        members = np.zeros((max(B, 1), W), dtype=np.int32)
        plens = np.zeros(max(B, 1), dtype=np.int32)
        nc, wo = ctypes.c_int(), ctypes.c_int()
        rc = self._L.pa_bm_plan_cascade(self._h, _ptr(s), B, int(group), int(width or 0),
                                        _ptr(prefix), _ptr(members), _ptr(plens),
                                        ctypes.byref(nc), ctypes.byref(wo))
        self._check(rc, "plan_cascade")
        return _unpack_plan(prefix, members, plens, B, nc.value, wo.value)

    def tail_waste(self, sids) -> float:
        """Fraction of held slots that hold no token: only the unused tail of each
        sequence's last block (shared blocks counted once per sequence)."""
        held = sum(int(self._L.pa_bm_num_blocks_of(self._h, int(s))) * self.block_size
                   for s in sids)
        used = sum(self.context_len(s) for s in sids)
        return 0.0 if held == 0 else (held - used) / held
