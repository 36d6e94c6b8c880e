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
"""
from __future__ import annotations

from collections import deque

import numpy as np


class PoolExhausted(MemoryError):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = range(num_blocks) if free_order is None else [int(b) for b in free_order]
        self._free = deque(order)
        if len(self._free) != num_blocks or len(set(self._free)) != num_blocks:
            raise ValueError("free_order must be a permutation of the pool")
        self._ref = np.zeros(num_blocks, dtype=np.int32)
        self._tables: dict[int, list[int]] = {}
        self._lens: dict[int, int] = {}
        self._next_id = 0

    # ---------------------------------------------------------------- allocation
    @property
    def free_blocks(self) -> int:
        return len(self._free)

    def refcount(self, block: int) -> int:
        return int(self._ref[block])

    def _take(self) -> int:
        if not self._free:
            raise PoolExhausted("no free KV block left")
        b = self._free.popleft()
        self._ref[b] = 1
        return b

    def _blocks_for(self, n_tokens: int) -> int:
        return -(-n_tokens // self.block_size)

    def allocate(self, n_tokens: int) -> int:
        """New sequence holding n_tokens cached tokens; returns its id."""
        need = self._blocks_for(n_tokens)
        if need > len(self._free):
            raise PoolExhausted("need %d blocks, %d free" % (need, len(self._free)))
        sid = self._next_id
        self._next_id += 1
        self._tables[sid] = [self._take() for _ in range(need)]
        self._lens[sid] = n_tokens
        return sid

    def fork(self, sid: int) -> int:
        """New sequence sharing every block of `sid` (parallel sampling / beams)."""
        child = self._next_id
        self._next_id += 1
        self._tables[child] = list(self._tables[sid])
        self._lens[child] = self._lens[sid]
        for b in self._tables[child]:
            self._ref[b] += 1
        return child

    def append_token(self, sid: int):
        """Reserve the slot of the next token of `sid`.

        Returns (slot, cow): slot = physical_block * block_size + offset, and cow is
        None or the (src, dst) block pair to copy before the new token is written."""
        pos = self._lens[sid]
        lb, off = divmod(pos, self.block_size)
        table = self._tables[sid]
        cow = None
        if lb == len(table):
            table.append(self._take())
        elif self._ref[table[lb]] > 1:
            src = table[lb]
            dst = self._take()
            self._ref[src] -= 1
            table[lb] = dst
            cow = (src, dst)
        self._lens[sid] = pos + 1
        return table[lb] * self.block_size + off, cow

    def release(self, sid: int) -> None:
        for b in self._tables.pop(sid):
            self._ref[b] -= 1
            if self._ref[b] == 0:
                self._free.append(b)
        del self._lens[sid]

    # ---------------------------------------------------------------- views
    def table(self, sid: int) -> list[int]:
        return list(self._tables[sid])

    def context_len(self, sid: int) -> int:
        return self._lens[sid]

    def slot_of(self, sid: int, pos: int) -> int:
        """Flat slot of logical position `pos` of `sid`."""
        lb, off = divmod(pos, self.block_size)
        return self._tables[sid][lb] * self.block_size + off

    def block_tables(self, sids, width: int | None = None, fill: int = 0) -> np.ndarray:
        w = max([len(self._tables[s]) for s in sids] + [1]) if width is None else width
        out = np.full((len(sids), w), fill, dtype=np.int32)
        for i, s in enumerate(sids):
            t = self._tables[s]
            if len(t) > w:
                raise ValueError("block table wider than width")
            out[i, :len(t)] = t
        return out

    def context_lens(self, sids) -> np.ndarray:
        return np.array([self._lens[s] for s in sids], dtype=np.int32)

    def tail_waste(self, sids) -> float:
        """Fraction of held slots that hold no token: only the unused tail of each
        sequence's last block (shared blocks counted once per sequence)."""
        held = sum(len(self._tables[s]) * self.block_size for s in sids)
        used = sum(self._lens[s] for s in sids)
        return 0.0 if held == 0 else (held - used) / held
