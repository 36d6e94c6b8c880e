"""Reference block bookkeeping (pure Python, no arithmetic on values).

TEST INFRASTRUCTURE ONLY -- part of the oracle package.

Follows:
  * "PagedAttention in Production: Boosting LLM Serving Throughput with Paged KV Cache",
    section "Core Principle": logical blocks, physical blocks, a block table per
    request, blocks allocated on demand and returned to the pool when a request ends.
  * "Paged Attention and Memory Efficiency in Production LLM Serving", section
    "How PagedAttention borrows OS paging": requests with an identical prefix point
    their block tables at the same physical blocks; a new block is allocated only once
    a sequence diverges (copy-on-write).
  * "PagedAttention -- The KV Cache Problem", section "How It Works": fixed-size blocks,
    one block table per sequence, allocate on demand, free when the sequence finishes.
  * "Paged Attention and Memory Efficiency in Production LLM Serving", section "Why KV
    cache memory was the bottleneck": when the cache runs out, in-flight requests are
    preempted.  Preemption here is a swap: the sequence's blocks are given back to the
    pool (as on release) after their contents are saved, and the sequence, which keeps
    its length, later takes fresh blocks for the saved contents.

Free blocks are handed out in the order given to the constructor (lowest index of the
remaining list first), so a run is fully determined by that order.
"""
from __future__ import annotations


class RefBlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.bs = block_size
        self.free = list(range(num_blocks)) if free_order is None else list(free_order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.ctx: dict[int, int] = {}
        self.swapped: set[int] = set()
        self._next = 0

    def _alloc(self) -> int:
        if not self.free:
            raise MemoryError("block pool exhausted")
        b = self.free.pop(0)
        assert self.ref[b] == 0
        self.ref[b] = 1
        return b

    def new_seq(self, n_tokens: int) -> int:
        """A sequence whose first n_tokens positions are already held (prefill)."""
        sid = self._next
        self._next += 1
        nblk = -(-n_tokens // self.bs)
        self.tables[sid] = [self._alloc() for _ in range(nblk)]
        self.ctx[sid] = n_tokens
        return sid

    def fork(self, sid: int) -> int:
        """A child that shares every block of `sid` (parallel sampling)."""
        child = self._next
        self._next += 1
        self.tables[child] = list(self.tables[sid])
        self.ctx[child] = self.ctx[sid]
        for b in self.tables[child]:
            self.ref[b] += 1
        return child

    def append_slot(self, sid: int):
        """Reserve the slot of the next token of `sid`.

        Returns (slot, cow) where slot = physical_block * block_size + offset and
        cow is None or the (src, dst) pair that must be copied before the write."""
        t = self.ctx[sid]
        lb, off = divmod(t, self.bs)
        table = self.tables[sid]
        cow = None
        if lb == len(table):                       # crossing into a new logical block
            table.append(self._alloc())
        else:
            b = table[lb]
            if self.ref[b] > 1:                    # shared partial block: diverge
                nb = self._alloc()
                self.ref[b] -= 1
                table[lb] = nb
                cow = (b, nb)
        self.ctx[sid] = t + 1
        return table[lb] * self.bs + off, cow

    def release(self, sid: int) -> None:
        for b in self.tables.pop(sid):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        self.ctx.pop(sid)
        self.swapped.discard(sid)

    def swap_out(self, sid: int) -> list[int]:
        """Preempt `sid`: returns its blocks in table order (their contents are to be
        saved first); each block's count goes down by one, blocks reaching zero return to
        the back of the free list, and `sid` keeps its length but holds no block."""
        assert sid not in self.swapped
        blocks = self.tables[sid]
        self.tables[sid] = []
        for b in blocks:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        self.swapped.add(sid)
        return list(blocks)

    def swap_in(self, sid: int) -> list[int]:
        """Resume a swapped-out `sid`: ceil(len / block_size) fresh blocks from the front
        of the free list, in table order (the saved contents go there).  Raises
        MemoryError and changes nothing if the pool cannot hold them."""
        assert sid in self.swapped
        need = -(-self.ctx[sid] // self.bs)
        if len(self.free) < need:
            raise MemoryError("block pool exhausted")
        self.tables[sid] = [self._alloc() for _ in range(need)]
        self.swapped.discard(sid)
        return list(self.tables[sid])
