"""Reference shared-prefix planner (pure Python bookkeeping, no arithmetic on values).

TEST INFRASTRUCTURE ONLY -- part of the oracle package.

Follows "Paged Attention and Memory Efficiency in Production LLM Serving", section
"How PagedAttention borrows OS paging": requests with an identical prefix point their
block tables at the same physical blocks, so the tokens those blocks hold are the same
K/V for every request that names them.  A shared-prefix decode may therefore read those
tokens once for all of the sharers.  The planner restates which rows of a batch share
which prefix:

  1. rows with at least one cached token are grouped by the physical block their table
     names first (groups in order of first appearance, members in row order);
  2. a group's prefix is the run of leading table entries that every member names
     identically, counted in tokens and capped at the member with the fewest tokens;
  3. a group of one row, or one whose prefix is empty, shares nothing;
  4. the members of a sharing group are dealt, in row order, into chunks of at most
     `width` rows (the last chunk padded with -1), each carrying the group's prefix.

The chunk width is a scheduling choice the pages leave open (a chunk's query rows are the
columns of one decode tile, at most 64).  When the caller gives none, the width is the
smallest that still puts each sharing group in the fewest chunks of at most 64 // group
rows: for a group of m rows that is ceil(m / ceil(m / Wmax)), and the batch takes the
largest over its sharing groups (Wmax when no group shares anything).
"""
from __future__ import annotations

import numpy as np


def plan_cascade(tables, ctx, block_size: int, group: int, width: int | None = None):
    """Returns (prefix_lens int32 [B], chunk_members int32 [C, W],
    chunk_prefix_lens int32 [C]); W = width, or fitted to the sharing groups (see the
    module docstring)."""
    tables = np.asarray(tables)
    ctx = [int(c) for c in np.asarray(ctx)]
    wmax = max(1, 64 // group)
    order, groups = [], {}
    for i, c in enumerate(ctx):
        if c <= 0:
            continue
        first = int(tables[i][0])
        if first not in groups:
            groups[first] = []
            order.append(first)
        groups[first].append(i)
    sharing = []                                       # (rows, prefix) of each sharing group
    for first in order:
        rows = groups[first]
        if len(rows) < 2:
            continue
        shortest = min(ctx[i] for i in rows)
        usable = -(-shortest // block_size)            # blocks every member holds
        k = 0
        while k < usable and len({int(tables[i][k]) for i in rows}) == 1:
            k += 1
        plen = min(k * block_size, shortest)
        if plen > 0:
            sharing.append((rows, plen))
    if width:
        W = width
    elif sharing:
        W = max(-(-len(rows) // -(-len(rows) // wmax)) for rows, _ in sharing)
    else:
        W = wmax
    prefix = [0] * len(ctx)
    chunks, plens = [], []
    for rows, plen in sharing:
        for start in range(0, len(rows), W):
            part = rows[start:start + W]
            chunks.append(part + [-1] * (W - len(part)))
            plens.append(plen)
            for i in part:
                prefix[i] = plen
    members = np.array(chunks, dtype=np.int32).reshape(len(chunks), W)
    return np.array(prefix, dtype=np.int32), members, np.array(plens, dtype=np.int32)
