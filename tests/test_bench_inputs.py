"""The oracle arm of bench.py builds its inputs without the library (the oracle's
reference block manager and the seeded generators): they must be exactly the GPU
workload's layer 0 (tables, lengths and value bits).  CPU only."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import bench
from paged_kv_cache_348_b200 import inputs
from paged_kv_cache_348_b200 import workload as wl
from tests.helpers import bits


@pytest.mark.parametrize("name,bs", [("tiny", 16), ("llama8b", 16), ("heavytail", 8),
                                     ("prefix", 16)])
def test_oracle_arm_inputs_equal_the_workload(name, bs):
    w = inputs.WORKLOADS[name]
    q, k, v, tables, ctx = bench.oracle_inputs(w, bs)
    b = wl.build(w, device="cpu", block_size=bs, layers=1) if name != "prefix" else \
        wl.build_prefix_decode(w, device="cpu")
    assert np.array_equal(ctx, b.context_lens.numpy())
    n = [(-(-int(c) // bs)) for c in ctx]
    for i, m in enumerate(n):                        # entries past a table's end are junk
        assert np.array_equal(tables[i, :m], b.block_tables.numpy()[i, :m])
    assert np.array_equal(q, bits(b.q[0]))
    assert np.array_equal(k, bits(b.k_caches[0])) and np.array_equal(v, bits(b.v_caches[0]))
