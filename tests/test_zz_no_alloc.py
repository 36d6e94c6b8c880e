"""pa_decode_noalloc: the decode entry point for callers that cannot allocate device
memory (a plug-in inside a host process whose allocator owns the GPU memory, or a
path where cudaMalloc's implicit synchronisation is not allowed).  Its scratch is a
fixed array inside the library; it must give the same results as pa_decode with a
caller workspace, call after call, although each call finds the previous call's
leftovers in that array.

This file is named to be collected last; it passes alone or after the other tests."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_348_b200 import pagedkv as pk
from tests.helpers import from_bits, make_case

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2


def _upload(case):
    dt = case["dtype"]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return (from_bits(case["q"], dt).cuda(), from_bits(case["k"], dt).cuda(),
            from_bits(case["v"], dt).cuda(), t(case["tables"]), t(case["ctx"]))


def _close(a: torch.Tensor, b: torch.Tensor):
    x, y = a.double().cpu().numpy(), b.double().cpu().numpy()
    assert np.isfinite(x).all()
    assert (np.abs(x - y) <= ATOL + RTOL * np.abs(y)).all(), np.abs(x - y).max()


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # two different batches back to back: long contexts so segments are split over CTAs
    # and the shared scratch holds partials; the second call sees the first's leftovers.
    # The third and fourth have 16 and 64 query rows per kv head: the tcgen05 kernel, whose
    # partials hold 64 rows per CTA.
    cases = [make_case(6, 64, 8, 128, 16, [7000, 5, 3000, 9100, 64, 4100], dtype="bf16", seed=81),
             make_case(9, 32, 8, 128, 8, [1, 2500, 700, 16, 8000, 333, 0, 4097, 60],
                       dtype="f16", seed=82),
             make_case(5, 128, 8, 128, 16, [9000, 3, 4500, 8191, 600], dtype="bf16", seed=84),
             make_case(4, 64, 1, 128, 32, [6000, 12000, 1, 2049], dtype="f16", seed=85)]
    st = pk.new_status()
    for case in cases:
        q, k, v, tables, ctx = _upload(case)
        ws = pk.new_workspace(case["B"], case["Hq"], case["Hkv"], case["D"])
        ref = torch.empty_like(q)
        pk.pa_decode(ref, q, k, v, tables, ctx, case["scale"], ws, st)
        out = torch.full_like(q, float("nan"))
        pk.pa_decode_noalloc(out, q, k, v, tables, ctx, case["scale"], st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        _close(out, ref)
        r64, _ = oracle.decode(case["q"], case["k"], case["v"], case["tables"], case["ctx"],
                               case["scale"], case["dtype"], nthreads=8)
        _close(out, torch.from_numpy(r64))


def test_noalloc_rejects_batches_beyond_its_scratch():
    case = make_case(2, 8, 2, 128, 16, [40, 50], dtype="f16", seed=83)
    q, k, v, tables, ctx = _upload(case)
    n = pk.NOALLOC_MAX_SEQS + 1
    big_q = q[:1].expand(n, -1, -1).contiguous()
    big_t = tables[:1].expand(n, -1).contiguous()
    big_c = ctx[:1].expand(n).contiguous()
    with pytest.raises(pk.PagedKVError, match="invalid argument"):
        pk.pa_decode_noalloc(torch.empty_like(big_q), big_q, k, v, big_t, big_c, 0.1)


def test_noalloc_allocates_no_device_memory():
    # one warm-up call loads the kernel instance this configuration uses; after it, calls
    # with other batch sizes (same dtype, head_dim, block_size and group) must leave the
    # device's free memory exactly as it was
    case = make_case(12, 32, 8, 128, 16, [900, 3, 4100, 17, 0, 2048, 65, 1, 700, 5000, 33, 129],
                     dtype="f16", seed=84)
    q, k, v, tables, ctx = _upload(case)
    out = torch.empty_like(q)
    st = pk.new_status()
    pk.pa_decode_noalloc(out, q, k, v, tables, ctx, case["scale"], st)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for n in (1, 5, 12, 7, 12, 2):
        pk.pa_decode_noalloc(out[:n], q[:n], k, v, tables[:n], ctx[:n], case["scale"], st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(st.item()) == 0
