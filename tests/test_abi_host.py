"""The C-ABI library builds for sm_100a, loads, exports every symbol its header
declares, and validates arguments on the host (no GPU needed: nothing here launches)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest
import torch

from paged_kv_cache_348_b200 import build as pbuild
from paged_kv_cache_348_b200 import pagedkv as pk

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "pagedkv.h")


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return pk.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(pa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_exports(lib):
    names = declared_functions()
    assert names == sorted(pk.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.pa_version() == 100
    assert lib.pa_status_string(0) == b"ok"
    assert lib.pa_status_string(2) == b"unsupported shape or dtype"


P = ctypes.c_void_p


def _decode(lib, B=4, Hq=8, Hkv=2, D=128, bs=16, M=4, N=64, dtype=0, ptr=P(4096), ws=1 << 30):
    return lib.pa_decode(ptr, ptr, ptr, ptr, ptr, ptr, B, Hq, Hkv, D, bs, M, N, 0.1, dtype, ptr, ws,
                         None, None)


def test_decode_host_validation(lib):
    assert _decode(lib, D=96) == pk.PA_ERR_UNSUPPORTED
    assert _decode(lib, bs=4) == pk.PA_ERR_UNSUPPORTED
    assert _decode(lib, Hq=9, Hkv=2) == pk.PA_ERR_INVALID
    assert _decode(lib, Hq=72, Hkv=1) == pk.PA_ERR_UNSUPPORTED      # group 72 > 64
    assert _decode(lib, dtype=7) == pk.PA_ERR_UNSUPPORTED
    assert _decode(lib, B=0) == pk.PA_OK                              # nothing to do
    assert _decode(lib, ptr=P(0)) == pk.PA_ERR_INVALID                # null pointers
    assert _decode(lib, ptr=P(4104)) == pk.PA_ERR_INVALID             # not 16-byte aligned
    assert _decode(lib, N=1 << 30) == pk.PA_ERR_INVALID               # rows overflow int32
    if not torch.cuda.is_available():
        assert _decode(lib) == pk.PA_ERR_CUDA                         # no device to run on
        assert lib.pa_decode_workspace_bytes(4, 8, 2, 128) == 0


def test_append_and_copy_host_validation(lib):
    p = P(4096)
    assert lib.pa_cache_append(p, p, p, p, p, 0, 8, 128, 16, 10, 0, None, None) == pk.PA_OK
    assert lib.pa_cache_append(p, p, p, P(0), p, 3, 8, 128, 16, 10, 0, None, None) == \
        pk.PA_ERR_INVALID
    assert lib.pa_cache_append(p, p, p, p, p, 3, 8, 100, 16, 10, 5, None, None) == \
        pk.PA_ERR_UNSUPPORTED
    arr = (ctypes.c_void_p * 2)(4096, 8192)
    assert lib.pa_copy_blocks(arr, arr, 2, p, 0, 10, 4096, None, None) == pk.PA_OK
    assert lib.pa_copy_blocks(arr, arr, 2, p, 3, 10, 4100, None, None) == pk.PA_ERR_INVALID
    bad = (ctypes.c_void_p * 2)(4096, 0)
    assert lib.pa_copy_blocks(bad, arr, 2, p, 3, 10, 4096, None, None) == pk.PA_ERR_INVALID


def test_wait_check_host_validation(lib):
    """pa_check_bounded_waits rejects a null or misaligned result and limits out of range
    on the host, before anything is launched."""
    assert lib.pa_check_bounded_waits(None, 100, None) == pk.PA_ERR_INVALID
    assert lib.pa_check_bounded_waits(P(4098), 100, None) == pk.PA_ERR_INVALID
    assert lib.pa_check_bounded_waits(P(4096), 0, None) == pk.PA_ERR_INVALID
    assert lib.pa_check_bounded_waits(P(4096), 2000001, None) == pk.PA_ERR_INVALID


def test_binding_refuses_cpu_tensors(lib):
    q = torch.zeros(2, 4, 64, dtype=torch.float16)
    with pytest.raises(pk.PagedKVError, match="CUDA tensor"):
        pk.pa_decode(q, q, q.view(2, 4, 1, 64), q.view(2, 4, 1, 64),
                     torch.zeros(2, 1, dtype=torch.int32), torch.zeros(2, dtype=torch.int32), 1.0,
                     torch.zeros(16, dtype=torch.uint8))
