"""ctypes binding of libpagedkv (the C ABI in include/pagedkv.h).

Argument marshalling only: shapes are read from torch tensors, pointers and the
current CUDA stream are passed through, and every step runs in the CUDA library.
There is no fallback: if ``libpagedkv.so`` is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_NO_BLOCKS, PA_ERR_NO_MEMORY = \
    0, 1, 2, 3, 4, 5
PA_F16, PA_BF16 = 0, 1
DEV_BAD_BLOCK_ID, DEV_BAD_SLOT, DEV_BAD_PAIR, DEV_BAD_CONTEXT_LEN, DEV_TIMEOUT = (
    0x1, 0x2, 0x4, 0x8, 0x10)

# every symbol include/pagedkv.h declares
EXPORTS = ("pa_version", "pa_status_string", "pa_decode_workspace_bytes", "pa_decode",
           "pa_decode_multi", "pa_decode_append", "pa_cache_append_e4m3", "pa_decode_e4m3",
           "pa_decode_cascade_workspace_bytes",
           "pa_decode_cascade",
           "pa_cache_append", "pa_copy_blocks", "pa_decode_noalloc",
           "pa_bm_create", "pa_bm_destroy", "pa_bm_free_blocks", "pa_bm_refcount",
           "pa_bm_allocate", "pa_bm_fork", "pa_bm_append_tokens", "pa_bm_release",
           "pa_bm_context_len", "pa_bm_num_blocks_of", "pa_bm_max_blocks", "pa_bm_block_tables",
           "pa_bm_slot_of", "pa_bm_plan_cascade", "pa_plan_cascade", "pa_bm_swap_out",
           "pa_bm_swap_in", "pa_swap_out_blocks", "pa_swap_in_blocks", "pa_cache_append_e4m3_bs",
           "pa_decode_e4m3_bs", "pa_decode_cascade_e4m3_bs", "pa_decode_append_e4m3_bs",
           "pa_check_bounded_waits")

_lib = None
_lock = threading.Lock()


class PagedKVError(RuntimeError):
    pass


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise PagedKVError("libpagedkv.so not found at %s: build it with "
                               "`python paged_kv_cache_348_b200/build.py`" % path)
        L = ctypes.CDLL(path)
        P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.pa_version.restype = i32
        L.pa_version.argtypes = []
        L.pa_status_string.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [i32]
        L.pa_decode_workspace_bytes.restype = sz
        L.pa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.pa_decode.restype = i32
        L.pa_decode.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                P, sz, P, P]
        L.pa_decode_multi.restype = i32
        L.pa_decode_multi.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, i32,
                                      f32, i32, P, sz, P, P]
        L.pa_check_bounded_waits.restype = i32
        L.pa_check_bounded_waits.argtypes = [P, i32, P]
        L.pa_decode_append.restype = i32
        L.pa_decode_append.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                       f32, i32, P, sz, P, P]
        L.pa_cache_append_e4m3.restype = i32
        L.pa_cache_append_e4m3.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, f32,
                                           P, P]
        L.pa_decode_e4m3.restype = i32
        L.pa_decode_e4m3.argtypes = [P, P, P, P, f32, f32, P, P, i32, i32, i32, i32, i32, i32, i32,
                                     f32, i32, P, sz, P, P]
        L.pa_cache_append_e4m3_bs.restype = i32
        L.pa_cache_append_e4m3_bs.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                              P, P]
        L.pa_decode_e4m3_bs.restype = i32
        L.pa_decode_e4m3_bs.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                        i32, f32, i32, P, sz, P, P]
        L.pa_decode_cascade_e4m3_bs.restype = i32
        L.pa_decode_cascade_e4m3_bs.argtypes = [P, P, P, P, P, P, P, P, P, i32, P, i32, P, i32,
                                                i32, i32, i32, i32, i32, i32, f32, i32, P, sz, P,
                                                P]
        L.pa_decode_append_e4m3_bs.restype = i32
        L.pa_decode_append_e4m3_bs.argtypes = [P, P, P, P, P, P, P, P, P, P, i32, i32, i32, i32,
                                               i32, i32, i32, f32, i32, P, sz, P, P]
        L.pa_decode_cascade_workspace_bytes.restype = sz
        L.pa_decode_cascade_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.pa_decode_cascade.restype = i32
        L.pa_decode_cascade.argtypes = [P, P, P, P, P, P, P, i32, P, i32, P, i32, i32, i32, i32,
                                        i32, i32, i32, f32, i32, P, sz, P, P]
        L.pa_cache_append.restype = i32
        L.pa_cache_append.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, P, P]
        L.pa_copy_blocks.restype = i32
        L.pa_copy_blocks.argtypes = [P, P, i32, P, i32, i32, sz, P, P]
        L.pa_swap_out_blocks.restype = i32
        L.pa_swap_out_blocks.argtypes = [P, P, P, i32, P, i32, i32, sz, P, P]
        L.pa_swap_in_blocks.restype = i32
        L.pa_swap_in_blocks.argtypes = [P, P, i32, P, i32, i32, P, sz, P, P]
        _lib = L
        return L


def _check(rc: int, what: str):
    if rc != PA_OK:
        msg = load().pa_status_string(rc).decode()
        raise PagedKVError("%s failed: %s (%d)" % (what, msg, rc))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise PagedKVError("unsupported dtype %s" % t.dtype)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not t.is_cuda:
        raise PagedKVError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise PagedKVError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise PagedKVError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if ndim is not None and t.dim() != ndim:
        raise PagedKVError("%s must have %d dims" % (name, ndim))


def pa_version() -> int:
    return load().pa_version()


def pa_decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                              head_dim: int) -> int:
    return int(load().pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim))


def new_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, device=None) -> torch.Tensor:
    n = pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pa_check_bounded_waits(limit_us: int, stream=None) -> list:
    """Run the library's bounded-wait diagnostic (see pa_check_bounded_waits in
    include/pagedkv.h) on the current device and return its four results: barrier wait
    gave up, count wait gave up, and how long each took in microseconds."""
    result = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    _check(load().pa_check_bounded_waits(_ptr(result), int(limit_us), _stream(stream)),
           "pa_check_bounded_waits")
    return [int(x) for x in result.cpu()]


def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float, workspace,
              status=None, stream=None):
    """out[B,Hq,D] <- paged decode attention (see pa_decode in include/pagedkv.h)."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache, "k_cache", dtype=q.dtype, ndim=4)
    _need(v_cache, "v_cache", dtype=q.dtype, ndim=4)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PagedKVError("pa_decode: inconsistent shapes")
    rc = load().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                          _ptr(context_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], N,
                          float(scale), _dtype_code(q), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _ptr(status),
                          _stream(stream))
    _check(rc, "pa_decode")
    return out


def pa_decode_multi(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                    workspace, status=None, stream=None):
    """out[B,QL,Hq,D] <- paged decode of QL new tokens per sequence, causal among them
    (see pa_decode_multi in include/pagedkv.h)."""
    _need(q, "q", ndim=4)
    _need(out, "out", dtype=q.dtype, ndim=4)
    _need(k_cache, "k_cache", dtype=q.dtype, ndim=4)
    _need(v_cache, "v_cache", dtype=q.dtype, ndim=4)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, QL, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PagedKVError("pa_decode_multi: inconsistent shapes")
    rc = load().pa_decode_multi(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), _ptr(context_lens), B, QL, Hq, Hkv, D, bs,
                                block_tables.shape[1], N, float(scale), _dtype_code(q),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(status), _stream(stream))
    _check(rc, "pa_decode_multi")
    return out


def pa_decode_append(out, q, k_cache, v_cache, k_new, v_new, block_tables, context_lens,
                     scale: float, workspace, status=None, stream=None):
    """Append each sequence's newest token (k_new/v_new [B,Hkv,D], at position
    context_lens-1) into the caches and decode, in one launch (see pa_decode_append in
    include/pagedkv.h)."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache, "k_cache", dtype=q.dtype, ndim=4)
    _need(v_cache, "v_cache", dtype=q.dtype, ndim=4)
    _need(k_new, "k_new", dtype=q.dtype, ndim=3)
    _need(v_new, "v_new", dtype=q.dtype, ndim=3)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape or \
            k_new.shape != (B, Hkv, D) or v_new.shape != k_new.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PagedKVError("pa_decode_append: inconsistent shapes")
    rc = load().pa_decode_append(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new),
                                 _ptr(v_new), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
                                 D, bs, block_tables.shape[1], N, float(scale), _dtype_code(q),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _ptr(status), _stream(stream))
    _check(rc, "pa_decode_append")
    return out


def pa_cache_append_e4m3(k_cache8, v_cache8, k, v, slot_mapping, k_scale: float, v_scale: float,
                         status=None, stream=None):
    """Quantising scatter of 16-bit k/v [T,Hkv,D] into uint8 E4M3 pools (see
    pa_cache_append_e4m3 in include/pagedkv.h)."""
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(k, "k", ndim=3)
    _need(v, "v", dtype=k.dtype, ndim=3)
    _need(slot_mapping, "slot_mapping", dtype=torch.int64, ndim=1)
    N, Hkv, bs, D = k_cache8.shape
    T = k.shape[0]
    if v_cache8.shape != k_cache8.shape or k.shape != (T, Hkv, D) or v.shape != k.shape or \
            slot_mapping.shape[0] != T:
        raise PagedKVError("pa_cache_append_e4m3: inconsistent shapes")
    rc = load().pa_cache_append_e4m3(_ptr(k_cache8), _ptr(v_cache8), _ptr(k), _ptr(v),
                                     _ptr(slot_mapping), T, Hkv, D, bs, N, _dtype_code(k),
                                     float(k_scale), float(v_scale), _ptr(status), _stream(stream))
    _check(rc, "pa_cache_append_e4m3")


def pa_decode_e4m3(out, q, k_cache8, v_cache8, k_scale: float, v_scale: float, block_tables,
                   context_lens, scale: float, workspace, status=None, stream=None):
    """out[B,Hq,D] <- paged decode over uint8 E4M3 pools (see pa_decode_e4m3)."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache8.shape
    if out.shape != q.shape or D2 != D or v_cache8.shape != k_cache8.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PagedKVError("pa_decode_e4m3: inconsistent shapes")
    rc = load().pa_decode_e4m3(_ptr(out), _ptr(q), _ptr(k_cache8), _ptr(v_cache8), float(k_scale),
                               float(v_scale), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv,
                               D, bs, block_tables.shape[1], N, float(scale), _dtype_code(q),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(status), _stream(stream))
    _check(rc, "pa_decode_e4m3")
    return out


def pa_cache_append_e4m3_bs(k_cache8, v_cache8, k_scales, v_scales, k, v, slot_mapping,
                            status=None, stream=None):
    """Quantising scatter of 16-bit k/v [T,Hkv,D] into uint8 E4M3 pools with per-(block,
    kv head) scales (float32 [N,Hkv], set for blocks whose offset 0 is written); see
    pa_cache_append_e4m3_bs in include/pagedkv.h."""
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(k_scales, "k_scales", dtype=torch.float32, ndim=2)
    _need(v_scales, "v_scales", dtype=torch.float32, ndim=2)
    _need(k, "k", ndim=3)
    _need(v, "v", dtype=k.dtype, ndim=3)
    _need(slot_mapping, "slot_mapping", dtype=torch.int64, ndim=1)
    N, Hkv, bs, D = k_cache8.shape
    T = k.shape[0]
    if v_cache8.shape != k_cache8.shape or k.shape != (T, Hkv, D) or v.shape != k.shape or \
            slot_mapping.shape[0] != T or k_scales.shape != (N, Hkv) or \
            v_scales.shape != (N, Hkv):
        raise PagedKVError("pa_cache_append_e4m3_bs: inconsistent shapes")
    rc = load().pa_cache_append_e4m3_bs(_ptr(k_cache8), _ptr(v_cache8), _ptr(k_scales),
                                        _ptr(v_scales), _ptr(k), _ptr(v), _ptr(slot_mapping), T,
                                        Hkv, D, bs, N, _dtype_code(k), _ptr(status),
                                        _stream(stream))
    _check(rc, "pa_cache_append_e4m3_bs")


def pa_decode_e4m3_bs(out, q, k_cache8, v_cache8, k_scales, v_scales, block_tables,
                      context_lens, scale: float, workspace, status=None, stream=None):
    """out <- paged decode over uint8 E4M3 pools with per-(block, kv head) scales; q and
    out [B,Hq,D] (one new token) or [B,QL,Hq,D] (QL new tokens, causal); see
    pa_decode_e4m3_bs in include/pagedkv.h."""
    if q.dim() not in (3, 4):
        raise PagedKVError("q must have 3 or 4 dims")
    _need(q, "q")
    _need(out, "out", dtype=q.dtype, ndim=q.dim())
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(k_scales, "k_scales", dtype=torch.float32, ndim=2)
    _need(v_scales, "v_scales", dtype=torch.float32, ndim=2)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, QL = q.shape[0], (q.shape[1] if q.dim() == 4 else 1)
    Hq, D = q.shape[-2], q.shape[-1]
    N, Hkv, bs, D2 = k_cache8.shape
    if out.shape != q.shape or D2 != D or v_cache8.shape != k_cache8.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B or \
            k_scales.shape != (N, Hkv) or v_scales.shape != (N, Hkv):
        raise PagedKVError("pa_decode_e4m3_bs: inconsistent shapes")
    rc = load().pa_decode_e4m3_bs(_ptr(out), _ptr(q), _ptr(k_cache8), _ptr(v_cache8),
                                  _ptr(k_scales), _ptr(v_scales), _ptr(block_tables),
                                  _ptr(context_lens), B, QL, Hq, Hkv, D, bs,
                                  block_tables.shape[1], N, float(scale), _dtype_code(q),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _ptr(status), _stream(stream))
    _check(rc, "pa_decode_e4m3_bs")
    return out


def new_cascade_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, device=None):
    n = int(load().pa_decode_cascade_workspace_bytes(num_seqs, num_q_heads, num_kv_heads,
                                                     head_dim))
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def pa_decode_cascade(out, q, k_cache, v_cache, block_tables, context_lens, prefix_lens,
                      chunk_members, chunk_prefix_lens, scale: float, workspace, status=None,
                      stream=None):
    """out[B,Hq,D] <- paged decode where chunks of sequences share a KV prefix (see
    pa_decode_cascade in include/pagedkv.h).  chunk_members is int32 [C, W] (-1 pad,
    group * W <= 64), chunk_prefix_lens int32 [C], prefix_lens int32 [B]."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache, "k_cache", dtype=q.dtype, ndim=4)
    _need(v_cache, "v_cache", dtype=q.dtype, ndim=4)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(prefix_lens, "prefix_lens", dtype=torch.int32, ndim=1)
    _need(chunk_members, "chunk_members", dtype=torch.int32, ndim=2)
    _need(chunk_prefix_lens, "chunk_prefix_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    C = chunk_members.shape[0]
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B or \
            prefix_lens.shape[0] != B or chunk_prefix_lens.shape[0] != C:
        raise PagedKVError("pa_decode_cascade: inconsistent shapes")
    rc = load().pa_decode_cascade(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(block_tables), _ptr(context_lens), _ptr(prefix_lens), B,
                                  _ptr(chunk_members), chunk_members.shape[1],
                                  _ptr(chunk_prefix_lens), C, Hq, Hkv, D, bs,
                                  block_tables.shape[1], N, float(scale), _dtype_code(q),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _ptr(status), _stream(stream))
    _check(rc, "pa_decode_cascade")
    return out


def pa_decode_cascade_e4m3_bs(out, q, k_cache8, v_cache8, k_scales, v_scales, block_tables,
                              context_lens, prefix_lens, chunk_members, chunk_prefix_lens,
                              scale: float, workspace, status=None, stream=None):
    """pa_decode_cascade over uint8 E4M3 pools with per-(block, kv head) scales (float32
    [N,Hkv]); group * W <= 16 (see pa_decode_cascade_e4m3_bs in include/pagedkv.h)."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(k_scales, "k_scales", dtype=torch.float32, ndim=2)
    _need(v_scales, "v_scales", dtype=torch.float32, ndim=2)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(prefix_lens, "prefix_lens", dtype=torch.int32, ndim=1)
    _need(chunk_members, "chunk_members", dtype=torch.int32, ndim=2)
    _need(chunk_prefix_lens, "chunk_prefix_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache8.shape
    C = chunk_members.shape[0]
    if out.shape != q.shape or D2 != D or v_cache8.shape != k_cache8.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B or \
            prefix_lens.shape[0] != B or chunk_prefix_lens.shape[0] != C or \
            k_scales.shape != (N, Hkv) or v_scales.shape != (N, Hkv):
        raise PagedKVError("pa_decode_cascade_e4m3_bs: inconsistent shapes")
    rc = load().pa_decode_cascade_e4m3_bs(
        _ptr(out), _ptr(q), _ptr(k_cache8), _ptr(v_cache8), _ptr(k_scales), _ptr(v_scales),
        _ptr(block_tables), _ptr(context_lens), _ptr(prefix_lens), B, _ptr(chunk_members),
        chunk_members.shape[1], _ptr(chunk_prefix_lens), C, Hq, Hkv, D, bs,
        block_tables.shape[1], N, float(scale), _dtype_code(q), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(rc, "pa_decode_cascade_e4m3_bs")
    return out


def pa_decode_append_e4m3_bs(out, q, k_cache8, v_cache8, k_scales, v_scales, k_new, v_new,
                             block_tables, context_lens, scale: float, workspace, status=None,
                             stream=None):
    """Quantise each sequence's newest token (16-bit k_new/v_new [B,Hkv,D], position
    context_lens-1) into uint8 E4M3 pools with per-(block, kv head) scales and decode, in
    one launch (see pa_decode_append_e4m3_bs in include/pagedkv.h)."""
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache8, "k_cache", dtype=torch.uint8, ndim=4)
    _need(v_cache8, "v_cache", dtype=torch.uint8, ndim=4)
    _need(k_scales, "k_scales", dtype=torch.float32, ndim=2)
    _need(v_scales, "v_scales", dtype=torch.float32, ndim=2)
    _need(k_new, "k_new", dtype=q.dtype, ndim=3)
    _need(v_new, "v_new", dtype=q.dtype, ndim=3)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    _need(workspace, "workspace")
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache8.shape
    if out.shape != q.shape or D2 != D or v_cache8.shape != k_cache8.shape or \
            k_new.shape != (B, Hkv, D) or v_new.shape != k_new.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B or \
            k_scales.shape != (N, Hkv) or v_scales.shape != (N, Hkv):
        raise PagedKVError("pa_decode_append_e4m3_bs: inconsistent shapes")
    rc = load().pa_decode_append_e4m3_bs(
        _ptr(out), _ptr(q), _ptr(k_cache8), _ptr(v_cache8), _ptr(k_scales), _ptr(v_scales),
        _ptr(k_new), _ptr(v_new), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, D, bs,
        block_tables.shape[1], N, float(scale), _dtype_code(q), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream))
    _check(rc, "pa_decode_append_e4m3_bs")
    return out


def pa_cache_append(k_cache, v_cache, k, v, slot_mapping, status=None, stream=None):
    """Scatter k/v [T,Hkv,D] into the pools at slot_mapping (int64 [T])."""
    _need(k_cache, "k_cache", ndim=4)
    _need(v_cache, "v_cache", dtype=k_cache.dtype, ndim=4)
    _need(k, "k", dtype=k_cache.dtype, ndim=3)
    _need(v, "v", dtype=k_cache.dtype, ndim=3)
    _need(slot_mapping, "slot_mapping", dtype=torch.int64, ndim=1)
    N, Hkv, bs, D = k_cache.shape
    T = k.shape[0]
    if v_cache.shape != k_cache.shape or k.shape != (T, Hkv, D) or v.shape != k.shape or \
            slot_mapping.shape[0] != T:
        raise PagedKVError("pa_cache_append: inconsistent shapes")
    rc = load().pa_cache_append(_ptr(k_cache), _ptr(v_cache), _ptr(k), _ptr(v), _ptr(slot_mapping),
                                T, Hkv, D, bs, N, _dtype_code(k), _ptr(status), _stream(stream))
    _check(rc, "pa_cache_append")


def pa_copy_blocks(k_caches, v_caches, pairs, status=None, stream=None):
    """Copy block pairs[:,0] -> pairs[:,1] in every layer's K and V pool."""
    L = len(k_caches)
    if L != len(v_caches) or L == 0:
        raise PagedKVError("pa_copy_blocks: need the same non-zero number of K and V pools")
    shape, dt = k_caches[0].shape, k_caches[0].dtype
    for i, c in enumerate(list(k_caches) + list(v_caches)):
        _need(c, "cache[%d]" % i, dtype=dt, ndim=4)
        if c.shape != shape:
            raise PagedKVError("pa_copy_blocks: all pools must have one shape")
    _need(pairs, "pairs", dtype=torch.int32, ndim=2)
    if pairs.shape[1] != 2:
        raise PagedKVError("pairs must be [n, 2]")
    kp = (ctypes.c_void_p * L)(*[c.data_ptr() for c in k_caches])
    vp = (ctypes.c_void_p * L)(*[c.data_ptr() for c in v_caches])
    block_bytes = shape[1] * shape[2] * shape[3] * k_caches[0].element_size()
    rc = load().pa_copy_blocks(kp, vp, L, _ptr(pairs), pairs.shape[0], shape[0], block_bytes,
                               _ptr(status), _stream(stream))
    _check(rc, "pa_copy_blocks")


def _pool_args(k_caches, v_caches):
    L = len(k_caches)
    if L != len(v_caches) or L == 0:
        raise PagedKVError("need the same non-zero number of K and V pools")
    shape, dt = k_caches[0].shape, k_caches[0].dtype
    for i, c in enumerate(list(k_caches) + list(v_caches)):
        _need(c, "cache[%d]" % i, dtype=dt, ndim=4)
        if c.shape != shape:
            raise PagedKVError("all pools must have one shape")
    kp = (ctypes.c_void_p * L)(*[c.data_ptr() for c in k_caches])
    vp = (ctypes.c_void_p * L)(*[c.data_ptr() for c in v_caches])
    block_bytes = shape[1] * shape[2] * shape[3] * k_caches[0].element_size()
    return L, kp, vp, shape[0], block_bytes


def swap_buffer_bytes(k_caches, n: int) -> int:
    """Bytes of the buffer that holds n blocks of every layer's K and V pool."""
    c = k_caches[0]
    return len(k_caches) * 2 * n * c.shape[1] * c.shape[2] * c.shape[3] * c.element_size()


def pa_swap_out_blocks(buf, k_caches, v_caches, blocks, status=None, stream=None):
    """Save blocks (device int32 [n]) of every layer's K and V pool into buf (pinned host
    or device uint8, [layer][K|V][i][block]); see pa_swap_out_blocks in include/pagedkv.h."""
    L, kp, vp, N, bb = _pool_args(k_caches, v_caches)
    _need(blocks, "blocks", dtype=torch.int32, ndim=1)
    n = blocks.shape[0]
    if not buf.is_contiguous() or buf.numel() * buf.element_size() < L * 2 * n * bb:
        raise PagedKVError("pa_swap_out_blocks: buffer too small or not contiguous")
    rc = load().pa_swap_out_blocks(_ptr(buf), kp, vp, L, _ptr(blocks), n, N, bb, _ptr(status),
                                   _stream(stream))
    _check(rc, "pa_swap_out_blocks")


def pa_swap_in_blocks(k_caches, v_caches, blocks, buf, status=None, stream=None):
    """Restore buf (as written by pa_swap_out_blocks) into blocks (device int32 [n])."""
    L, kp, vp, N, bb = _pool_args(k_caches, v_caches)
    _need(blocks, "blocks", dtype=torch.int32, ndim=1)
    n = blocks.shape[0]
    if not buf.is_contiguous() or buf.numel() * buf.element_size() < L * 2 * n * bb:
        raise PagedKVError("pa_swap_in_blocks: buffer too small or not contiguous")
    rc = load().pa_swap_in_blocks(kp, vp, L, _ptr(blocks), n, N, _ptr(buf), bb, _ptr(status),
                                  _stream(stream))
    _check(rc, "pa_swap_in_blocks")


NOALLOC_MAX_SEQS = 16384


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                      status=None, stream=None):
    """pa_decode with the library's fixed device scratch instead of a workspace, for
    callers that cannot allocate device memory (see pa_decode_noalloc in
    include/pagedkv.h: at most NOALLOC_MAX_SEQS sequences; calls that may run at the
    same time on one device race on the shared scratch)."""
    L = load()
    fn = L.pa_decode_noalloc
    if fn.argtypes is None:
        P, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        fn.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, i32, P, P]
        fn.restype = i32
    _need(q, "q", ndim=3)
    _need(out, "out", dtype=q.dtype, ndim=3)
    _need(k_cache, "k_cache", dtype=q.dtype, ndim=4)
    _need(v_cache, "v_cache", dtype=q.dtype, ndim=4)
    _need(block_tables, "block_tables", dtype=torch.int32, ndim=2)
    _need(context_lens, "context_lens", dtype=torch.int32, ndim=1)
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape or \
            block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PagedKVError("pa_decode_noalloc: inconsistent shapes")
    rc = fn(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            _ptr(context_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], N, float(scale),
            _dtype_code(q), _ptr(status), _stream(stream))
    _check(rc, "pa_decode_noalloc")
    return out
