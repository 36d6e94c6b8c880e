"""CPU oracle for paged KV-cache decode.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It never touches a GPU
and shares no code with the CUDA library under ``paged_kv_cache_348_b200/``.

The arithmetic lives in ``pagedkv_oracle.c`` (plain C, fp64); this module only
builds it with gcc and marshals numpy arrays through ctypes.  The copy-on-write
planner (pure Python bookkeeping, no arithmetic on values) is in ``cow.py``.

All 16-bit tensors are passed as ``numpy.uint16`` bit patterns; ``dtype`` is
``"f16"`` or ``"bf16"``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

DTYPES = {"f16": 0, "bf16": 1}


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u16, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint16, ctypes.c_double
        L.orc_f16_to_f64.argtypes = [u16]; L.orc_f16_to_f64.restype = f64
        L.orc_bf16_to_f64.argtypes = [u16]; L.orc_bf16_to_f64.restype = f64
        L.orc_f64_to_f16.argtypes = [f64]; L.orc_f64_to_f16.restype = u16
        L.orc_f64_to_bf16.argtypes = [f64]; L.orc_f64_to_bf16.restype = u16
        L.orc_kv_bytes_per_token.argtypes = [i32, i32, i32, i32]
        L.orc_kv_bytes_per_token.restype = i64
        L.orc_gather.argtypes = [P, P, i32, i32, i32, i32, i32, P, i32, i32]
        L.orc_gather.restype = i32
        L.orc_decode.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                 f64, i32, P, i32, i32]
        L.orc_decode.restype = i32
        L.orc_decode_multi.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                       i32, f64, i32, P, i32, i32]
        L.orc_decode_multi.restype = i32
        u8, f32 = ctypes.c_uint8, ctypes.c_float
        L.orc_e4m3_to_f64.argtypes = [u8]; L.orc_e4m3_to_f64.restype = f64
        L.orc_f64_to_e4m3.argtypes = [f64]; L.orc_f64_to_e4m3.restype = u8
        L.orc_quantize_e4m3.argtypes = [u16, i32, f32]; L.orc_quantize_e4m3.restype = u8
        L.orc_decode_e4m3.argtypes = [P, P, P, P, P, f64, f64, P, P, i32, i32, i32, i32, i32, i32,
                                      i32, i32, f64, i32, P, i32, i32]
        L.orc_decode_e4m3.restype = i32
        L.orc_cache_append_e4m3.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, f32]
        L.orc_cache_append_e4m3.restype = i32
        L.orc_e4m3_block_scale.argtypes = [f32]; L.orc_e4m3_block_scale.restype = f32
        L.orc_cache_append_e4m3_bs.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32]
        L.orc_cache_append_e4m3_bs.restype = i32
        L.orc_decode_e4m3_bs.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                         i32, i32, f64, i32, P, i32, i32]
        L.orc_decode_e4m3_bs.restype = i32
        L.orc_cache_append.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32]
        L.orc_cache_append.restype = i32
        L.orc_copy_blocks.argtypes = [P, P, i32, P, i32, i64, i32]
        L.orc_copy_blocks.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ---- scalar conversions --------------------------------------------------------------
def to_f64(bits: int, dtype: str) -> float:
    L = _load()
    return L.orc_bf16_to_f64(bits) if dtype == "bf16" else L.orc_f16_to_f64(bits)


def from_f64(x: float, dtype: str) -> int:
    L = _load()
    return L.orc_f64_to_bf16(x) if dtype == "bf16" else L.orc_f64_to_f16(x)


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    return _load().orc_kv_bytes_per_token(layers, kv_heads, head_dim, elem_bytes)


# ---- gather / decode / append / copy -------------------------------------------------
def gather(cache: np.ndarray, dtype: str, table_row: np.ndarray, ctx: int, kvh: int) -> np.ndarray:
    """Logical rows 0..ctx-1 of one sequence/kv head, fp64 [ctx, D]."""
    cache = _c(cache, np.uint16)
    N, Hkv, bs, D = cache.shape
    tr = _c(table_row, np.int32)
    out = np.zeros((max(ctx, 0), D), dtype=np.float64)
    rc = _load().orc_gather(_p(out), _p(cache), DTYPES[dtype], N, Hkv, bs, D, _p(tr), ctx, kvh)
    if rc:
        raise ValueError("oracle gather: block id out of range")
    return out


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype: str,
           items=None, nthreads: int = 1):
    """fp64 paged decode.  Returns (out64 [B,Hq,D] float64, out16 [B,Hq,D] uint16).

    ``items`` restricts the computation to a list of sequence indices (the other
    rows are returned as zeros)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B
    out64 = np.zeros((B, Hq, D), dtype=np.float64)
    out16 = np.zeros((B, Hq, D), dtype=np.uint16)
    it = None if items is None else _c(items, np.int32)
    rc = _load().orc_decode(_p(out64), _p(out16), _p(q), _p(k_cache), _p(v_cache), _p(bt), _p(cl),
                            B, Hq, Hkv, D, bs, bt.shape[1], N, float(scale), DTYPES[dtype],
                            None if it is None else _p(it), 0 if it is None else len(it),
                            int(nthreads))
    if rc == -1:
        raise ValueError("oracle decode: block id out of range")
    if rc:
        raise ValueError("oracle decode: bad arguments (%d)" % rc)
    return out64, out16


def decode_multi(q, k_cache, v_cache, block_tables, context_lens, scale: float, dtype: str,
                 items=None, nthreads: int = 1):
    """fp64 paged decode of q_len new tokens per sequence, causal among them.

    q is [B, q_len, Hq, D]; new token j of sequence s sits at position
    ctx - q_len + j and attends to positions 0 .. ctx - q_len + j.  Returns
    (out64 [B,q_len,Hq,D] float64, out16 [B,q_len,Hq,D] uint16)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, QL, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B
    out64 = np.zeros((B, QL, Hq, D), dtype=np.float64)
    out16 = np.zeros((B, QL, Hq, D), dtype=np.uint16)
    it = None if items is None else _c(items, np.int32)
    rc = _load().orc_decode_multi(_p(out64), _p(out16), _p(q), _p(k_cache), _p(v_cache), _p(bt),
                                  _p(cl), B, QL, Hq, Hkv, D, bs, bt.shape[1], N, float(scale),
                                  DTYPES[dtype], None if it is None else _p(it),
                                  0 if it is None else len(it), int(nthreads))
    if rc == -1:
        raise ValueError("oracle decode: block id out of range")
    if rc:
        raise ValueError("oracle decode: bad arguments (%d)" % rc)
    return out64, out16


# ---- 8-bit E4M3 cache ----------------------------------------------------------------
def e4m3_to_f64(code: int) -> float:
    return _load().orc_e4m3_to_f64(int(code))


def f64_to_e4m3(x: float) -> int:
    """Round to nearest even, magnitudes above 448 clamped to 448, NaN kept."""
    return _load().orc_f64_to_e4m3(float(x))


def quantize_e4m3(bits: int, dtype: str, scale: float) -> int:
    """Code of a 16-bit value for a per-tensor scale (x / scale in binary32, then E4M3)."""
    return _load().orc_quantize_e4m3(int(bits), DTYPES[dtype], float(scale))


def cache_append_e4m3(k_cache8, v_cache8, k, v, slot_mapping, dtype: str, k_scale: float,
                      v_scale: float):
    """In-place quantising scatter of 16-bit k/v [T, Hkv, D] into uint8 E4M3 pools."""
    assert k_cache8.flags.c_contiguous and v_cache8.flags.c_contiguous
    assert k_cache8.dtype == np.uint8 and v_cache8.dtype == np.uint8
    N, Hkv, bs, D = k_cache8.shape
    k = _c(k, np.uint16); v = _c(v, np.uint16)
    sm = _c(slot_mapping, np.int64)
    rc = _load().orc_cache_append_e4m3(_p(k_cache8), _p(v_cache8), _p(k), _p(v), _p(sm), len(sm),
                                       Hkv, D, bs, N, DTYPES[dtype], float(k_scale), float(v_scale))
    if rc:
        raise ValueError("oracle append: slot out of range")


def decode_e4m3(q, k_cache8, v_cache8, k_scale: float, v_scale: float, block_tables,
                context_lens, scale: float, dtype: str, items=None, nthreads: int = 1):
    """fp64 paged decode over uint8 E4M3 pools (values k_scale * code, v_scale * code);
    q [B, Hq, D] or [B, q_len, Hq, D] in `dtype`.  Returns (out64, out16) shaped like q."""
    q = _c(q, np.uint16)
    k8 = _c(k_cache8, np.uint8)
    v8 = _c(v_cache8, np.uint8)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    shape = q.shape
    q4 = q.reshape(shape[0], 1, shape[1], shape[2]) if q.ndim == 3 else q
    B, QL, Hq, D = q4.shape
    N, Hkv, bs, D2 = k8.shape
    assert D2 == D and v8.shape == k8.shape and bt.shape[0] == B
    out64 = np.zeros((B, QL, Hq, D), dtype=np.float64)
    out16 = np.zeros((B, QL, Hq, D), dtype=np.uint16)
    it = None if items is None else _c(items, np.int32)
    rc = _load().orc_decode_e4m3(_p(out64), _p(out16), _p(q4), _p(k8), _p(v8), float(k_scale),
                                 float(v_scale), _p(bt), _p(cl), B, QL, Hq, Hkv, D, bs, bt.shape[1],
                                 N, float(scale), DTYPES[dtype], None if it is None else _p(it),
                                 0 if it is None else len(it), int(nthreads))
    if rc == -1:
        raise ValueError("oracle decode: block id out of range")
    if rc:
        raise ValueError("oracle decode: bad arguments (%d)" % rc)
    return out64.reshape(shape), out16.reshape(shape)


def e4m3_block_scale(amax: float) -> float:
    """Scale of an 8-bit block's (block, kv head) slice fixed by its offset-0 token, whose
    row has largest magnitude amax: 2^(ceil(log2(amax / 448)) + 3), 1 for amax 0."""
    return float(_load().orc_e4m3_block_scale(float(amax)))


def cache_append_e4m3_bs(k_cache8, v_cache8, k_scales, v_scales, k, v, slot_mapping, dtype: str):
    """In-place quantising scatter with per-(block, kv head) scales (float32 [N, Hkv],
    updated for the blocks whose offset 0 is written here)."""
    for a in (k_cache8, v_cache8, k_scales, v_scales):
        assert a.flags.c_contiguous
    assert k_cache8.dtype == np.uint8 and v_cache8.dtype == np.uint8
    assert k_scales.dtype == np.float32 and v_scales.dtype == np.float32
    N, Hkv, bs, D = k_cache8.shape
    assert k_scales.shape == (N, Hkv) and v_scales.shape == (N, Hkv)
    k = _c(k, np.uint16); v = _c(v, np.uint16)
    sm = _c(slot_mapping, np.int64)
    rc = _load().orc_cache_append_e4m3_bs(_p(k_cache8), _p(v_cache8), _p(k_scales), _p(v_scales),
                                          _p(k), _p(v), _p(sm), len(sm), Hkv, D, bs, N,
                                          DTYPES[dtype])
    if rc:
        raise ValueError("oracle append: slot out of range")


def decode_e4m3_bs(q, k_cache8, v_cache8, k_scales, v_scales, block_tables, context_lens,
                   scale: float, dtype: str, items=None, nthreads: int = 1):
    """fp64 paged decode over uint8 E4M3 pools with per-(block, kv head) scales (value of
    block b, head h = scales[b][h] * code); q [B, Hq, D] or [B, q_len, Hq, D]."""
    q = _c(q, np.uint16)
    k8 = _c(k_cache8, np.uint8)
    v8 = _c(v_cache8, np.uint8)
    ks = _c(k_scales, np.float32)
    vs = _c(v_scales, np.float32)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    shape = q.shape
    q4 = q.reshape(shape[0], 1, shape[1], shape[2]) if q.ndim == 3 else q
    B, QL, Hq, D = q4.shape
    N, Hkv, bs, D2 = k8.shape
    assert D2 == D and v8.shape == k8.shape and bt.shape[0] == B
    assert ks.shape == (N, Hkv) and vs.shape == (N, Hkv)
    out64 = np.zeros((B, QL, Hq, D), dtype=np.float64)
    out16 = np.zeros((B, QL, Hq, D), dtype=np.uint16)
    it = None if items is None else _c(items, np.int32)
    rc = _load().orc_decode_e4m3_bs(_p(out64), _p(out16), _p(q4), _p(k8), _p(v8), _p(ks), _p(vs),
                                    _p(bt), _p(cl), B, QL, Hq, Hkv, D, bs, bt.shape[1], N,
                                    float(scale), DTYPES[dtype], None if it is None else _p(it),
                                    0 if it is None else len(it), int(nthreads))
    if rc == -1:
        raise ValueError("oracle decode: block id out of range")
    if rc:
        raise ValueError("oracle decode: bad arguments (%d)" % rc)
    return out64.reshape(shape), out16.reshape(shape)


def cache_append(k_cache, v_cache, k, v, slot_mapping):
    """In-place scatter of k/v [T, Hkv, D] into the pools; negative slots are skipped."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    N, Hkv, bs, D = k_cache.shape
    k = _c(k, np.uint16); v = _c(v, np.uint16)
    sm = _c(slot_mapping, np.int64)
    rc = _load().orc_cache_append(_p(k_cache), _p(v_cache), _p(k), _p(v), _p(sm), len(sm), Hkv, D,
                                  bs, N)
    if rc:
        raise ValueError("oracle append: slot out of range")


def copy_blocks(k_caches, v_caches, pairs):
    """In-place copy of block src -> dst for every (src, dst) pair and every layer."""
    L = len(k_caches)
    N = k_caches[0].shape[0]
    block_elems = int(np.prod(k_caches[0].shape[1:]))
    for a in list(k_caches) + list(v_caches):
        assert a.flags.c_contiguous and a.dtype == np.uint16 and a.shape[0] == N
    kp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in k_caches])
    vp = (ctypes.c_void_p * L)(*[a.ctypes.data for a in v_caches])
    pr = _c(pairs, np.int32).reshape(-1, 2)
    rc = _load().orc_copy_blocks(kp, vp, L, _p(pr), len(pr), block_elems, N)
    if rc:
        raise ValueError("oracle copy_blocks: block id out of range")
