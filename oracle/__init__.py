"""CPU fp64 oracle for paged single-token decode attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``paged_kv_cache_395_b200``) never imports it, and this package imports
nothing from the product.

What it computes, and the passages it follows (page, section):

* decode attention ``out = softmax(scale * q . K^T) . V`` over the logical
  tokens of each sequence (lqnn.cn/news/235768 section 1.2), with the token
  being decoded already appended (same page, section 2.2);
* the gather through the block table of fixed 16-token blocks
  (lqnn.cn/news/235768 section 3.2; chanyi.net.cn/article/49 section 三);
* GQA: query head ``h`` reads KV head ``h // (H_q // H_kv)``
  (lqnn.cn/news/235768 section 4.2; contiguous grouping is this library's
  reading);
* per-partition results and their log-sum-exp merge (the split form; exact
  algebra of the softmax, checked against the unsplit form);
* cache append (byte scatter), copy-on-write block copy (byte copy) and the
  symmetric absmax int8 quantiser with one scale per (block, KV head)
  (lqnn.cn/news/235768 section 4.1), its 4-bit form, and the append of single
  tokens into an int8 cache that raises a tile's scale when needed (this
  library's reading of the same section).

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64 loops).  This module
only marshals numpy arrays.  ``dense.py`` is an independent NumPy brute force
on unpaged K/V used to pin the C code.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32, F16, BF16, I8, I4 = 0, 1, 2, 3, 4

_lib = None


def load(path):
    """ctypes handle on an oracle library built at ``path``."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_half_to_double.restype = dbl
    L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_double.restype = dbl
    L.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, i64, i64]
    L.oracle_block_copy.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32]
    L.oracle_quantize_int8.argtypes = [P, i32, P, P, i64, i32, i32, i32]
    L.oracle_quantize_int4.argtypes = [P, i32, P, P, i64, i32, i32, i32]
    L.oracle_append_int8.argtypes = [P, P, i32, P, P, P, P, P, i64, i32, i32, i32, i64]
    L.oracle_decode.argtypes = [P, P, P, P, i32, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                i64, dbl, P, i64, i32]
    L.oracle_decode_partials.argtypes = [P, P, P, P, P, i32, P, P, P, P, i32, i32, i32, i32,
                                         i32, i32, i64, dbl, i32, i32, i32]
    L.oracle_decode_multi.argtypes = [P, P, P, P, i32, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                      i32, i64, dbl, i32]
    L.oracle_merge.argtypes = [P, P, P, i64, i32, i32]
    L.oracle_kv_bytes_per_token.argtypes = [i32, i32, i32, i32]
    L.oracle_kv_bytes_per_token.restype = i64
    for name in ("oracle_reshape_and_cache", "oracle_block_copy", "oracle_quantize_int8", "oracle_quantize_int4",
                 "oracle_decode", "oracle_decode_multi", "oracle_decode_partials", "oracle_merge"):
        getattr(L, name).restype = i32
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def dtype_code(dt) -> int:
    """Storage dtype -> oracle code.  bf16 arrays are carried as uint16 bit patterns."""
    dt = np.dtype(dt) if not isinstance(dt, str) else dt
    if dt == "bfloat16":
        return BF16
    # uint8 caches hold packed 4-bit values (two per byte)
    return {np.dtype(np.float32): F32, np.dtype(np.float16): F16, np.dtype(np.int8): I8,
            np.dtype(np.uint8): I4}[dt]


def _ptr(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def nthreads_default() -> int:
    return int(os.environ.get("PA_ORACLE_THREADS", os.cpu_count() or 1))


def half_to_double(bits: int) -> float:
    return lib().oracle_half_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits))


def reshape_and_cache(k, v, key_cache, value_cache, slot_mapping, code=None):
    """Scatter k, v ([T][H_kv][d], contiguous per token) into the caches in place."""
    T, H, d = k.shape
    N, Hc, bs, dc = key_cache.shape
    assert (H, d) == (Hc, dc) and v.shape == k.shape
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    code = dtype_code(key_cache.dtype) if code is None else code
    _check(lib().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(key_cache), _ptr(value_cache),
                                          _ptr(sm), T, H, d, bs, N, code, H * d, H * d),
           "oracle_reshape_and_cache")


def block_copy(key_cache, value_cache, pairs, k_scales=None, v_scales=None, code=None):
    N, H, bs, d = key_cache.shape
    pr = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    code = dtype_code(key_cache.dtype) if code is None else code
    head_dim = 2 * d if code == I4 else d  # a packed 4-bit row holds two values per byte
    _check(lib().oracle_block_copy(_ptr(key_cache), _ptr(value_cache), _ptr(k_scales),
                                   _ptr(v_scales), _ptr(pr), pr.shape[0], H, head_dim, bs, N, code),
           "oracle_block_copy")


def quantize_int8(src_cache, code=None):
    """Return (int8 cache, fp32 scales [N][H_kv]) for a [N][H_kv][bs][d] cache."""
    N, H, bs, d = src_cache.shape
    src = np.ascontiguousarray(src_cache)
    code = dtype_code(src.dtype) if code is None else code
    dst = np.empty(src.shape, dtype=np.int8)
    scales = np.empty((N, H), dtype=np.float32)
    _check(lib().oracle_quantize_int8(_ptr(src), code, _ptr(dst), _ptr(scales), N, H, d, bs),
           "oracle_quantize_int8")
    return dst, scales


def append_int8(k, v, key_cache8, value_cache8, k_scales, v_scales, slot_mapping, code=None):
    """Append tokens k, v ([T][H_kv][d], fp32/fp16/bf16) into int8 caches
    [N][H_kv][bs][d] with fp32 scales [N][H_kv], in place, raising a tile's scale
    and re-rounding its other codes when the token needs it (see pa_oracle.c)."""
    T, H, d = k.shape
    N, Hc, bs, dc = key_cache8.shape
    assert (H, d) == (Hc, dc) and v.shape == k.shape
    for a in (key_cache8, value_cache8, k_scales, v_scales):
        assert a.flags["C_CONTIGUOUS"]
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    code = dtype_code(k.dtype) if code is None else code
    _check(lib().oracle_append_int8(_ptr(k), _ptr(v), code, _ptr(key_cache8), _ptr(value_cache8),
                                    _ptr(k_scales), _ptr(v_scales), _ptr(sm), T, H, d, bs, N),
           "oracle_append_int8")


def quantize_int4(src_cache, code=None):
    """Return (packed 4-bit cache uint8 [N][H_kv][bs][d/2], fp32 scales [N][H_kv])
    for a [N][H_kv][bs][d] cache."""
    N, H, bs, d = src_cache.shape
    src = np.ascontiguousarray(src_cache)
    code = dtype_code(src.dtype) if code is None else code
    dst = np.zeros((N, H, bs, d // 2), dtype=np.uint8)
    scales = np.empty((N, H), dtype=np.float32)
    _check(lib().oracle_quantize_int4(_ptr(src), code, _ptr(dst), _ptr(scales), N, H, d, bs),
           "oracle_quantize_int4")
    return dst, scales


def _q64(q):
    if q.dtype == np.uint16:  # bf16 bit patterns
        return (q.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(q, dtype=np.float64)


def decode(q, key_cache, value_cache, block_tables, seq_lens, scale, k_scales=None,
           v_scales=None, kv_code=None, bh=None, nthreads=None):
    """fp64 decode output [B][H_q][d].  ``bh``: optional int array [n][2] of
    (sequence, query head) rows to compute (the others are left NaN)."""
    q64 = _q64(q)
    B, Hq, d = q64.shape
    N, Hkv, bs, d2 = key_cache.shape
    code = dtype_code(key_cache.dtype) if kv_code is None else kv_code
    assert d == (2 * d2 if code == I4 else d2)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.full((B, Hq, d), np.nan, dtype=np.float64)
    bhl = None if bh is None else np.ascontiguousarray(bh, dtype=np.int32).reshape(-1, 2)
    nt = nthreads_default() if nthreads is None else nthreads
    _check(lib().oracle_decode(_ptr(out), _ptr(q64), _ptr(key_cache), _ptr(value_cache), code,
                               _ptr(k_scales), _ptr(v_scales), _ptr(bt), _ptr(sl), B, Hq, Hkv, d,
                               bs, bt.shape[1] if bt.ndim == 2 else 0, N, float(scale), _ptr(bhl),
                               0 if bhl is None else bhl.shape[0], nt),
           "oracle_decode")
    return out


def decode_multi(q, key_cache, value_cache, block_tables, seq_lens, scale, k_scales=None,
                 v_scales=None, kv_code=None, nthreads=None):
    """fp64 multi-query decode output [B][Q][H_q][d] for q [B][Q][H_q][d]: query
    token i of sequence b attends to its first seq_lens[b] - Q + i + 1 tokens."""
    q64 = _q64(q)
    B, Q, Hq, d = q64.shape
    N, Hkv, bs, d2 = key_cache.shape
    code = dtype_code(key_cache.dtype) if kv_code is None else kv_code
    assert d == (2 * d2 if code == I4 else d2)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    out = np.full((B, Q, Hq, d), np.nan, dtype=np.float64)
    nt = nthreads_default() if nthreads is None else nthreads
    _check(lib().oracle_decode_multi(_ptr(out), _ptr(q64), _ptr(key_cache), _ptr(value_cache), code,
                                     _ptr(k_scales), _ptr(v_scales), _ptr(bt), _ptr(sl), B, Q, Hq, Hkv,
                                     d, bs, bt.shape[1] if bt.ndim == 2 else 0, N, float(scale), nt),
           "oracle_decode_multi")
    return out


def decode_partials(q, key_cache, value_cache, block_tables, seq_lens, scale, partition_size,
                    max_parts, k_scales=None, v_scales=None, kv_code=None, nthreads=None):
    """Per-partition normalised outputs [B][H_q][P][d] and lse [B][H_q][P] (natural log)."""
    q64 = _q64(q)
    B, Hq, d = q64.shape
    N, Hkv, bs, _ = key_cache.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    code = dtype_code(key_cache.dtype) if kv_code is None else kv_code
    o = np.empty((B, Hq, max_parts, d), dtype=np.float64)
    lse = np.empty((B, Hq, max_parts), dtype=np.float64)
    nt = nthreads_default() if nthreads is None else nthreads
    _check(lib().oracle_decode_partials(_ptr(o), _ptr(lse), _ptr(q64), _ptr(key_cache),
                                        _ptr(value_cache), code, _ptr(k_scales), _ptr(v_scales),
                                        _ptr(bt), _ptr(sl), B, Hq, Hkv, d, bs, bt.shape[1], N,
                                        float(scale), int(partition_size), int(max_parts), nt),
           "oracle_decode_partials")
    return o, lse


def merge(o_part, lse_part):
    """Log-sum-exp merge of [..][P][d] partials with [..][P] lse -> [..][d]."""
    o = np.ascontiguousarray(o_part, dtype=np.float64)
    lse = np.ascontiguousarray(lse_part, dtype=np.float64)
    P, d = o.shape[-2:]
    rows = int(np.prod(o.shape[:-2]))
    out = np.empty(o.shape[:-2] + (d,), dtype=np.float64)
    _check(lib().oracle_merge(_ptr(out), _ptr(o), _ptr(lse), rows, P, d), "oracle_merge")
    return out


def kv_bytes_per_token(num_layers, num_kv_heads, head_dim, elem_size) -> int:
    return int(lib().oracle_kv_bytes_per_token(num_layers, num_kv_heads, head_dim, elem_size))
