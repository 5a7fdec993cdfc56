"""Python binding of ``libpa.so`` (ctypes; argument marshalling only).

The names mirror the C ABI in ``include/pa.h``:

* ``pa_reshape_and_cache``, ``pa_decode``, ``pa_decode_append``,
  ``pa_decode_append_fused``, ``pa_decode_fixed_scratch``,
  ``pa_decode_stall_selftest``, ``pa_block_copy``, ``pa_quantize_int8``,
  ``pa_quantize_int4``, ``pa_append_int8``, ``pa_decode_workspace_size``,
  ``pa_decode_algo``, ``pa_get_error_flags`` take torch CUDA tensors (or raw device pointers via ``lib``), check device,
  dtype and contiguity, and call the library on
  ``torch.cuda.current_stream()``.  Every step of the computation runs in the
  library's kernels; there is no fallback of any kind.  If ``libpa.so`` is
  missing, importing this module raises ImportError.

PyTorch is used only for device memory, streams and ``data_ptr()``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK, PA_ERR_NULL, PA_ERR_SHAPE, PA_ERR_DTYPE = 0, -1, -2, -3
PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA, PA_ERR_ALIGN = -4, -5, -6, -7
PA_F32, PA_F16, PA_BF16, PA_I8, PA_I4 = 0, 1, 2, 3, 4
PA_ALGO_AUTO, PA_ALGO_SIMT, PA_ALGO_TENSOR, PA_ALGO_TCGEN05 = 0, 1, 2, 3
PA_EFLAG_BAD_BLOCK, PA_EFLAG_BAD_SLOT, PA_EFLAG_BAD_PAIR, PA_EFLAG_WAIT_TIMEOUT = 1, 2, 4, 8
PA_EFLAG_APPEND_SLOT = 16
PA_DECODE_INPUTS_READY, PA_DECODE_OUT_F32 = 1, 2
PA_APPEND_OVERLAP_PREVIOUS = 1
BLOCK_SIZE = 16

# a uint8 cache tensor [N][H_kv][16][d/2] holds 4-bit values, two per byte
_TORCH_DTYPE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
                torch.int8: PA_I8, torch.uint8: PA_I4}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m paged_kv_cache_395_b200.build` (no fallback exists)")


class PaDecodeParams(ctypes.Structure):
    """Mirror of ``pa_decode_params``."""
    _fields_ = [
        ("num_seqs", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int64),
        ("max_seq_len", ctypes.c_int),
        ("q_dtype", ctypes.c_int),
        ("kv_dtype", ctypes.c_int),
        ("k_scales", ctypes.c_void_p),
        ("v_scales", ctypes.c_void_p),
        ("partition_size", ctypes.c_int),
        ("algo", ctypes.c_int),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("flags", ctypes.c_int),
        ("query_len", ctypes.c_int),
    ]


def _load():
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    L.pa_reshape_and_cache.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, i64, i64, P]
    L.pa_reshape_and_cache_ex.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, i64, i64, i32, P]
    L.pa_decode.argtypes = [P, P, P, P, P, P, f32, ctypes.POINTER(PaDecodeParams), P]
    L.pa_decode_fixed_scratch.argtypes = [P, P, P, P, P, P, f32, ctypes.POINTER(PaDecodeParams), P]
    L.pa_decode_append.argtypes = [P, P, P, P, P, i64, i64, P, P, P, P, f32, ctypes.POINTER(PaDecodeParams), P]
    L.pa_decode_append_fused.argtypes = [ctypes.POINTER(PaDecodeParams), P, P, P, i64, i64]
    L.pa_decode_workspace_size.argtypes = [ctypes.POINTER(PaDecodeParams)]
    L.pa_decode_workspace_size.restype = ctypes.c_size_t
    L.pa_decode_algo.argtypes = [ctypes.POINTER(PaDecodeParams), P]
    L.pa_decode_launches.argtypes = [ctypes.POINTER(PaDecodeParams), P]
    L.pa_decode_stall_selftest.argtypes = [P, P, P, P, P, P, f32, ctypes.POINTER(PaDecodeParams), i32,
                                           ctypes.c_uint64, P]
    L.pa_block_copy.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, P]
    L.pa_quantize_int8.argtypes = [P, i32, P, P, i64, i32, i32, i32, P]
    L.pa_append_int8.argtypes = [P, P, i32, P, P, P, P, P, i64, i32, i32, i32, i64, i64, i64, P]
    L.pa_quantize_int4.argtypes = [P, i32, P, P, i64, i32, i32, i32, P]
    L.pa_get_error_flags.argtypes = [ctypes.POINTER(ctypes.c_uint), i32, P]
    L.pa_status_string.argtypes = [i32]
    L.pa_status_string.restype = ctypes.c_char_p
    L.pa_version.argtypes = []
    for n in ("pa_reshape_and_cache", "pa_reshape_and_cache_ex", "pa_append_int8", "pa_decode", "pa_decode_append",
              "pa_decode_append_fused", "pa_decode_fixed_scratch",
              "pa_decode_stall_selftest", "pa_decode_algo", "pa_decode_launches", "pa_block_copy",
              "pa_quantize_int8", "pa_quantize_int4", "pa_get_error_flags", "pa_version"):
        getattr(L, n).restype = i32
    return L


lib = _load()

# the C-ABI symbols include/pa.h declares
EXPORTED = ("pa_reshape_and_cache", "pa_reshape_and_cache_ex", "pa_append_int8", "pa_decode_workspace_size",
            "pa_decode_algo", "pa_decode_launches", "pa_decode", "pa_decode_append", "pa_decode_append_fused",
            "pa_decode_fixed_scratch", "pa_decode_stall_selftest", "pa_block_copy", "pa_quantize_int8",
            "pa_quantize_int4", "pa_get_error_flags", "pa_status_string", "pa_version")
FIXED_SCRATCH_BYTES = 32 << 20  # PA_FIXED_SCRATCH_BYTES


class PaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {lib.pa_status_string(status).decode()} ({status})")
        self.status = status


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PaError(status, what)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


def dtype_code(dt: torch.dtype) -> int:
    return _TORCH_DTYPE[dt]


def pa_reshape_and_cache(k, v, key_cache, value_cache, slot_mapping, stream=None, flags=0):
    """k, v [T][H_kv][d] (rows contiguous; token stride free) -> caches [N][H_kv][16][d].
    flags: 0 or PA_APPEND_OVERLAP_PREVIOUS (see include/pa.h)."""
    _dev(k, v, key_cache, value_cache, slot_mapping)
    T, H, d = k.shape
    N = key_cache.shape[0]
    if k.stride(2) != 1 or k.stride(1) != d or v.stride(2) != 1 or v.stride(1) != d:
        raise ValueError("k/v heads must be contiguous rows of head_dim elements")
    if slot_mapping.dtype != torch.int64 or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be contiguous int64")
    if not (key_cache.is_contiguous() and value_cache.is_contiguous()):
        raise ValueError("caches must be contiguous")
    _check(lib.pa_reshape_and_cache_ex(_ptr(k), _ptr(v), _ptr(key_cache), _ptr(value_cache),
                                       _ptr(slot_mapping), T, H, d, key_cache.shape[2], N,
                                       dtype_code(k.dtype), k.stride(0), v.stride(0), int(flags),
                                       _stream(stream)),
           "pa_reshape_and_cache")


def make_params(q, key_cache, block_tables, max_seq_len, k_scales=None, v_scales=None,
                partition_size=0, workspace=None, algo=PA_ALGO_AUTO, flags=0) -> PaDecodeParams:
    """q is [B][H_q][d], or [B][Q][H_q][d] for Q new tokens per sequence."""
    if q.dim() == 4:
        B, Q, Hq, d = q.shape
    else:
        (B, Hq, d), Q = q.shape, 1
    N, Hkv, bs, _ = key_cache.shape
    p = PaDecodeParams()
    p.num_seqs, p.num_q_heads, p.num_kv_heads, p.head_dim, p.block_size = B, Hq, Hkv, d, bs
    p.max_blocks_per_seq = block_tables.shape[1] if block_tables.dim() == 2 else 1
    p.num_blocks = N
    p.max_seq_len = int(max_seq_len)
    p.q_dtype = dtype_code(q.dtype)
    p.kv_dtype = dtype_code(key_cache.dtype)
    p.k_scales = None if k_scales is None else k_scales.data_ptr()
    p.v_scales = None if v_scales is None else v_scales.data_ptr()
    p.partition_size = int(partition_size)
    p.algo = int(algo)
    p.workspace = None if workspace is None else workspace.data_ptr()
    p.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    p.flags = int(flags)
    p.query_len = int(Q)
    return p


def pa_decode_algo(q, key_cache, block_tables, max_seq_len, partition_size=0, k_scales=None,
                   v_scales=None, algo=PA_ALGO_AUTO) -> int:
    """The kernel family pa_decode runs for these operands, as the library
    reports it: PA_ALGO_TENSOR, PA_ALGO_SIMT or PA_ALGO_TCGEN05."""
    p = make_params(q, key_cache, block_tables, max_seq_len, k_scales, v_scales, partition_size,
                    None, algo)
    r = int(lib.pa_decode_algo(ctypes.byref(p), _ptr(q)))
    _check(min(r, 0), "pa_decode_algo")
    return r


def pa_decode_launches(q, key_cache, block_tables, max_seq_len, partition_size=0, k_scales=None,
                       v_scales=None, algo=PA_ALGO_AUTO) -> int:
    """Kernel launches of one pa_decode call with these operands (1 or 2), as the
    library reports it."""
    p = make_params(q, key_cache, block_tables, max_seq_len, k_scales, v_scales, partition_size,
                    None, algo)
    r = int(lib.pa_decode_launches(ctypes.byref(p), _ptr(q)))
    _check(min(r, 0), "pa_decode_launches")
    return r


def pa_decode_workspace_size(q, key_cache, block_tables, max_seq_len, partition_size=0,
                             k_scales=None, v_scales=None, algo=PA_ALGO_AUTO) -> int:
    p = make_params(q, key_cache, block_tables, max_seq_len, k_scales, v_scales, partition_size,
                    None, algo)
    return int(lib.pa_decode_workspace_size(ctypes.byref(p)))


def alloc_workspace(nbytes: int, device) -> torch.Tensor | None:
    """Split-K workspace (left uninitialised: pa_decode needs none)."""
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _out_flag(out, q) -> int:
    """out matches q in shape, and in dtype or is fp32 (PA_DECODE_OUT_F32)."""
    if out.shape != q.shape or out.dtype not in (q.dtype, torch.float32):
        raise ValueError("out must match q in shape, and in dtype or be float32")
    return PA_DECODE_OUT_F32 if out.dtype != q.dtype else 0


def pa_decode(out, q, key_cache, value_cache, block_tables, seq_lens, scale, max_seq_len,
              k_scales=None, v_scales=None, partition_size=0, workspace=None,
              algo=PA_ALGO_AUTO, stream=None, params=None, flags=0):
    """out, q [B][H_q][d] (or [B][Q][H_q][d]: Q new tokens per sequence, causal
    among them); caches [N][H_kv][16][d]; block_tables int32 [B][M]; seq_lens int32
    [B] (including the new tokens).  flags: 0 or PA_DECODE_INPUTS_READY (see
    include/pa.h).  A float32 out of an fp16/bf16 q receives the fp32 result
    before its rounding (PA_DECODE_OUT_F32 is added)."""
    _dev(out, q, key_cache, value_cache, block_tables, seq_lens, k_scales, v_scales, workspace)
    for t, n in ((out, "out"), (q, "q"), (key_cache, "key_cache"), (value_cache, "value_cache"),
                 (block_tables, "block_tables"), (seq_lens, "seq_lens")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    flags |= _out_flag(out, q)
    p = params if params is not None else make_params(
        q, key_cache, block_tables, max_seq_len, k_scales, v_scales, partition_size, workspace, algo,
        flags)
    _check(lib.pa_decode(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache),
                         _ptr(block_tables), _ptr(seq_lens), ctypes.c_float(scale),
                         ctypes.byref(p), _stream(stream)), "pa_decode")


def _new_rows(k_new, v_new, slot_mapping, key_cache):
    """k_new / v_new [B][H_kv][d] (token stride free, heads contiguous rows), int64 slots [B]."""
    _, H, _, d = key_cache.shape
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        if t.dim() != 3 or t.shape[1:] != (H, d) or t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{n} must be [B][H_kv][d] with contiguous head rows")
        if t.dtype != key_cache.dtype:
            raise ValueError(f"{n} must have the cache's dtype")
    if slot_mapping.dtype != torch.int64 or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be contiguous int64")


def pa_decode_append(out, q, k_new, v_new, slot_mapping, key_cache, value_cache, block_tables, seq_lens,
                     scale, max_seq_len, partition_size=0, workspace=None, algo=PA_ALGO_AUTO, stream=None,
                     flags=0):
    """pa_reshape_and_cache of one new token per sequence (k_new / v_new row b,
    slot_mapping[b]) then pa_decode, as one kernel where pa_decode_append_fused
    says so (include/pa.h).  seq_lens count the new token."""
    _dev(out, q, k_new, v_new, slot_mapping, key_cache, value_cache, block_tables, seq_lens, workspace)
    for t, n in ((out, "out"), (q, "q"), (key_cache, "key_cache"), (value_cache, "value_cache"),
                 (block_tables, "block_tables"), (seq_lens, "seq_lens")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    _new_rows(k_new, v_new, slot_mapping, key_cache)
    if k_new.shape[0] != q.shape[0] or slot_mapping.numel() != q.shape[0]:
        raise ValueError("one new token per sequence")
    flags |= _out_flag(out, q)
    p = make_params(q, key_cache, block_tables, max_seq_len, None, None, partition_size, workspace, algo,
                    flags)
    _check(lib.pa_decode_append(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
                                k_new.stride(0), v_new.stride(0), _ptr(key_cache), _ptr(value_cache),
                                _ptr(block_tables), _ptr(seq_lens), ctypes.c_float(scale), ctypes.byref(p),
                                _stream(stream)), "pa_decode_append")


def pa_decode_append_fused(q, k_new, v_new, key_cache, block_tables, max_seq_len, partition_size=0,
                           algo=PA_ALGO_AUTO) -> bool:
    """Whether pa_decode_append with these operands runs as one kernel."""
    p = make_params(q, key_cache, block_tables, max_seq_len, None, None, partition_size, None, algo)
    r = int(lib.pa_decode_append_fused(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new),
                                       k_new.stride(0), v_new.stride(0)))
    _check(min(r, 0), "pa_decode_append_fused")
    return r == 1


def pa_decode_fixed_scratch(out, q, key_cache, value_cache, block_tables, seq_lens, scale,
                            max_seq_len, k_scales=None, v_scales=None, partition_size=-1,
                            algo=PA_ALGO_AUTO, stream=None):
    """pa_decode for callers that cannot allocate a workspace: the split-K
    scratch is the fixed area compiled into the library (FIXED_SCRATCH_BYTES per
    device).  Calls on one device must not overlap; the first call on a device
    looks up the area's address and should come before any stream capture."""
    _dev(out, q, key_cache, value_cache, block_tables, seq_lens, k_scales, v_scales)
    for t, n in ((out, "out"), (q, "q"), (key_cache, "key_cache"), (value_cache, "value_cache"),
                 (block_tables, "block_tables"), (seq_lens, "seq_lens")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    p = make_params(q, key_cache, block_tables, max_seq_len, k_scales, v_scales, partition_size,
                    None, algo, _out_flag(out, q))
    _check(lib.pa_decode_fixed_scratch(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache),
                                       _ptr(block_tables), _ptr(seq_lens), ctypes.c_float(scale),
                                       ctypes.byref(p), _stream(stream)), "pa_decode_fixed_scratch")


def pa_decode_stall_selftest(out, q, key_cache, value_cache, block_tables, seq_lens, scale, max_seq_len,
                             stall_at, limit_ns, partition_size=-1, workspace=None, stream=None,
                             algo=PA_ALGO_TENSOR):
    """pa_decode on the tensor-core family (algo PA_ALGO_TENSOR or PA_ALGO_TCGEN05)
    with the failure path exercised: the first worker leaves its stall_at-th copy
    unissued, so its bounded wait runs out after limit_ns (see include/pa.h).
    Returns after the launch; the error word then holds PA_EFLAG_WAIT_TIMEOUT."""
    _dev(out, q, key_cache, value_cache, block_tables, seq_lens, workspace)
    p = make_params(q, key_cache, block_tables, max_seq_len, None, None, partition_size, workspace,
                    algo, _out_flag(out, q))
    _check(lib.pa_decode_stall_selftest(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache),
                                        _ptr(block_tables), _ptr(seq_lens), ctypes.c_float(scale),
                                        ctypes.byref(p), int(stall_at), int(limit_ns), _stream(stream)),
           "pa_decode_stall_selftest")


def pa_block_copy(key_cache, value_cache, pairs, k_scales=None, v_scales=None, stream=None):
    """pairs int64 [n][2] (src, dst) on the device.  A uint8 (4-bit) cache
    [N][H_kv][16][d/2] is copied as such."""
    _dev(key_cache, value_cache, pairs, k_scales, v_scales)
    N, H, bs, d = key_cache.shape
    if key_cache.dtype == torch.uint8:
        d *= 2  # head_dim of a 4-bit cache
    if pairs.dtype != torch.int64 or not pairs.is_contiguous():
        raise ValueError("pairs must be contiguous int64")
    n = pairs.numel() // 2
    _check(lib.pa_block_copy(_ptr(key_cache), _ptr(value_cache), _ptr(k_scales), _ptr(v_scales),
                             _ptr(pairs), n, H, d, bs, N, dtype_code(key_cache.dtype),
                             _stream(stream)), "pa_block_copy")


def pa_quantize_int8(src_cache, dst_cache, scales, stream=None):
    """src [N][H_kv][16][d] fp32/fp16/bf16 -> dst int8 (same shape), scales fp32 [N][H_kv]."""
    _dev(src_cache, dst_cache, scales)
    N, H, bs, d = src_cache.shape
    if dst_cache.dtype != torch.int8 or scales.dtype != torch.float32:
        raise ValueError("dst must be int8 and scales float32")
    _check(lib.pa_quantize_int8(_ptr(src_cache), dtype_code(src_cache.dtype), _ptr(dst_cache),
                                _ptr(scales), N, H, d, bs, _stream(stream)), "pa_quantize_int8")


def pa_append_int8(k, v, key_cache, value_cache, k_scales, v_scales, slot_mapping, stream=None):
    """Append tokens k, v ([T][H_kv][d] fp32/fp16/bf16, rows contiguous) into int8
    caches [N][H_kv][16][d] with fp32 scales [N][H_kv], raising a tile's scale and
    re-rounding its other codes when a token needs it.  The tokens of one call must
    fall in distinct blocks (see include/pa.h)."""
    _dev(k, v, key_cache, value_cache, k_scales, v_scales, slot_mapping)
    T, H, d = k.shape
    N = key_cache.shape[0]
    if k.stride(2) != 1 or k.stride(1) != d or v.stride(2) != 1 or v.stride(1) != d or v.shape != k.shape:
        raise ValueError("k/v heads must be contiguous rows of head_dim elements")
    if k.dtype != v.dtype:
        raise ValueError("k and v must share a dtype")
    if key_cache.dtype != torch.int8 or value_cache.dtype != torch.int8:
        raise ValueError("caches must be int8")
    if k_scales.dtype != torch.float32 or v_scales.dtype != torch.float32:
        raise ValueError("scales must be float32")
    if tuple(key_cache.shape) != (N, H, 16, d) or value_cache.shape != key_cache.shape or \
            tuple(k_scales.shape) != (N, H) or v_scales.shape != k_scales.shape:
        raise ValueError("caches must be [N][H_kv][16][d] and scales [N][H_kv]")
    for t in (key_cache, value_cache, k_scales, v_scales):
        if not t.is_contiguous():
            raise ValueError("caches and scales must be contiguous")
    if slot_mapping.dtype != torch.int64 or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be contiguous int64")
    _check(lib.pa_append_int8(_ptr(k), _ptr(v), dtype_code(k.dtype), _ptr(key_cache), _ptr(value_cache),
                              _ptr(k_scales), _ptr(v_scales), _ptr(slot_mapping), T, H, d, 16, N,
                              k.stride(0), v.stride(0), _stream(stream)), "pa_append_int8")


def pa_quantize_int4(src_cache, dst_cache, scales, stream=None):
    """src [N][H_kv][16][d] fp32/fp16/bf16 -> dst uint8 [N][H_kv][16][d/2] (4-bit
    values q + 8, element 2k in the low half of byte k), scales fp32 [N][H_kv]."""
    _dev(src_cache, dst_cache, scales)
    N, H, bs, d = src_cache.shape
    if dst_cache.dtype != torch.uint8 or tuple(dst_cache.shape) != (N, H, bs, d // 2):
        raise ValueError("dst must be uint8 [N][H_kv][16][d/2]")
    if scales.dtype != torch.float32:
        raise ValueError("scales must be float32")
    _check(lib.pa_quantize_int4(_ptr(src_cache), dtype_code(src_cache.dtype), _ptr(dst_cache),
                                _ptr(scales), N, H, d, bs, _stream(stream)), "pa_quantize_int4")


def pa_get_error_flags(reset: bool = True, stream=None) -> int:
    f = ctypes.c_uint(0)
    _check(lib.pa_get_error_flags(ctypes.byref(f), int(reset), _stream(stream)),
           "pa_get_error_flags")
    return int(f.value)


def version() -> int:
    return int(lib.pa_version())
