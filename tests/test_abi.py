"""The C-ABI library on the host (no GPU needed): it loads, exports every
function include/pa.h declares, and rejects invalid arguments with the
documented status codes before any launch."""
import ctypes
import os
import re

import pytest

from paged_kv_cache_395_b200 import pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(pa_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_expected_entry_points():
    names = header_functions()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_block_copy", "pa_decode_workspace_size"):
        assert n in names
    assert set(names) == set(pa.EXPORTED)


@pytest.mark.parametrize("name", header_functions())
def test_library_exports(name):
    lib = ctypes.CDLL(pa.LIB_PATH)
    assert getattr(lib, name) is not None


def test_status_strings_and_version():
    assert pa.lib.pa_status_string(0) == b"ok"
    for s in range(-7, 0):
        assert pa.lib.pa_status_string(s) != b"unknown status"
    assert pa.version() >= 100


def params(**kw):
    p = pa.PaDecodeParams()
    base = dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                max_blocks_per_seq=4, num_blocks=8, max_seq_len=64, q_dtype=pa.PA_F16,
                kv_dtype=pa.PA_F16, partition_size=0, algo=0)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), pa.PA_ERR_UNSUPPORTED),
    (dict(head_dim=0), pa.PA_ERR_SHAPE),
    (dict(block_size=32), pa.PA_ERR_UNSUPPORTED),
    (dict(num_q_heads=6, num_kv_heads=4), pa.PA_ERR_SHAPE),
    (dict(num_q_heads=6, num_kv_heads=2, algo=pa.PA_ALGO_SIMT), pa.PA_ERR_UNSUPPORTED),  # G = 3
    (dict(num_q_heads=6, num_kv_heads=2, q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),
    (dict(query_len=2, algo=pa.PA_ALGO_SIMT), pa.PA_ERR_UNSUPPORTED),  # several new tokens: TC only
    (dict(query_len=-1), pa.PA_ERR_SHAPE),
    (dict(query_len=129, num_q_heads=8, num_kv_heads=2), pa.PA_ERR_UNSUPPORTED),  # 516 pairs per KV head
    (dict(q_dtype=pa.PA_F32, kv_dtype=pa.PA_F16), pa.PA_ERR_DTYPE),
    (dict(q_dtype=pa.PA_I8, kv_dtype=pa.PA_I8), pa.PA_ERR_DTYPE),
    (dict(q_dtype=pa.PA_BF16, kv_dtype=pa.PA_I4), pa.PA_ERR_DTYPE),   # 4-bit caches take fp16 q
    (dict(kv_dtype=pa.PA_I4, algo=pa.PA_ALGO_SIMT), pa.PA_ERR_UNSUPPORTED),
    (dict(kv_dtype=pa.PA_I4, head_dim=64, algo=pa.PA_ALGO_TENSOR), pa.PA_ERR_UNSUPPORTED),
    (dict(q_dtype=9), pa.PA_ERR_DTYPE),
    (dict(partition_size=24), pa.PA_ERR_SHAPE),
    (dict(partition_size=-2), pa.PA_ERR_SHAPE),
    (dict(flags=4), pa.PA_ERR_UNSUPPORTED),          # unknown flag bit
    (dict(num_q_heads=1024, num_kv_heads=1), pa.PA_ERR_UNSUPPORTED),  # G = 1024
    (dict(head_dim=256, q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32), pa.PA_ERR_UNSUPPORTED),
    (dict(num_seqs=-1), pa.PA_ERR_SHAPE),
    (dict(algo=7), pa.PA_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_params(kw, status):
    p = params(**kw)
    rc = pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p), None)
    assert rc == status
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) == 0


def test_decode_null_and_workspace_checks():
    p = params()
    rc = pa.lib.pa_decode(None, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p), None)
    assert rc == pa.PA_ERR_NULL
    rc = pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), None, None)
    assert rc == pa.PA_ERR_NULL
    p = params(kv_dtype=pa.PA_I8)  # int8 without scales
    rc = pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p), None)
    assert rc == pa.PA_ERR_NULL
    p = params(partition_size=16, algo=pa.PA_ALGO_SIMT)  # split-K without a workspace
    need = pa.lib.pa_decode_workspace_size(ctypes.byref(p))
    # CUDA-core family: 2 seqs x 8 heads x 4 partitions x 128 floats and their 64
    # lse floats, each region rounded up to 256 B
    assert need == 2 * 8 * 4 * 128 * 4 + 256
    rc = pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p), None)
    assert rc == pa.PA_ERR_WORKSPACE
    p.workspace, p.workspace_bytes = 0x1000, need - 1
    rc = pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p), None)
    assert rc == pa.PA_ERR_WORKSPACE
    # tensor-core family: 2 x 2 rows x 4 blocks = 16 blocks in chunks of 1 block ->
    # 32 partial slots of 4 heads x (128 + 1) floats
    p = params(partition_size=16, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) == 32 * 4 * 128 * 4 + 512
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(params(partition_size=0, algo=pa.PA_ALGO_TENSOR))) == 0
    # auto schedule on the tensor-core family: at most 2048 chunks (one per warp),
    # two partial slots each
    p = params(partition_size=-1, algo=pa.PA_ALGO_TENSOR, num_seqs=64, max_blocks_per_seq=264,
               max_seq_len=4224)
    slots = 2 * 2048
    up = lambda x: (x + 255) // 256 * 256
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) == \
        up(slots * 4 * 128 * 4) + up(slots * 4 * 4)
    # the tensor-core family needs fp16/bf16 q and cache
    p = params(q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p),
                            None) == pa.PA_ERR_UNSUPPORTED
    p = params()
    rc = pa.lib.pa_decode(FAKE, FAKE, ctypes.c_void_p(0x1008), FAKE, FAKE, FAKE, ctypes.c_float(0.1),
                          ctypes.byref(p), None)
    assert rc == pa.PA_ERR_ALIGN
    # a partition as long as the longest sequence needs no workspace (CUDA-core family)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(params(partition_size=64, algo=pa.PA_ALGO_SIMT))) == 0
    # empty batch is a no-op
    assert pa.lib.pa_decode(None, None, None, None, None, None, ctypes.c_float(0.1),
                            ctypes.byref(params(num_seqs=0)), None) == pa.PA_OK


def test_cache_ops_reject_bad_args():
    L = pa.lib
    assert L.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 32, 8, pa.PA_F16, 128, 128, None) == pa.PA_ERR_UNSUPPORTED
    assert L.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, pa.PA_I8, 128, 128, None) == pa.PA_ERR_UNSUPPORTED
    assert L.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 11, 128, 128, None) == pa.PA_ERR_DTYPE
    assert L.pa_reshape_and_cache(None, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, pa.PA_F16, 128, 128, None) == pa.PA_ERR_NULL
    assert L.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, pa.PA_F16, 100, 128, None) == pa.PA_ERR_SHAPE
    assert L.pa_reshape_and_cache(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 2, 64, 16, 8, pa.PA_F16, 128, 128, None) == pa.PA_ERR_SHAPE
    assert L.pa_reshape_and_cache(None, None, None, None, None, 0, 2, 64, 16, 8, pa.PA_F16, 128, 128, None) == pa.PA_OK
    assert L.pa_block_copy(FAKE, FAKE, None, None, FAKE, 1, 2, 64, 8, 8, pa.PA_F16, None) == pa.PA_ERR_UNSUPPORTED
    assert L.pa_block_copy(FAKE, None, None, None, FAKE, 1, 2, 64, 16, 8, pa.PA_F16, None) == pa.PA_ERR_NULL
    assert L.pa_block_copy(FAKE, FAKE, FAKE, None, FAKE, 1, 2, 64, 16, 8, pa.PA_I8, None) == pa.PA_ERR_NULL
    assert L.pa_block_copy(None, None, None, None, None, 0, 2, 64, 16, 8, pa.PA_F16, None) == pa.PA_OK
    assert L.pa_quantize_int8(FAKE, pa.PA_I8, FAKE, FAKE, 4, 2, 64, 16, None) == pa.PA_ERR_DTYPE
    assert L.pa_quantize_int8(FAKE, pa.PA_F16, None, FAKE, 4, 2, 64, 16, None) == pa.PA_ERR_NULL
    assert L.pa_quantize_int8(FAKE, pa.PA_F16, FAKE, FAKE, 4, 2, 64, 8, None) == pa.PA_ERR_UNSUPPORTED
    assert L.pa_get_error_flags(None, 0, None) == pa.PA_ERR_NULL


def test_product_path_does_not_touch_oracle():
    """The package never imports the oracle (it is test infrastructure)."""
    pkg = os.path.join(ROOT, "paged_kv_cache_395_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), f
                assert not re.search(r"#include\s*[<\"][^>\"]*oracle", src), f
                assert "liboracle" not in src and "pa_oracle" not in src, f


def test_large_groups_and_head_dim_256_are_planned():
    """G = 16, 32, 64 run as 8-head groups: the workspace of a G = 32, H_kv = 1
    decode equals that of G = 8, H_kv = 4 (same query heads, same rows); head_dim
    256 is accepted on both families."""
    big = params(num_q_heads=32, num_kv_heads=1, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    same = params(num_q_heads=32, num_kv_heads=4, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    n = pa.lib.pa_decode_workspace_size(ctypes.byref(big))
    assert n > 0 and n == pa.lib.pa_decode_workspace_size(ctypes.byref(same))
    for g in (16, 64):
        p = params(num_q_heads=g, num_kv_heads=1, partition_size=16)
        assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0
    p = params(head_dim=256, partition_size=16, algo=pa.PA_ALGO_SIMT)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0
    # the tensor-core family takes fp16/bf16 and int8 head_dim 256 too (not 4-bit caches)
    p = params(head_dim=256, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0
    p = params(head_dim=256, kv_dtype=pa.PA_I8, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0
    p = params(head_dim=256, kv_dtype=pa.PA_I4, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.1), ctypes.byref(p),
                            None) == pa.PA_ERR_UNSUPPORTED


def test_multi_query_and_padded_groups_are_planned():
    """Q new tokens per sequence and group sizes that are not powers of two run
    on the tensor-core family: Q x G (query token, head) pairs per KV head fill
    rows of 8 columns (padded up to a power of two below 8)."""
    for kw in (dict(query_len=2), dict(query_len=3, num_q_heads=8, num_kv_heads=8),
               dict(num_q_heads=6, num_kv_heads=2), dict(num_q_heads=48, num_kv_heads=2),
               dict(query_len=4, num_q_heads=32, num_kv_heads=8)):
        p = params(partition_size=16, algo=pa.PA_ALGO_TENSOR, **kw)
        assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0, kw
    # G = 24 is three full 8-head groups: the CUDA-core family takes it too
    p = params(num_q_heads=48, num_kv_heads=2, partition_size=16, algo=pa.PA_ALGO_SIMT)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) > 0
    # Q = 2 at G = 4 fills exactly the 8 columns of one row per KV head: same
    # workspace as a G = 8 single-token decode over the same KV heads
    a = params(query_len=2, num_q_heads=8, num_kv_heads=2, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    b = params(num_q_heads=16, num_kv_heads=2, partition_size=16, algo=pa.PA_ALGO_TENSOR)
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(a)) == pa.lib.pa_decode_workspace_size(ctypes.byref(b))


def test_decode_algo_reports_the_family():
    """pa_decode_algo returns the family pa_decode would run (host only, q not read)."""
    q16, q8 = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)
    algo = lambda p, q=q16: pa.lib.pa_decode_algo(ctypes.byref(p), q)  # noqa: E731
    assert algo(params()) == pa.PA_ALGO_TENSOR
    assert algo(params(algo=pa.PA_ALGO_SIMT)) == pa.PA_ALGO_SIMT
    assert algo(params(q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32)) == pa.PA_ALGO_SIMT
    assert algo(params(head_dim=256)) == pa.PA_ALGO_TENSOR
    assert algo(params(head_dim=256, q_dtype=pa.PA_BF16, kv_dtype=pa.PA_BF16)) == pa.PA_ALGO_TENSOR
    assert algo(params(head_dim=256, kv_dtype=pa.PA_I8)) == pa.PA_ALGO_TENSOR
    assert algo(params(head_dim=256, kv_dtype=pa.PA_I8, q_dtype=pa.PA_BF16)) == pa.PA_ALGO_SIMT
    assert algo(params(kv_dtype=pa.PA_I8, q_dtype=pa.PA_BF16)) == pa.PA_ALGO_SIMT
    assert algo(params(kv_dtype=pa.PA_I8)) == pa.PA_ALGO_TENSOR
    # a q that is not 16-byte aligned goes to the CUDA-core family, or is refused
    assert algo(params(), q8) == pa.PA_ALGO_SIMT
    assert algo(params(algo=pa.PA_ALGO_TENSOR), q8) == pa.PA_ERR_ALIGN
    assert algo(params(head_dim=96)) == pa.PA_ERR_UNSUPPORTED
    assert algo(params(flags=pa.PA_DECODE_OUT_F32 | pa.PA_DECODE_INPUTS_READY)) == pa.PA_ALGO_TENSOR


def test_large_groups_plan_the_cooperative_mode():
    """Groups of 16, 32 or 64 fp16/bf16 query heads per KV head at head_dim 64/128
    split in the cooperative mode: one partial slot holds all G columns of a cache
    row, chunks are cut over cache rows.  Its workspace: 2 slots per chunk of the
    cache-row stream (at most 2048 chunks) x G x (d + 1) floats."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for hq, hkv in ((16, 1), (32, 1), (64, 1), (32, 2)):
        p = params(num_seqs=4, num_q_heads=hq, num_kv_heads=hkv, max_blocks_per_seq=64, max_seq_len=1024,
                   partition_size=-1, algo=pa.PA_ALGO_TENSOR)
        chunks = min(4 * hkv * 64, 2048)
        assert pa.lib.pa_decode_workspace_size(ctypes.byref(p)) == \
            up(2 * chunks * (hq // hkv) * 128 * 4) + up(2 * chunks * (hq // hkv) * 4), (hq, hkv)


def test_stall_selftest_rejects_bad_args():
    """The failure-path self-test validates like pa_decode, needs a stage index
    and a positive limit, and runs only on the tensor-core family."""
    L = pa.lib
    p = params()
    f = ctypes.c_float(0.1)
    assert L.pa_decode_stall_selftest(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f, ctypes.byref(p), -1, 1000, None) \
        == pa.PA_ERR_SHAPE
    assert L.pa_decode_stall_selftest(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f, ctypes.byref(p), 0, 0, None) \
        == pa.PA_ERR_SHAPE
    p = params(head_dim=96)
    assert L.pa_decode_stall_selftest(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f, ctypes.byref(p), 0, 1000, None) \
        == pa.PA_ERR_UNSUPPORTED
    p = params(algo=pa.PA_ALGO_SIMT)
    assert L.pa_decode_stall_selftest(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, f, ctypes.byref(p), 0, 1000, None) \
        == pa.PA_ERR_UNSUPPORTED


def test_decode_append_reports_when_it_fuses():
    """pa_decode_append runs as one kernel on the tensor-core family's per-warp
    decode of single-token fp16/bf16 rows with 16-byte aligned q and new-token
    rows; otherwise as pa_reshape_and_cache then pa_decode (0); arguments it would
    reject give their status.  No pointer is read."""
    A = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced
    def fused(p, kn=A, vn=A, ks=None, vs=None):
        row = p.num_kv_heads * p.head_dim
        return pa.lib.pa_decode_append_fused(ctypes.byref(p), A, kn, vn, row if ks is None else ks,
                                             row if vs is None else vs)
    assert fused(params()) == 1
    assert fused(params(q_dtype=pa.PA_BF16, kv_dtype=pa.PA_BF16, partition_size=-1)) == 1
    assert fused(params(head_dim=256, partition_size=16)) == 1
    assert fused(params(head_dim=64, num_q_heads=2, num_kv_heads=2)) == 1
    assert fused(params(q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32)) == 0          # CUDA-core family
    assert fused(params(algo=pa.PA_ALGO_SIMT)) == 0
    assert fused(params(num_q_heads=32, num_kv_heads=1, partition_size=-1)) == 0  # cooperative mode
    assert fused(params(num_q_heads=32, num_kv_heads=1, partition_size=0)) == 1   # rows of 8 heads
    assert fused(params(), kn=ctypes.c_void_p(0x10008)) == 0                   # k_new not 16-byte aligned
    assert fused(params(), ks=2 * 128 + 4) == 0                                 # stride not 8 elements
    assert fused(params(query_len=2)) == pa.PA_ERR_UNSUPPORTED
    assert fused(params(kv_dtype=pa.PA_I8)) == pa.PA_ERR_DTYPE
    assert fused(params(), ks=100) == pa.PA_ERR_SHAPE
    assert fused(params(head_dim=96)) == pa.PA_ERR_UNSUPPORTED


def test_decode_append_rejects_before_any_launch():
    p = params()
    out = q = kc = vc = bt = sl = FAKE
    args = lambda slots, **kw: (out, q, FAKE, FAKE, slots, 256, 256, kc, vc, bt, sl,  # noqa: E731
                                ctypes.c_float(0.1), ctypes.byref(params(**kw)), None)
    assert pa.lib.pa_decode_append(*args(None)) == pa.PA_ERR_NULL
    assert pa.lib.pa_decode_append(*args(FAKE, query_len=3)) == pa.PA_ERR_UNSUPPORTED
    assert pa.lib.pa_decode_append(*args(FAKE, kv_dtype=pa.PA_I8, q_dtype=pa.PA_F16)) == pa.PA_ERR_DTYPE
    # split-K without a workspace
    assert pa.lib.pa_decode_append(*args(FAKE, partition_size=16)) == pa.PA_ERR_WORKSPACE
    del p


def test_tcgen05_is_planned_only_for_its_groups():
    """PA_ALGO_TCGEN05 takes groups of 32 or 64 fp16/bf16 query heads per KV head at
    head_dim 128 in split-K mode (the cooperative workspace layout), and nothing else."""
    algo = lambda p: pa.lib.pa_decode_algo(ctypes.byref(p), ctypes.c_void_p(0x1000))  # noqa: E731
    ok = dict(num_q_heads=32, num_kv_heads=1, partition_size=-1, algo=pa.PA_ALGO_TCGEN05)
    assert algo(params(**ok)) == pa.PA_ALGO_TCGEN05
    assert algo(params(**dict(ok, num_q_heads=64))) == pa.PA_ALGO_TCGEN05
    assert algo(params(**dict(ok, num_q_heads=64, num_kv_heads=2, q_dtype=pa.PA_BF16,
                              kv_dtype=pa.PA_BF16))) == pa.PA_ALGO_TCGEN05
    a = params(**ok)
    b = params(**dict(ok, algo=pa.PA_ALGO_TENSOR))
    assert pa.lib.pa_decode_workspace_size(ctypes.byref(a)) == pa.lib.pa_decode_workspace_size(ctypes.byref(b)) > 0
    for kw in (dict(num_q_heads=16), dict(num_q_heads=8), dict(head_dim=64), dict(partition_size=0),
               dict(q_dtype=pa.PA_F32, kv_dtype=pa.PA_F32), dict(kv_dtype=pa.PA_I8), dict(query_len=2),
               dict(num_seqs=4096, max_blocks_per_seq=1)):
        assert algo(params(**dict(ok, **kw))) == pa.PA_ERR_UNSUPPORTED, kw
    assert algo(params(algo=4)) == pa.PA_ERR_UNSUPPORTED


def test_decode_launches_reports_the_merge_kernel():
    """pa_decode_launches: one decode kernel, followed by a merge kernel when the
    call splits on the family it runs."""
    L = pa.lib
    aligned, unaligned = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1008)

    def n(q=aligned, **kw):
        return L.pa_decode_launches(ctypes.byref(params(**kw)), q)
    assert n(partition_size=0) == 1
    assert n(partition_size=-1, algo=pa.PA_ALGO_TENSOR) == 2
    assert n(partition_size=16, algo=pa.PA_ALGO_TENSOR) == 2
    assert n(partition_size=16, algo=pa.PA_ALGO_SIMT) == 2
    assert n(partition_size=0, algo=pa.PA_ALGO_SIMT) == 1
    # an unaligned q leaves the tensor-core family under PA_ALGO_AUTO (the CUDA-core
    # family's own plan: one partition of 64 tokens is one pass)
    assert n(q=unaligned, partition_size=16) == 2
    assert n(q=unaligned, partition_size=64) == 1
    assert n(partition_size=64) == 2
    assert n(q=unaligned, partition_size=16, algo=pa.PA_ALGO_TENSOR) == pa.PA_ERR_ALIGN
    # the cooperative mode
    big = dict(num_seqs=4, num_q_heads=32, num_kv_heads=1, max_blocks_per_seq=64, max_seq_len=1024)
    assert n(partition_size=-1, **big) == 2
    assert n(partition_size=0, **big) == 1
    assert n(partition_size=-1, algo=pa.PA_ALGO_TCGEN05, **big) == 2
    # invalid parameters: the status pa_decode would return
    assert n(head_dim=96) == pa.PA_ERR_UNSUPPORTED


def test_auto_picks_tcgen05_for_groups_of_64():
    """PA_ALGO_AUTO runs the tcgen05 kernel for split decodes of 64 fp16/bf16 query heads
    per KV head (where it measured faster), the cooperative mma.sync kernel for groups of
    16 and 32, and the tensor-core per-row kernel in one pass; PA_ALGO_TENSOR keeps the
    mma.sync family."""
    q = ctypes.c_void_p(0x1000)
    algo = lambda **kw: pa.lib.pa_decode_algo(ctypes.byref(params(**kw)), q)  # noqa: E731
    g64 = dict(num_seqs=4, num_q_heads=64, num_kv_heads=1, max_blocks_per_seq=64, max_seq_len=1024)
    assert algo(partition_size=-1, **g64) == pa.PA_ALGO_TCGEN05
    assert algo(partition_size=64, **dict(g64, q_dtype=pa.PA_BF16, kv_dtype=pa.PA_BF16)) == pa.PA_ALGO_TCGEN05
    assert algo(partition_size=-1, **dict(g64, num_q_heads=128, num_kv_heads=2)) == pa.PA_ALGO_TCGEN05
    assert algo(partition_size=0, **g64) == pa.PA_ALGO_TENSOR
    assert algo(partition_size=-1, algo=pa.PA_ALGO_TENSOR, **g64) == pa.PA_ALGO_TENSOR
    assert algo(partition_size=-1, **dict(g64, num_q_heads=32)) == pa.PA_ALGO_TENSOR
    assert algo(partition_size=-1, **dict(g64, num_q_heads=16)) == pa.PA_ALGO_TENSOR
    assert algo(partition_size=-1, **dict(g64, head_dim=64)) == pa.PA_ALGO_TENSOR
    assert algo(partition_size=-1, **dict(g64, query_len=2)) == pa.PA_ALGO_TENSOR
    # an unaligned q still leaves the tensor-core families
    assert pa.lib.pa_decode_algo(ctypes.byref(params(partition_size=-1, **g64)), ctypes.c_void_p(0x1008)) == \
        pa.PA_ALGO_SIMT
