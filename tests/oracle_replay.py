"""Replay a workload through the CPU oracle (tests only)."""
import numpy as np

import oracle
from paged_kv_cache_395_b200 import workloads as W

# NaN bit patterns used to fill never-written slots: a kernel that lets an
# unwritten slot reach an output turns it into NaN.
NAN_BITS = {"float16": 0x7E00, "bfloat16": 0x7FC0}


def make_pool(w, fill_nan=True):
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    dt = w.storage_dtype()
    if w.dtype == "bfloat16":
        kc = np.full(shape, NAN_BITS["bfloat16"] if fill_nan else 0, dtype=np.uint16)
    else:
        kc = np.full(shape, np.nan if fill_nan else 0, dtype=dt)
    return kc, kc.copy()


def code_of(w):
    return {"float32": oracle.F32, "float16": oracle.F16, "bfloat16": oracle.BF16}[w.dtype]


def apply(op, w, kc, vc, k_scales=None, v_scales=None):
    if isinstance(op, W.Reshape):
        oracle.reshape_and_cache(op.k, op.v, kc, vc, op.slot_mapping, code=code_of(w))
    elif isinstance(op, W.Copy):
        if op.pairs.size:
            oracle.block_copy(kc, vc, op.pairs, k_scales, v_scales, code=code_of(w))
    else:
        raise TypeError(op)


def replay(w, want=None, fill_nan=True, bh=None):
    """Run every op of ``w``; return ({step: fp64 decode output}, kc, vc).

    ``want(step)`` selects the steps whose decode is computed (default all);
    ``bh`` optionally restricts the computed (sequence, head) rows."""
    kc, vc = make_pool(w, fill_nan)
    for op in w.setup:
        apply(op, w, kc, vc)
    outs = {}
    for si, ops in enumerate(w.steps):
        for op in ops:
            if isinstance(op, W.Decode):
                if want is None or want(si):
                    if op.q.ndim == 4:  # query_len new tokens per sequence
                        outs[si] = oracle.decode_multi(op.q, kc, vc, op.block_tables, op.seq_lens,
                                                       w.scale, kv_code=code_of(w))
                    else:
                        outs[si] = oracle.decode(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale,
                                                 kv_code=code_of(w), bh=bh)
            else:
                apply(op, w, kc, vc)
    return outs, kc, vc


def to_f64(x, dtype):
    if dtype == "bfloat16":
        return (np.asarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)
