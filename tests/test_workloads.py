"""The synthetic workload recipes hold the shapes the configurations name (heads,
head_dim, dtype, batch, lengths, pool), draw the same arrays from the same seed,
and keep the block tables consistent with the pool.  Host only."""
import numpy as np
import pytest

from paged_kv_cache_395_b200 import workloads as W


_CACHE = {}


def _make(name):
    """Each recipe built once per test session (the large ones take seconds)."""
    if name not in _CACHE:
        _CACHE[name] = getattr(W, name)()
    return _CACHE[name]


def _decode(w, step=0):
    return [op for op in w.steps[step] if isinstance(op, W.Decode)][0]


@pytest.mark.parametrize("name,hq,hkv,d,dtype,batch,lmin,lmax", [
    ("tiny", 4, 2, 64, "float32", 3, 5, 33),
    ("gqa_b8", 32, 8, 128, "float16", 8, 1024, 1024),
    ("long", 32, 8, 128, "float16", 16, 8192, 8192),
    ("mqa", 32, 1, 128, "float16", 128, 4096, 4096),
    ("d256", 16, 8, 256, "float16", 16, 4096, 4096),
    ("mha_prefix", 32, 32, 128, "float16", 16, 1000 + 64, 1000 + 1048),
])
def test_recipe_shapes(name, hq, hkv, d, dtype, batch, lmin, lmax):
    w = _make(name)
    dec = _decode(w)
    assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.dtype) == (hq, hkv, d, dtype)
    assert dec.q.shape == (batch, hq, d)
    assert lmin <= dec.seq_lens.min() and dec.seq_lens.max() <= lmax
    assert w.scale == pytest.approx(1 / np.sqrt(d))


def test_tiny_lengths_and_pool():
    """The tiny configuration: post-append lengths {5, 17, 33} in a 16-block pool."""
    w = W.tiny()
    assert sorted(_decode(w).seq_lens.tolist()) == [5, 17, 33] and w.num_blocks == 16


def test_ragged_trace_recipe():
    """Batch 64, lengths within [16, 4096] plus the steps' appends, 128 steps of one
    new token per sequence, a pool of 64 * ceil(4224 / 16) blocks."""
    w = _make("ragged")
    assert len(w.steps) == 128 and w.num_blocks == 64 * -(-4224 // 16)
    first = _decode(w, 0)
    assert first.q.shape == (64, 32, 128)
    assert first.seq_lens.min() >= 16 and first.seq_lens.max() <= 4096 + 1
    for s in range(1, len(w.steps)):
        dec = _decode(w, s)
        assert dec.seq_lens.max() <= 4096 + 128 and dec.seq_lens.min() >= 16


def test_specdec_recipe():
    """Speculative verification: 2 new tokens per sequence, q [B][2][H_q][d]."""
    w = W.specdec()
    dec = _decode(w)
    assert dec.q.shape == (64, 2, 32, 128) and len(w.steps) == 16
    assert dec.seq_lens.min() >= 512 + 2 - 2 and dec.seq_lens.max() <= 4096 + 2 * 16


@pytest.mark.parametrize("name", ["tiny", "gqa_b8", "long", "mha_prefix"])
def test_same_seed_same_arrays(name):
    a, b = _make(name), getattr(W, name)()
    da, db = _decode(a), _decode(b)
    assert np.array_equal(da.q, db.q) and np.array_equal(da.block_tables, db.block_tables)
    for ra, rb in zip(a.setup, b.setup):
        assert np.array_equal(ra.k, rb.k) and np.array_equal(ra.slot_mapping, rb.slot_mapping)


@pytest.mark.parametrize("name", ["tiny", "gqa_b8", "long", "mqa", "d256", "mha_prefix"])
def test_tables_stay_in_the_pool(name):
    """Every table entry a decode reads is a block of the pool, and every slot the
    setup writes lies in the pool."""
    w = _make(name)
    dec = _decode(w)
    for b, L in enumerate(dec.seq_lens):
        used = dec.block_tables[b, : -(-int(L) // 16)]
        assert used.min() >= 0 and used.max() < w.num_blocks
    for r in w.setup:
        s = r.slot_mapping[r.slot_mapping >= 0]
        assert s.max() < w.num_blocks * 16
