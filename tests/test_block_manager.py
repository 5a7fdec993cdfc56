"""Host block manager: property tests and the recipes' paging structure."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from paged_kv_cache_395_b200 import workloads as W
from paged_kv_cache_395_b200.block_manager import BlockManager, OutOfBlocks


def test_alloc_order_follows_free_order():
    bm = BlockManager(5, 16, free_order=[3, 1, 4, 0, 2])
    slots = bm.add_sequence("a", 33)  # 3 blocks
    assert bm.tables["a"] == [3, 1, 4]
    assert slots[0] == 48 and slots[16] == 16 and slots[32] == 64
    bm.free_sequence("a")
    # LIFO: the last freed block comes back first
    assert bm.add_sequence("b", 1).tolist() == [64]
    bm.check_invariants()


def test_append_crosses_block_boundary():
    bm = BlockManager(4, 16)
    bm.add_sequence(0, 16)
    slot, cow = bm.append_slot(0)
    assert cow is None and slot == 16 and bm.tables[0] == [0, 1] and bm.lens[0] == 17


def test_out_of_blocks_is_all_or_nothing():
    bm = BlockManager(3, 16)
    bm.add_sequence(0, 32)
    with pytest.raises(OutOfBlocks):
        bm.add_sequence(1, 17)
    assert 1 not in bm.tables and bm.num_free == 1
    bm.check_invariants()


def test_double_free_detected():
    bm = BlockManager(2, 16)
    bm.add_sequence(0, 3)
    bm._release(0)
    with pytest.raises(RuntimeError):
        bm._release(0)


def test_copy_on_write_rule():
    """Fork 3 sequences from a prefix ending in a partial block: the first two
    appends copy the shared block, the last sharer writes in place, and the
    shared full blocks stay shared."""
    bm = BlockManager(10, 16)
    bm.add_sequence(0, 20)  # blocks 0 (full), 1 (4 tokens)
    bm.fork(0, 1)
    bm.fork(0, 2)
    assert bm.refcount[0] == 3 and bm.refcount[1] == 3
    s0, c0 = bm.append_slot(0)
    s1, c1 = bm.append_slot(1)
    s2, c2 = bm.append_slot(2)
    assert c0 == (1, 2) and c1 == (1, 3) and c2 is None
    assert s0 == 2 * 16 + 4 and s1 == 3 * 16 + 4 and s2 == 1 * 16 + 4
    assert bm.tables[2] == [0, 1] and bm.refcount[0] == 3 and bm.refcount[1] == 1
    bm.check_invariants()
    for s in (0, 1, 2):
        bm.free_sequence(s)
    assert bm.num_free == 10
    bm.check_invariants()


@settings(max_examples=60, deadline=None)
@given(st.lists(st.tuples(st.sampled_from(["add", "append", "fork", "free"]),
                          st.integers(0, 7), st.integers(1, 70)), max_size=80))
def test_random_operations_keep_invariants(ops):
    bm = BlockManager(24, 16)
    live = []
    nid = 0
    for kind, pick, n in ops:
        try:
            if kind == "add" or not live:
                bm.add_sequence(nid, n)
                live.append(nid)
                nid += 1
            elif kind == "append":
                s = live[pick % len(live)]
                before = {o: list(bm.tables[o]) for o in live if o != s}
                _, cow = bm.append_slot(s)
                # no other sequence's table changes
                assert all(bm.tables[o] == t for o, t in before.items())
                if cow is not None:
                    assert cow[0] != cow[1] and bm.refcount[cow[1]] == 1
            elif kind == "fork":
                bm.fork(live[pick % len(live)], nid)
                live.append(nid)
                nid += 1
            else:
                bm.free_sequence(live.pop(pick % len(live)))
        except OutOfBlocks:
            pass
        bm.check_invariants()
    for s in live:
        bm.free_sequence(s)
    assert bm.num_free == 24
    bm.check_invariants()


def test_tiny_recipe_layout():
    w = W.tiny()
    dec = w.steps[0][1]
    assert dec.seq_lens.tolist() == [5, 17, 33]
    perm = np.random.default_rng(1).permutation(16)
    bt = dec.block_tables
    used = [bt[0, 0], bt[1, 0], bt[1, 1], bt[2, 0], bt[2, 1], bt[2, 2]]
    assert sorted(used) == sorted(perm[:6].tolist())
    # appended tokens: offset 4 of block 0, offset 0 of logical block 1 and 2
    slots = w.steps[0][0].slot_mapping
    assert slots.tolist() == [bt[0, 0] * 16 + 4, bt[1, 1] * 16, bt[2, 2] * 16]


def test_mha_prefix_recipe():
    w = W.mha_prefix()
    cp, rs, dec = w.steps[0]
    assert cp.pairs.shape == (15, 2)  # sequences 0..14 copy, 15 writes in place
    assert len(set(cp.pairs[:, 0].tolist())) == 1  # all copies read the shared partial block
    assert np.all(dec.seq_lens >= 1064) and np.all(dec.seq_lens <= 2048)
    bt = dec.block_tables
    assert np.all(bt[:, :62] == bt[0, :62])  # full prefix blocks shared by all
    assert len(set(bt[:, 62].tolist())) == 16  # the partial block is private after CoW


@pytest.mark.slow
def test_ragged_recipe_replays_without_leak():
    w = W.ragged(num_steps=128)
    assert len(w.steps) == 128
    lens0 = w.steps[0][1].seq_lens
    assert lens0.min() >= 17 and lens0.max() <= 4097
    for ops in w.steps:
        dec = ops[1]
        assert dec.block_tables.shape == (64, 264)
        nblk = -(-dec.seq_lens // 16)
        for b in range(64):
            row = dec.block_tables[b]
            assert np.all(row[: nblk[b]] >= 0) and np.all(row[nblk[b]:] == -1)
        # every (block, offset) written this step is distinct
        s = ops[0].slot_mapping
        assert len(np.unique(s)) == len(s)


def test_deferred_free_holds_blocks_back_one_step():
    """free_sequence(defer=True) keeps the blocks off the free list until
    release_deferred(); an immediate free hands the same block out next (LIFO)."""
    bm = BlockManager(4, 16)
    bm.add_sequence("a", 16)
    a_block = bm.tables["a"][0]
    bm.free_sequence("a")
    bm.add_sequence("b", 16)
    assert bm.tables["b"][0] == a_block  # immediate reuse
    bm.free_sequence("b", defer=True)
    bm.check_invariants()
    bm.add_sequence("c", 16)
    assert bm.tables["c"][0] != a_block and bm.num_free == 2
    bm.release_deferred()
    bm.add_sequence("d", 16)
    assert bm.tables["d"][0] == a_block
    bm.check_invariants()


@pytest.mark.parametrize("name", ["ragged", "specdec"])
def test_appends_never_touch_the_previous_decode(name):
    """The recipes that mark appends_overlap_previous (so their appends run with
    PA_APPEND_OVERLAP_PREVIOUS): no slot that step i + 1's appends write lies
    within a sequence's length in step i's decode, the prompts of newly admitted
    sequences included."""
    w = getattr(W, name)()
    assert w.appends_overlap_previous
    for i in range(len(w.steps) - 1):
        dec = [op for op in w.steps[i] if isinstance(op, W.Decode)][0]
        read = []
        for b, L in enumerate(dec.seq_lens):
            t = np.arange(int(L), dtype=np.int64)
            read.append(dec.block_tables[b][t // 16].astype(np.int64) * 16 + t % 16)
        read = np.concatenate(read)
        written = np.concatenate([op.slot_mapping for op in w.steps[i + 1] if isinstance(op, W.Reshape)])
        written = written[written >= 0]
        assert not np.isin(written, read).any(), f"step {i + 1} appends into slots step {i} reads"
