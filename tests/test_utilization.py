"""KV memory accounting (paged blocks against contiguous preallocation) on the
host: closed forms on small traces, bounds on the ragged trace, sharing."""
import numpy as np
import pytest

from paged_kv_cache_395_b200 import utilization as U, workloads as W


def test_tiny_closed_form():
    """Lengths 5, 17, 33 hold 1 + 2 + 3 blocks = 96 slots for 55 tokens; a
    contiguous scheme reserving the 48-token table width holds 3 x 48."""
    (u,) = U.account(W.tiny())
    assert (u.tokens, u.paged_slots, u.paged_used, u.contiguous_slots) == (55, 96, 55, 144)
    assert u.paged_utilization == pytest.approx(55 / 96)
    assert u.contiguous_utilization == pytest.approx(55 / 144)


def test_block_multiple_lengths_fill_every_slot():
    """Every length a multiple of 16 (the 7B-GQA batch-8 config, 1024 tokens):
    no slot of any block is empty, and a 1024-token reservation is also full."""
    (u,) = U.account(W.gqa_b8())
    assert u.paged_utilization == 1.0 and u.contiguous_utilization == 1.0 and u.sharing == 1.0


def test_random_lengths_against_direct_count():
    lens = [1, 15, 16, 17, 100, 257]
    w = W.random_case(lens, seed=3)
    (u,) = U.account(w, max_len=300)
    blocks = sum(-(-L // 16) for L in lens)
    assert u.paged_slots == 16 * blocks and u.paged_used == sum(lens)
    assert u.contiguous_slots == 300 * len(lens)
    # paged waste is under one block per sequence
    assert u.paged_slots - u.paged_used < 16 * len(lens)


@pytest.fixture(scope="module")
def ragged_usage():
    return U.account(W.ragged())


def test_ragged_waste_bounds(ragged_usage):
    for u in ragged_usage:
        assert 0 <= u.paged_slots - u.paged_used < 16 * u.sequences
        assert u.sharing == 1.0  # no prefix sharing in this trace


def test_ragged_reproduces_the_pages_contrast(ragged_usage):
    """The pages put contiguous preallocation at 20-40 % use (60-80 % wasted)
    and paged blocks above 90 % (chanyi.net.cn/article/49 section 三;
    hdu-wiki.cn/courses/inference-kvcache-vllm section 9.1).  On the ragged trace,
    reserving the 4224-token table width per request:"""
    s = U.summary(ragged_usage)
    assert s["paged_utilization"] > 0.9
    assert 0.6 <= s["contiguous_waste"] <= 0.9
    assert s["concurrency_gain"] > 2  # the pages report about twice the concurrency


def test_shared_prefix_counts_blocks_once():
    """MHA with a 1000-token prefix shared by 16 sequences: the prefix blocks
    are held once, so logical tokens exceed physical ones."""
    w = W.mha_prefix()
    (u,) = U.account(w)
    unique = int(w.notes.split("unique_blocks=")[1])
    assert u.paged_slots == 16 * unique
    assert u.sharing > 2
    assert 0.9 < u.paged_utilization <= 1.0
