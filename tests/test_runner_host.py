"""Host logic of the runner (no GPU): which steps pa_decode_append can take."""
import numpy as np

from paged_kv_cache_395_b200 import runner, workloads as W


def test_ragged_steps_end_with_one_token_per_sequence():
    """Every ragged step's append ends with its sequences' new tokens, each at the
    slot of its sequence's last position: the leading tokens are the admitted
    prompts."""
    w = W.ragged(num_steps=6, batch=8, finish_p=0.3)
    saw_prompts = False
    for ops in w.steps:
        lead = runner.new_token_split(ops)
        r, d = ops
        B = len(d.seq_lens)
        assert lead == len(r.slot_mapping) - B
        saw_prompts |= lead > 0
        for b in range(B):
            pos = int(d.seq_lens[b]) - 1
            assert r.slot_mapping[lead + b] == d.block_tables[b, pos // 16] * 16 + pos % 16
    assert saw_prompts


def test_steps_without_a_trailing_new_token_are_not_split():
    w = W.random_case([5, 17, 33], seed=3)
    assert runner.new_token_split(w.steps[0]) is None          # the step is a decode alone
    w = W.ragged(num_steps=2, batch=4)
    ops = w.steps[1]
    bad = W.Reshape(ops[0].k, ops[0].v, ops[0].slot_mapping.copy())
    bad.slot_mapping[-1] += 1                                  # not the last position's slot
    assert runner.new_token_split([bad, ops[1]]) is None
    short = W.Reshape(ops[0].k[:2], ops[0].v[:2], ops[0].slot_mapping[:2])
    assert runner.new_token_split([short, ops[1]]) is None     # fewer tokens than sequences
    sd = W.specdec(num_steps=1, batch=4)
    assert runner.new_token_split(sd.steps[0]) is None         # two new tokens per sequence


def test_an_empty_sequence_takes_no_new_token():
    w = W.random_case([4, 0, 9], num_q_heads=4, num_kv_heads=2, seed=5)
    dec = w.steps[0][0]
    tok = W.Reshape(np.zeros((3, 2, 64), np.float16), np.zeros((3, 2, 64), np.float16),
                    np.array([dec.block_tables[0, 0] * 16 + 3, -1, dec.block_tables[2, 0] * 16 + 8]))
    assert runner.new_token_split([tok, dec]) == 0
    tok.slot_mapping[1] = 5
    assert runner.new_token_split([tok, dec]) is None
