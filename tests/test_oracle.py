"""The CPU oracle against its pins (see oracle_pins.py), and planted mistakes."""
import os
import tempfile

import pytest

import oracle
from oracle import build as oracle_build

from . import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# Each planted mistake (see MUT(n) in pa_oracle.c) must make at least one pin fail.
MUTATIONS = {
    1: "GQA head mapping h % H_kv",
    2: "gather offset off by one",
    3: "softmax scale dropped",
    4: "appended token not attended",
    5: "merge not normalised",
    6: "int8 scale absmax / 128",
    7: "append writes K into the V cache",
    8: "K used in place of V (transposed operand)",
    9: "partition lse without log l",
    10: "block copy skips V",
    11: "multi-query causal range one token short",
    12: "int4 nibbles read in swapped order",
    13: "int4 scale absmax / 8",
    14: "int8 append re-rounds with the old scale",
}

# pins cheap enough to run once per mutant
FAST_PINS = [p for p in pins.ALL_PINS if p not in (pins.pin_half_exhaustive, pins.pin_bf16_exhaustive)]


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_oracle_mutations(mutation):
    with tempfile.TemporaryDirectory() as tmp:
        path = oracle_build.build(out=os.path.join(tmp, f"liboracle_m{mutation}.so"),
                                  mutation=mutation)
        saved = oracle._lib
        oracle._lib = oracle.load(path)
        failed = []
        try:
            for pin in FAST_PINS:
                try:
                    pin()
                except (AssertionError, RuntimeError) as e:
                    failed.append((pin.__name__, str(e)[:80]))
        finally:
            oracle._lib = saved
    assert failed, f"no pin caught mutation {mutation}: {MUTATIONS[mutation]}"


def test_bf16_output_rounding_alone_can_exceed_the_bound():
    """Why the bf16 parity check puts 2e-3 + 2e-3 |ref| on the fp32 result before
    the output's rounding: bf16 keeps 8 significant bits, so the correctly rounded
    value of the exact (oracle) result is off by up to 2^-8 |ref|, which exceeds
    2e-3 + 2e-3 |ref| once |ref| >= 2 (half a unit in the last place there is
    2^-7 >= 0.0078 against a bound of 0.006 at |ref| = 2).  On short bf16 sequences,
    whose outputs reach |ref| > 2, the best possible bf16 output already breaks the
    bound on some elements, and only on elements with |ref| >= 2."""
    import numpy as np

    from paged_kv_cache_395_b200 import workloads as W

    from .oracle_replay import replay
    w = W.random_case([2, 3, 5, 33], num_q_heads=16, num_kv_heads=2, head_dim=128, dtype="bfloat16", seed=7)
    ref = replay(w)[0][0]
    f = ref.astype(np.float32)
    u = f.view(np.uint32)
    rne = ((u + np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1))) & np.uint32(0xFFFF0000)).view(np.float32)
    err = np.abs(rne.astype(np.float64) - ref)
    over = err > 2e-3 + 2e-3 * np.abs(ref)
    assert over.any()
    assert np.all(np.abs(ref[over]) >= 2.0)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-12)
