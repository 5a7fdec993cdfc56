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
