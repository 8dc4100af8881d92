"""Each planted mistake in the oracle must fail at least one pin (CPU only).

The mistakes are compiled into separate copies of the oracle (oracle.c,
AGREF_MUTANT) inside pytest's temporary folder; the real oracle is untouched.
"""
import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

MUTANTS = {
    1: "bias read transposed (key block as row)",
    2: "cap applied before the bias is added",
    3: "1/sqrt(D) dropped",
    4: "bias scaled by 1/sqrt(D)",
    5: "query block index off by one",
    6: "lse without the max term",
    7: "softmax weights not normalised",
    8: "projection output p and q swapped",
    9: "projection W read as [H, Cp]",
    10: "values read from K",
    11: "every head uses query head 0",
    12: "soft cap dropped",
    13: "every batch item reads item 0's bias",
    14: "partial last block dropped from the bias layout",
    15: "backward: derivative of the soft cap dropped",
    16: "backward: softmax Jacobian without the delta term",
    17: "backward: 1/sqrt(D) missing from dk",
    18: "backward: a shared bias's gradient taken from item 0 only",
}


@pytest.mark.parametrize("mid", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_mutant_is_caught(tmp_path, mid):
    lib = oracle_build.build(str(tmp_path / f"liboracle_m{mid}.so"), mutant=mid)
    o = oracle.Oracle(lib)
    assert o.mutant == mid
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError) as e:
            failed.append((pin.__name__, str(e).splitlines()[0][:80]))
    assert failed, f"mutant {mid} ({MUTANTS[mid]}) passed every pin"
