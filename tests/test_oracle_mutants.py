"""Mutation check of the pins: each deliberate mistake compiled into the oracle
(ORACLE_MUTANT in dsa_oracle.c) must make at least one pin fail.  The mistakes are
planted only in CPU builds of the oracle (mutants 9..13 in the oracle's Python
functions)."""
import pytest

import oracle_pins as P
from oracle import oracle as O

MUTANTS = {
    1: "ReLU dropped",
    2: "head weight dropped",
    3: "diagonal key excluded",
    4: "last indexer dim dropped",
    5: "ties go to the higher index",
    6: "softmax scale dropped",
    7: "value read from the wrong slice",
    8: "lse without the max",
    9: "E4M3 exponent bias 8",
    10: "E4M3 subnormals decoded as normals",
    11: "E4M3 encoder ties away from zero",
    12: "fp8 attention output without kv_scale",
    13: "varlen indices without the packed offset",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_mutant_is_caught(mutant):
    assert O.load(mutant).oracle_mutant_id() == mutant
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {mutant} ({MUTANTS[mutant]})"
