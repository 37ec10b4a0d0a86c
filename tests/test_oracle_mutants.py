"""Every planted mistake in the oracle fails at least one pin.

Each mutant is a build of oracle.c with -DORACLE_MUTANT=n: a digit order
reversed, a wrong trit-to-digit map, a wrong pad digit, missing validity
checks, a wrong binary16 subnormal decode, a dropped term, a flipped sign
and a reversed index.  The pins are run in this process against each build.
"""
import pytest

import oracle
import oracle_pins

MUTANTS = {
    1: "pack writes the most significant digit first",
    2: "trit maps to t mod 3 instead of t + 1",
    3: "partial byte padded with digit 0 instead of a 0-trit",
    4: "2-bit field value 3 accepted",
    5: "1.6-bit bytes >= 243 accepted",
    6: "binary16 subnormals decoded with the implicit bit",
    7: "last reduction term dropped",
    8: "trit sign flipped",
    9: "reduction index reversed",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_mutant_is_caught(mutant):
    o = oracle.Oracle(mutant)
    assert oracle_pins.failing_pins(o), f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"


def test_unmodified_oracle_passes_every_pin():
    assert oracle_pins.failing_pins(oracle.get()) == []
