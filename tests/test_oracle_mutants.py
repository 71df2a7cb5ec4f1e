"""The pins catch plausible mistakes: each planted mistake in a copy of the oracle fails a pin.

Every mutant is a separate build of oracle/kda_oracle.cpp with one -DKDA_ORACLE_MUTANT value; the
default build (used everywhere else) compiles none of them. Mistakes are planted on the CPU only.
"""

import pytest

import oracle
from test_oracle_pins import CHECKS

MUTANTS = {
    1: "decays the value axis instead of the key axis",
    2: "reads out before the write",
    3: "drops beta",
    4: "writes k and delta on swapped axes",
    5: "carries the state across document boundaries",
    6: "sign error in the gate",
    7: "ignores the initial state",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m].replace(" ", "-"))
def test_some_pin_fails_on_planted_mistake(mutant):
    orc = oracle.Oracle(mutant)
    failed = []
    for check in CHECKS:
        try:
            check(orc)
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, "no pin caught mutant %d (%s)" % (mutant, MUTANTS[mutant])


def test_default_build_passes_every_pin():
    orc = oracle.default()
    for check in CHECKS:
        check(orc)
