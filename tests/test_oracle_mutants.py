"""Plant a known mistake in the oracle (compile-time ORACLE_MUTANT, on the CPU)
and check that at least one pin rejects each variant."""
import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    1: "scale dropped from the scores",
    2: "bias subtracted instead of added",
    3: "causal diagonal off by one",
    4: "GQA heads grouped by modulo instead of by block",
    5: "row max dropped from LSE",
    6: "wrong sign in dS = P (dP - D)",
    7: "scale dropped from dQ",
    8: "dS used in place of P for dV",
    9: "running state not rescaled when the max grows",
    10: "K used in place of V in the output",
    11: "local window one key short on the left",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, mutant):
    lib = oracle.build(tmp_path / f"liboracle_m{mutant}.so", mutant=mutant)
    orc = oracle.Oracle(lib)
    failed = [name for name, pin in ALL_PINS.items() if not pin(orc)[0]]
    assert failed, f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"
