"""The pins have teeth: each deliberately wrong build of the oracle fails one.

The oracle source carries mutation points that are off in the shipped build
(LA_ORACLE_MUTANT = 0).  Each mutant below is a plausible mistake; it is
compiled into its own library on the CPU and must fail at least one pin.
"""
import os

import pytest

import oracle
from oracle import build as obuild
import oracle_pins

MUTANTS = {
    1: "strict causal mask (j < i): diagonal dropped",
    2: "RMSNorm eps added outside the square root",
    3: "state transposed in the recurrent readout",
    4: "inter-block term dropped in the blocked form",
    5: "recurrent readout before the state update",
    6: "decode readout before the state update",
    7: "intra-block mask not confined to the block (double count)",
    8: "RMSNorm over the sum instead of the mean of squares",
    9: "initial state left out of the quadratic-form readout",
    10: "initial state transposed in the recurrent and blocked forms",
    11: "initial state left out of the quadratic-form final state",
}


@pytest.mark.parametrize("mid", sorted(MUTANTS), ids=lambda m: f"mutant{m}")
def test_mutant_is_caught(mid, tmp_path):
    lib = obuild.build(force=True, out=os.path.join(tmp_path, f"libmut{mid}.so"),
                       defines=[f"LA_ORACLE_MUTANT={mid}"])
    failed = []
    with oracle.use_library(lib):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                # ValueError: the broken build produced a non-finite value, which the
                # error metric refuses to compare (every pin passes on the real build)
                failed.append(pin.__name__)
    assert failed, f"no pin catches mutant {mid}: {MUTANTS[mid]}"
