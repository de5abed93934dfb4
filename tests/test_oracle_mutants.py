"""Planted mistakes in the oracle are caught by its pins.

Each value of ORACLE_MUTANT compiles the oracle with one plausible error (a
transposed slot number, a wrong tie rule, an ignored low part of the exact
sum, a dropped forget gate, a flipped delta sign, a read before the write, a
dropped sparse weight, uniform weights, sum instead of mean in the RMS-norm,
a missing bf16 rounding, a decayed unselected slot, and in the backward a
dropped factor or term, an undecayed adjoint, a read gradient from the wrong
state, a softmax derivative without its mean, swapped score halves). The test rebuilds the
oracle on the CPU for each and requires that at least one pin fails.
"""

import pytest

import oracle as oracle_pkg
import oracle_pins

MUTANTS = {
    1: "slot numbered column-major",
    2: "ties to the highest slot",
    3: "low part of the exact sum ignored",
    4: "forget gate dropped",
    5: "delta sign flipped",
    6: "read before the write",
    7: "sparse write weight dropped",
    8: "uniform weights",
    9: "RMS-norm over the sum, not the mean",
    10: "bf16 state not rounded",
    11: "unselected slot decayed",
    12: "backward: (1 - beta k) dropped from dalpha",
    13: "backward: adjoint not decayed by the write",
    14: "backward: read gradient from the state before the write",
    15: "backward: dk without its m~ term",
    16: "backward: softmax mean not subtracted",
    17: "backward: score halves swapped",
    18: "backward: RMS-norm normaliser treated as a constant",
    19: "fp8 state: block maximum above 448 clipped (scale one binade too low)",
    20: "fp8 state: rounding toward zero",
    21: "fp8 state: overflow to the NaN code",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, tmp_path):
    lib = oracle_pkg.build(mutant=mutant, out=tmp_path / f"liboracle_m{mutant}.so", force=True)
    failed = oracle_pins.failing_pins(oracle_pkg.Oracle(lib))
    assert failed, f"no pin catches mutant {mutant} ({MUTANTS[mutant]})"
