"""Plant mistakes in the oracle (on the CPU) and check that the pins catch each one.

Every ORACLE_MUTATION build in oracle/gqa_oracle.cpp is a plausible slip: an
interleaved head map, a dropped scale, a carry rescaled with the wrong sign, an
output not divided by the partition, a transposed cache layout, partial states
merged without rescaling, a dropped last key, keys used as values, a bias added
before the scale, a top-k index one past a sequence's end accepted, the code
word's fields swapped, a carry whose acc is not rescaled, a bias read by the
key's position in its sequence, empty states (carry or merge input) raising the
maximum, binary16 subnormals off by a factor of two.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

MUTATIONS = {1: "interleaved head map", 2: "scale dropped", 3: "carry sign flipped",
             4: "not divided by partition", 5: "cache layout transposed",
             6: "merge without rescaling", 7: "last key dropped", 8: "keys used as values",
             9: "bias inside the scale", 10: "top-k admits one past the end",
             11: "code word fields swapped", 12: "carry acc not rescaled",
             13: "bias indexed by sequence position", 14: "empty carry raises the maximum",
             15: "merge counts empty states in the maximum", 16: "f16 subnormals halved"}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_pins_catch_mutation(tmp_path, mutation):
    path = os.path.join(str(tmp_path), f"liboracle_mut{mutation}.so")
    oracle_build.build(path, mutation)
    handle = oracle_pins.OracleHandle(oracle, oracle.load(path))
    failed = oracle_pins.run_all(handle)
    assert failed, f"no pin caught mutation {mutation} ({MUTATIONS[mutation]})"
