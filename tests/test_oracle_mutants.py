"""Each planted mistake in the oracle (FDO_MUTANT in fd_oracle.c) must be
caught by at least one pin: this shows the pins constrain every step of the
oracle (scale, group mapping, sequence length, log base, value operand,
normalisation, split reduction, causal offset, dequantisation, the dot product's terms, the value operand's index)."""
import pytest

import oracle
from oracle import build as oracle_build
from oracle_pins import ALL_PINS

MUTANTS = {
    1: "scale dropped from the logits",
    2: "query head i reads kv head i % Hkv",
    3: "last token of each row dropped",
    4: "log-sum-exp in base 2",
    5: "keys used as values",
    6: "softmax weights not normalised",
    7: "split weights not rescaled by the total log-sum-exp",
    8: "each of several queries sees one token too few",
    9: "E4M3 subnormal codes decoded as normals",
    10: "values dequantised with the key scale",
    11: "int8 codes read as unsigned",
    12: "dot product drops the last head-dim term",
    13: "E4M3 exponent bias 8 instead of 7",
    14: "output dimension d reads value dimension D-1-d",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_pins_catch_mutant(tmp_path, mutant):
    path = oracle_build.build(str(tmp_path / f"libfd_oracle_m{mutant}.so"), mutant=mutant)
    orc = oracle.Oracle(path)
    assert orc.mutant == mutant
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError as e:
            failed.append(f"{pin.__name__}: {e}")
    assert failed, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
