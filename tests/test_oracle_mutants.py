"""Each planted mistake in the oracle (compile-time ORACLE_MUTANT) must fail at least one pin.

Mutants: 1 no max subtraction, 2 wrong exponent sign, 3 interleaved GQA groups, 4 top-left
causal alignment, 5 V read transposed, 6 LSE without its max term, 7 scale dropped,
8 probabilities not normalised, 9 fp16 subnormals widened with an implicit leading one,
10 a block list read as an upper bound, 11 split weights of the merge not divided by their sum,
12 the transposed flow's probabilities renormalised over the query axis, 13 the transposed
flow's final transpose left out, 14 listed blocks exempt from the causal rule.
"""
import pytest

from oracle import oracle
from tests import oracle_pins

MUTANTS = list(range(1, 15))


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(mutant):
    oracle.build(mutant)
    assert oracle._lib(mutant).oracle_mutant_id() == mutant
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"mutant {mutant} passed every pin"
