"""Plant known mistakes in the oracle (on the CPU) and check that a pin catches each.

The mistakes are compiled into copies of the C oracle with PA_ORACLE_MUTANT=n:
  1 scale dropped              2 off-by-one offset inside a block
  3 heads and tokens swapped inside a block            4 interleaved GQA groups
  5 per-block softmax sum (unnormalised)               6 softmax denominator left out
  7 fp16 exponent bias off by one                      8 cache write to the neighbouring slot
  9 newest-token slot one position late                10 floor instead of ceil for block counts
 11 fp8 codes rounded toward zero              12 causal mask one token late (prefill)
"""
import pytest

import oracle as oracle_pkg
import pins

MUTANTS = list(range(1, 13))


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("mutant", MUTANTS)
def test_some_pin_catches_mutant(mutant, mutant_dir):
    o = oracle_pkg.load_mutant(mutant, mutant_dir)
    assert o.mutant == mutant
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches planted mistake {mutant}"
