"""Planted mistakes in the oracle must each fail at least one pin.

Each mutant is the oracle's C source compiled with ORACLE_MUTANT=k, which
plants one plausible mistake (mutant 20: the paged cache's key and value planes
swapped; mutant 21: a prefill window one key short): a dropped square in the l2 correction, n_eff =
l/l2, a flipped gate sign, an off-by-one causal bound, a transposed GQA
mapping, a sample (not population) std, a log2 temperature, a dropped factor 2
under the null-floor root, a missing unit-sphere projection, and the wrong
head's count vector; in the backward, a dropped null-floor spread term, a
flipped sign on the squared-sum gradient, dv taken without the direction's
projection, and a dropped argmax term of the gate; in the memory channel, the decay gate
left off the erase term, the key/query normalisation skipped, a read taken
before the write, the operands of the update's matrix product swapped, and a
read through the transposed state.
"""
import pytest

import oracle
import oracle_pins as P

MUTANTS = list(range(1, 22))


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    for m in MUTANTS:
        oracle.build(m, build_dir=d)
    return d


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(mutant, mutant_dir):
    assert oracle.mutant_id(mutant, mutant_dir) == mutant
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(mutant=mutant, bd=mutant_dir)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {mutant} passed every pin"
