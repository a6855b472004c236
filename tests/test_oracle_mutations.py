"""Each planted mistake in the oracle is caught by at least one pin.

The mistakes are compiled into separate builds of the oracle's C file
(-DORACLE_PLANT=n); the committed oracle (n = 0) is untouched.
  1 scale ignored (1 instead of 1/sqrt(D))     6 -- (unused)
  2 gate dropped (q = q_fixed + q_dyn)          7 last key dropped (off by one)
  3 synthesis reads k instead of k0             8 q_fixed indexed by batch, not head
  4 encode uses the keys as values              9 exponent sign flipped
  5 decode swaps latent keys and values        10 softmax normalisation dropped
 11 synthesis normalisation by the L2 norm     12 synthesis keys/values not normalised
(11 and 12 are planted in the oracle's Python normalisation step.)
"""
import pytest

import oracle
from oracle_pins import PINS  # noqa: E402

PLANTS = [1, 2, 3, 4, 5, 7, 8, 9, 10, 11, 12]


@pytest.mark.parametrize("plant", PLANTS)
def test_planted_mistake_is_caught(plant):
    oracle.build(plant)
    failed = [name for name, fn in PINS.items() if not fn(plant)]
    assert failed, f"planted mistake {plant} passes every pin"
