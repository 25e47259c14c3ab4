"""Each planted mistake in the oracle (built with -DORC_MUTANT=n) must fail at least one pin.

This shows the pins are strong enough to catch a plausible slip anywhere in the oracle: ReLU
after the head sum, weights dropped, top-left instead of right-down causal alignment, reversed
tie order, -0 kept, head/row strides exchanged, block table ignored, TND keys offset by the
query cumulative lengths, ReLU dropped, output offset dropped, wrong padding, compressed keys kept
when their first token is visible, a wrong fp16 exponent bias, a merge that drops a list, fp8 keys
without their scale, the backward's dI with the wrong sign, its target left unnormalised, the attention's rope
term dropped."""
import pytest

import oracle_pins
from oracle import oracle as orc_mod

MUTANTS = list(range(1, 19))


@pytest.mark.parametrize("mutant", MUTANTS)
def test_mutant_is_caught(tmp_path, mutant):
    orc = orc_mod.Oracle(orc_mod.build(mutant=mutant, out_dir=tmp_path))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {mutant} passed every pin"
