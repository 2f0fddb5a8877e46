"""Each planted mistake in the oracle must be caught by at least one pin (CPU only).

The mutants are builds of the same C source with one plausible slip switched on
(see ORC_MUTANT in minf_oracle.c): no causal limit in the estimate, an
off-by-one diagonal, the main diagonal not forced, the Block-Sparse diagonal not
forced, an A-shape window one key short, a key counted twice in Vertical-Slash,
a Tri-shape tail one row short, a whole-slash-tile range one key too wide,
top-p slashes that ignore the forced diagonal's mass.
"""
import pytest

import oracle
import pins

MUTANTS = {
    1: "estimate without causal limit",
    2: "diagonal offset off by one",
    3: "slash offset 0 not forced",
    4: "block diagonal not forced",
    5: "A-shape window one short",
    6: "VS key counted twice",
    7: "Tri-shape dense tail one row short",
    8: "whole-slash-tile range one key too wide",
    9: "top-p without the forced diagonal's mass",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m])
def test_pins_catch_planted_mistake(tmp_path, mutant):
    orc = oracle.Oracle(mutant, out_dir=str(tmp_path))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError as e:
            caught.append((pin.__name__, str(e)))
    assert caught, f"no pin caught mutant {mutant} ({MUTANTS[mutant]})"
