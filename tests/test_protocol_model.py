"""The attention kernel's mbarrier protocol, model-checked on random schedules (CPU only): no
data hazard and no deadlock in any of the kernel's layouts, and each planted protocol mistake
is caught."""
import random

import pytest

from protocol_model import LAYOUTS, MUTANTS, Deadlock, Violation, random_units, run

SEEDS = 300


@pytest.mark.parametrize("layout", LAYOUTS, ids=[f"nt{a}_nsm{b}_qt{int(c)}_k{d}_v{e}_pipe{int(f)}"
                                                 for a, b, c, d, e, f in LAYOUTS])
def test_protocol_holds(layout):
    NT, NSM, q_tmem, NK, NV, pipe = layout
    for seed in range(SEEDS):
        units = random_units(random.Random(seed * 7 + NT))
        run(units, NT, NSM, q_tmem, NK, NV, seed, pipe=pipe)


@pytest.mark.parametrize("layout", [x for x in LAYOUTS if x[0] == 2 and not x[5]],
                         ids=lambda x: f"k{x[3]}_v{x[4]}_qt{int(x[2])}")
def test_protocol_holds_with_late_turn(layout):
    """The E4M3 layout's order: each tile waits for and loads its own S before its turn."""
    NT, NSM, q_tmem, NK, NV, pipe = layout
    for seed in range(SEEDS):
        units = random_units(random.Random(seed * 11 + NT))
        run(units, NT, NSM, q_tmem, NK, NV, seed, pipe=pipe, late_turn=True)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_model_catches_planted_mistake(mutant):
    caught = 0
    for NT, NSM, q_tmem, NK, NV, pipe in LAYOUTS:
        for seed in range(60):
            units = random_units(random.Random(seed * 7 + NT))
            try:
                run(units, NT, NSM, q_tmem, NK, NV, seed, mutant=mutant, pipe=pipe)
            except (Violation, Deadlock):
                caught += 1
    assert caught > 0, f"the model did not catch: {MUTANTS[mutant]}"
