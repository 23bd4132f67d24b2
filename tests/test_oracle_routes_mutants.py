"""The top-k / top-p pins must catch plausible mistakes in the oracle's selection code.

Each case plants one mistake into a copy of oracle/sol_ref_routes.py (in memory, on the CPU) and
checks that at least one pin of tests/test_oracle_routes.py rejects it.
"""
import inspect
import types

import pytest

import test_oracle_routes as pins
from oracle import sol_ref_routes

MUTANTS = {
    "ascending_order": ("np.argsort(-np.asarray(row, np.float64)", "np.argsort(np.asarray(row, np.float64)"),
    "ties_by_high_index": ('return np.argsort(-np.asarray(row, np.float64), kind="stable")',
                           'n = len(row)\n    return n - 1 - np.argsort(-np.asarray(row, np.float64)[::-1], kind="stable")'),
    "topk_one_extra": ("mask[u, order_desc(proxy[u])[:kk]] = 1", "mask[u, order_desc(proxy[u])[:kk + 1]] = 1"),
    "topp_strict": ("cum >= target", "cum > target"),
    "topp_one_short": ("mask[u, order[:t + 1]] = 1", "mask[u, order[:max(t, 1)]] = 1"),
    "topp_linear_mass": ("w = np.exp(s - s.max())", "w = s - s.min()"),
}

PINS = [
    lambda: pins.test_topk_equals_rank_definition(3),
    lambda: pins.test_topk_equals_rank_definition(5),
    lambda: pins.test_topp_equals_rank_definition(0.5),
    lambda: pins.test_topp_equals_rank_definition(0.77),
    pins.test_topp_two_block_closed_form,
    pins.test_topp_exact_mass_tie_keeps_the_shortest_prefix,
    pins.test_topk_nested_in_k,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    old, new = MUTANTS[name]
    src = inspect.getsource(sol_ref_routes)
    assert src.count(old) == 1, name
    mod = types.ModuleType("mutant_routes")
    exec(compile(src.replace(old, new), "mutant_routes", "exec"), mod.__dict__)
    monkeypatch.setattr(pins, "rr", mod)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ArithmeticError):   # a wrong value, or a crash on a pin's input
            caught += 1
    assert caught > 0, f"mutant {name} passed every pin"


def test_unmutated_module_passes_the_same_pins():
    for pin in PINS:
        pin()
