"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import oracle_pins as P


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def test_schedules_and_offsets_golden():
    P.pin_schedules()


def test_inputs_module_uses_golden_values():
    from structured_sparse_attention_fibonacci_b200 import inputs
    assert inputs.FIB15 == P.FIB
    lin = inputs.alpha_linear_stagger().tolist()
    cop = inputs.alpha_coprime_stagger().tolist()
    for l, a, src in P.golden_alpha_schedules():
        assert abs(lin[l] - a) < 1e-7
        assert cop[l] == lin[src]


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
