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


def _settings():
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "workload_settings.txt")
    out = {}
    with open(path) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                key, *vals = ln.split()
                out[key] = [int(v) for v in vals]
    return out


def test_workloads_take_the_pages_settings():
    """The benchmark workloads' shapes and settings against the golden values
    cited from the pages (model shape, windows, lengths, the periodic skip)."""
    from structured_sparse_attention_fibonacci_b200.inputs import WORKLOADS
    g = _settings()
    for name in ("paper_fwd", "learned_train", "extrap_4x", "pi_skip", "pi_gate_train"):
        wl = WORKLOADS[name]
        assert wl.L == g["layers"][0], name
        assert wl.H * wl.D == g["hidden"][0], name
    for name in ("paper_fwd", "learned_train", "extrap_4x"):
        assert WORKLOADS[name].window in g["windows"]
        assert WORKLOADS[name].window == g["best_window"][0]
    assert WORKLOADS["paper_fwd"].T == WORKLOADS["learned_train"].T == g["train_len"][0]
    assert WORKLOADS["extrap_4x"].T == g["eval_len"][0]
    # the power-of-2 control at the evaluation length, with the linear stagger
    p2 = WORKLOADS["pow2_extrap"]
    assert p2.T == g["eval_len"][0] and p2.offsets == tuple(g["pow2_eval_ladder"])
    assert max(p2.offsets) < p2.T <= 2 * max(p2.offsets)
    assert p2.alpha_kind == "linear" and p2.window == g["best_window"][0]
    assert p2.L == g["layers"][0] and p2.H * p2.D == g["hidden"][0]
    # the autoregressive periodic skip: the k previous keys plus the current
    # one, and one offset pi at alpha = 1
    for name in ("pi_skip", "pi_gate_train"):
        wl = WORKLOADS[name]
        assert wl.window == g["pi_k"][0] + 1 and wl.offsets == tuple(g["pi_period"])
        assert wl.alpha_kind == "fixed"
