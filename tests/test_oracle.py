"""The fp64 oracle against its pins (no GPU)."""
import numpy as np
import pytest

import oracle
from oracle_pins import all_pins, rand_case, run_oracle, rel_err

PINS = all_pins()


@pytest.mark.parametrize("name,pin", PINS, ids=[n for n, _ in PINS])
def test_pin(name, pin):
    pin(oracle.default())


@pytest.mark.parametrize("kind", [oracle.LINEAR, oracle.LINEAR_LN, oracle.MLP_LN])
def test_dual_form_at_working_size(kind):
    """The dual-form pin at the working head size (d = 64, h = 256, b = 16)."""
    from oracle_pins import pin_dual_form
    pin_dual_form(oracle.default(), kind, seed=11, B=1, H=1, T=48, d=64, b=16, eps=1e-6)


def test_thread_count_does_not_change_results():
    c = rand_case(oracle.LINEAR_LN, 3, B=3, H=2, T=8, b=4)
    Z1, W1 = run_oracle(oracle.default(), c, nthreads=1)
    Z4, W4 = run_oracle(oracle.default(), c, nthreads=4)
    assert np.array_equal(Z1, Z4) and np.array_equal(W1, W4)


def test_bad_arguments_are_rejected():
    c = rand_case(oracle.LINEAR, 0, T=12, b=4)
    with pytest.raises(ValueError):
        oracle.default().forward(oracle.LINEAR, c["Q"], c["K"], c["V"], c["eta"], c["params"], 5)
    with pytest.raises(ValueError):  # LN without gamma/beta
        oracle.default().forward(oracle.LINEAR_LN, c["Q"], c["K"], c["V"], c["eta"], c["params"], 4)


def test_empty_sequence_returns_initial_state():
    c = rand_case(oracle.LINEAR, 0, T=0, b=4)
    Z, W = run_oracle(oracle.default(), c)
    assert Z.shape[2] == 0
    assert np.array_equal(W[0], c["params"]) and np.array_equal(W[1], c["params"])
