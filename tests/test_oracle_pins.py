"""The fp64 oracle against results the mathematics fixes (CPU only)."""
import math

import numpy as np
import pytest

import oracle
import pins


def _rec(x, dt, A, B, C, D, init):
    return oracle.recurrence(x, dt, A, B, C, D, init)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_recurrence_pin(pin):
    pin(_rec)


def _step_as_rec(x, dt, A, B, C, D, init):
    """Drive the decode-step oracle token by token, as a recurrence."""
    b, L, H, P = x.shape
    N = B.shape[3]
    state = np.zeros((b, H, P, N)) if init is None else init
    ys = []
    for t in range(L):
        y, state = oracle.step(state, x[:, t], dt[:, t], A, B[:, t], C[:, t], D)
        ys.append(y)
    return np.stack(ys, axis=1), state


@pytest.mark.parametrize("pin", [pins.pin_geometric, pins.pin_scalar_brute, pins.pin_dta_neg_inf,
                                 pins.pin_group_map, pins.pin_init_only],
                         ids=lambda p: p.__name__)
def test_step_pin(pin):
    """The decode step, iterated, obeys the same closed forms."""
    pin(_step_as_rec)


def test_step_does_not_modify_input_state():
    rng = np.random.default_rng(7)
    st = rng.standard_normal((2, 3, 4, 5))
    keep = st.copy()
    oracle.step(st, rng.standard_normal((2, 3, 4)), np.full((2, 3), 0.1), -np.ones(3),
                rng.standard_normal((2, 1, 5)), rng.standard_normal((2, 1, 5)), np.ones(3))
    assert np.array_equal(st, keep)


def test_empty_sequence_returns_init():
    rng = np.random.default_rng(8)
    init = rng.standard_normal((2, 3, 4, 5))
    y, f = oracle.recurrence(np.zeros((2, 0, 3, 4)), np.zeros((2, 0, 3)), -np.ones(3),
                             np.zeros((2, 0, 1, 5)), np.zeros((2, 0, 1, 5)), np.ones(3), init)
    assert y.shape == (2, 0, 3, 4)
    assert np.array_equal(f, init)


def test_rejects_bad_group_count():
    with pytest.raises((ValueError, AssertionError)):
        oracle.recurrence(np.zeros((1, 2, 3, 4)), np.zeros((1, 2, 3)), -np.ones(3),
                          np.zeros((1, 2, 2, 5)), np.zeros((1, 2, 2, 5)), np.ones(3))


def test_threads_do_not_change_result():
    rng = np.random.default_rng(9)
    args = pins._rand_case(rng, 3, 50, 5, 4, 6, 1, True)
    y1, f1 = oracle.recurrence(*args, threads=1)
    y4, f4 = oracle.recurrence(*args, threads=4)
    assert np.array_equal(y1, y4) and np.array_equal(f1, f4)


def test_long_decay_underflows_cleanly():
    """A strongly decaying head forgets its initial state: after enough
    tokens the contribution of h0 is below fp64 resolution and nothing is
    NaN or infinite (the regime of A_h = -16 over a 256-token chunk)."""
    L = 400
    dt = np.full((1, L, 1), 0.08)
    A = np.array([-16.0])
    x = np.zeros((1, L, 1, 1))
    B = np.ones((1, L, 1, 1))
    C = np.ones((1, L, 1, 1))
    y, f = oracle.recurrence(x, dt, A, B, C, np.zeros(1), np.ones((1, 1, 1, 1)))
    assert np.all(np.isfinite(y))
    expect_last = math.exp(L * 0.08 * -16.0)
    assert float(f.reshape(())) == pytest.approx(expect_last, rel=1e-12, abs=0.0)
