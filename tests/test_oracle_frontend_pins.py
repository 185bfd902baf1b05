"""The front-end oracle against pins that do not restate it: library routines
(scipy's logistic function, numpy's vector norm), exact special values and
invariants; and planted mistakes against the same pins (CPU)."""
import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle.kda_frontend import BETA_IS_LOGIT, GATE_IN_KERNEL, QK_L2NORM

ALL = QK_L2NORM | GATE_IN_KERNEL | BETA_IS_LOGIT
rng = np.random.default_rng(11)
T, H = 7, 3


def draw():
    return (rng.standard_normal((T, H, 128)), rng.standard_normal((T, H, 128)),
            rng.standard_normal((T, H, 128)), rng.standard_normal((T, H)),
            0.5 * rng.standard_normal(H), 0.5 * rng.standard_normal((H, 128)))


def pin_beta_is_logistic(f):
    q, k, a, b, A_log, dt = draw()
    _, _, _, beta = f(q, k, a, b, A_log, dt, -5.0, 1e-6, ALL)
    return np.allclose(beta, expit(b), rtol=1e-14, atol=0)


def pin_gate_half_at_minus_bias(f):
    # a = -dt_bias: the logistic argument is exactly 0, so g = lower_bound / 2
    q, k, _, b, A_log, dt = draw()
    a = np.broadcast_to(-dt[None], (T, H, 128)).copy()
    _, _, g, _ = f(q, k, a, b, A_log, dt, -3.0, 1e-6, ALL)
    return np.all(g == -1.5)


def pin_gate_unit_rate_is_logistic(f):
    # A_log = 0 (rate 1), dt_bias = 0: g = lower_bound * logistic(a)
    q, k, a, b, _, _ = draw()
    _, _, g, _ = f(q, k, a, b, np.zeros(H), np.zeros((H, 128)), -5.0, 1e-6, ALL)
    return np.allclose(g, -5.0 * expit(a), rtol=1e-14, atol=0)


def pin_gate_rate_is_exp_of_A_log(f):
    # A_log = log 2 doubles the argument
    q, k, a, b, _, dt = draw()
    _, _, g, _ = f(q, k, a, b, np.full(H, np.log(2.0)), dt, -4.0, 1e-6, ALL)
    return np.allclose(g, -4.0 * expit(2.0 * (a + dt[None])), rtol=1e-13, atol=0)


def pin_gate_range_and_monotone(f):
    q, k, a, b, A_log, dt = draw()
    lb = -2.5
    _, _, g1, _ = f(q, k, a, b, A_log, dt, lb, 1e-6, ALL)
    _, _, g2, _ = f(q, k, a + 0.25, b, A_log, dt, lb, 1e-6, ALL)
    return bool(np.all(g1 > lb) and np.all(g1 < 0) and np.all(g2 < g1))


def pin_l2norm_matches_numpy_norm(f):
    # eps = 0: unit rows along the input direction
    q, k, a, b, A_log, dt = draw()
    qh, kh, _, _ = f(q, k, a, b, A_log, dt, -5.0, 0.0, ALL)
    ok_q = np.allclose(qh, q / np.linalg.norm(q, axis=-1, keepdims=True), rtol=1e-14, atol=1e-16)
    ok_k = np.allclose(kh, k / np.linalg.norm(k, axis=-1, keepdims=True), rtol=1e-14, atol=1e-16)
    return ok_q and ok_k


def pin_l2norm_scale_invariant_and_zero_safe(f):
    q, k, a, b, A_log, dt = draw()
    _, k1, _, _ = f(q, k, a, b, A_log, dt, -5.0, 0.0, ALL)
    _, k2, _, _ = f(q, 37.0 * k, a, b, A_log, dt, -5.0, 0.0, ALL)
    z = k.copy()
    z[0, 0] = 0.0
    _, kz, _, _ = f(q, z, a, b, A_log, dt, -5.0, 1e-6, ALL)
    return np.allclose(k1, k2, rtol=1e-13, atol=1e-16) and np.all(kz[0, 0] == 0.0)


def pin_switches_pass_inputs_through(f):
    q, k, a, b, A_log, dt = draw()
    out = f(q, k, a, b, A_log, dt, -5.0, 1e-6, 0)
    return all(np.array_equal(x, y) for x, y in zip(out, (q, k, a, b)))


PINS = [pin_beta_is_logistic, pin_gate_half_at_minus_bias, pin_gate_unit_rate_is_logistic,
        pin_gate_rate_is_exp_of_A_log, pin_gate_range_and_monotone, pin_l2norm_matches_numpy_norm,
        pin_l2norm_scale_invariant_and_zero_safe, pin_switches_pass_inputs_through]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_frontend_oracle_meets_pin(pin):
    assert pin(oracle.frontend_f64)


MUTATIONS = {1: "dt_bias subtracted", 2: "A_log used as the rate", 3: "logistic of -x",
             4: "norm without the square root", 5: "beta logit not squashed"}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_planted_frontend_mistake_is_caught(mutation):
    f = lambda *a: oracle.frontend_f64(*a, mutation=mutation)
    assert not all(p(f) for p in PINS), MUTATIONS[mutation]
