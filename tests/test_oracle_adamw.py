"""Pins of the fp64 AdamW oracle against closed forms, a hand-derived worked
example and special cases, plus planted mistakes that each pin set catches.
No GPU."""
import math

import numpy as np
import pytest

from oracle import adamw_oracle as ora


def _first_step(step_fn):
    """Zero state, t = 1: the bias corrections cancel the (1 - beta)
    factors exactly, so the direction is g / (|g| + eps)."""
    rng = np.random.default_rng(0)
    g = rng.standard_normal(257) * 1e-2
    p0 = rng.standard_normal(257)
    p, m, v = step_fn(p0, g, np.zeros(257), np.zeros(257), 1e-3, 0.9, 0.95, 1e-8, 0.1, 1)
    want = p0 * (1 - 1e-3 * 0.1) - 1e-3 * g / (np.abs(g) + 1e-8)
    return np.allclose(p, want, rtol=0, atol=1e-15) and np.allclose(m, 0.1 * g, rtol=1e-15, atol=0)


def _constant_gradient(step_fn):
    """A constant gradient from zero state gives m_t = (1 - beta1^t) g, so
    the bias-corrected direction is g / (|g| + eps) at every step."""
    g = np.array([0.5, -2.0, 3e-3, -7.0])
    p = np.zeros(4)
    m = np.zeros(4)
    v = np.zeros(4)
    ok = True
    for t in range(1, 9):
        p_prev = p
        p, m, v = step_fn(p, g, m, v, 0.01, 0.8, 0.99, 0.0, 0.0, t)
        ok &= np.allclose(p - p_prev, -0.01 * np.sign(g), rtol=1e-12, atol=1e-15)
    return ok


def _unrolled_moments(step_fn):
    """m_t = (1 - b1) sum_k b1^(t-k) g_k and v_t = (1 - b2) sum_k b2^(t-k) g_k^2
    for an arbitrary gradient sequence; decay does not enter the moments."""
    rng = np.random.default_rng(1)
    gs = rng.standard_normal((6, 33))
    b1, b2 = 0.85, 0.97
    p = rng.standard_normal(33)
    m = np.zeros(33)
    v = np.zeros(33)
    for t in range(1, 7):
        p, m, v = step_fn(p, gs[t - 1], m, v, 0.05, b1, b2, 1e-8, 0.3, t)
    m_want = sum((1 - b1) * b1 ** (6 - k) * gs[k - 1] for k in range(1, 7))
    v_want = sum((1 - b2) * b2 ** (6 - k) * gs[k - 1] ** 2 for k in range(1, 7))
    return np.allclose(m, m_want, rtol=1e-13, atol=0) and np.allclose(v, v_want, rtol=1e-13, atol=0)


def _pure_decay(step_fn):
    """Zero gradient and state: the parameter only decays, (1 - lr wd)^t."""
    p0 = np.array([1.0, -3.0, 0.25])
    p, m, v = p0, np.zeros(3), np.zeros(3)
    for t in range(1, 6):
        p, m, v = step_fn(p, np.zeros(3), m, v, 0.1, 0.9, 0.999, 1e-8, 0.2, t)
    return np.allclose(p, p0 * 0.98 ** 5, rtol=1e-14, atol=0)


def _eps_outside_sqrt(step_fn):
    """eps is added to sqrt(vhat): at t = 1, g = 1e-10, eps = 1e-8 the
    direction is 1e-10 / (1e-10 + 1e-8) = 1/101."""
    p, _, _ = step_fn(np.zeros(1), np.array([1e-10]), np.zeros(1), np.zeros(1), 1.0, 0.9, 0.999, 1e-8, 0.0, 1)
    return abs(p[0] + 1.0 / 101.0) < 1e-15


def _worked_example(step_fn):
    """By hand, beta1 = 0.5, beta2 = 0.75, eps = 0, lr = 0.1, wd = 0.5,
    p0 = 2, g = 1 then 3:
      t = 1: m = 0.5, v = 0.25, mhat = vhat = 1, p1 = 2 * 0.95 - 0.1 = 1.8
      t = 2: m = 1.75, v = 2.4375, mhat = 7/3, vhat = 39/7,
             p2 = 1.8 * 0.95 - 0.1 * (7/3) / sqrt(39/7)."""
    p, m, v = step_fn(np.array([2.0]), np.array([1.0]), np.zeros(1), np.zeros(1), 0.1, 0.5, 0.75, 0.0, 0.5, 1)
    ok = abs(p[0] - 1.8) < 1e-15 and abs(m[0] - 0.5) < 1e-15 and abs(v[0] - 0.25) < 1e-15
    p, m, v = step_fn(p, np.array([3.0]), m, v, 0.1, 0.5, 0.75, 0.0, 0.5, 2)
    ok &= abs(m[0] - 1.75) < 1e-15 and abs(v[0] - 2.4375) < 1e-15
    return ok and abs(p[0] - (1.71 - 0.1 * (7 / 3) / math.sqrt(39 / 7))) < 1e-14


PINS = [_first_step, _constant_gradient, _unrolled_moments, _pure_decay, _eps_outside_sqrt, _worked_example]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__.strip("_") for p in PINS])
def test_adamw_oracle_pin(pin):
    assert pin(ora.adamw_step)


def test_adamw_step_counts_from_one():
    with pytest.raises(ValueError):
        ora.adamw_step(np.zeros(1), np.zeros(1), np.zeros(1), np.zeros(1), 0.1, 0.9, 0.99, 1e-8, 0.0, 0)


# planted mistakes: each must fail at least one pin
def _mut_no_bias_correction(p, g, m, v, lr, b1, b2, eps, wd, t):
    m2, v2 = ora.adamw_moments(g, m, v, b1, b2)
    return (1 - lr * wd) * p - lr * m2 / (np.sqrt(v2) + eps), m2, v2


def _mut_coupled_decay(p, g, m, v, lr, b1, b2, eps, wd, t):
    return ora.adamw_step(p, np.asarray(g) + wd * np.asarray(p), m, v, lr, b1, b2, eps, 0.0, t)


def _mut_eps_in_sqrt(p, g, m, v, lr, b1, b2, eps, wd, t):
    m2, v2 = ora.adamw_moments(g, m, v, b1, b2)
    mh, vh = m2 / (1 - b1 ** t), v2 / (1 - b2 ** t)
    return (1 - lr * wd) * p - lr * mh / np.sqrt(vh + eps), m2, v2


def _mut_swapped_corrections(p, g, m, v, lr, b1, b2, eps, wd, t):
    m2, v2 = ora.adamw_moments(g, m, v, b1, b2)
    mh, vh = m2 / (1 - b2 ** t), v2 / (1 - b1 ** t)
    return (1 - lr * wd) * p - lr * mh / (np.sqrt(vh) + eps), m2, v2


def _mut_decay_after_update(p, g, m, v, lr, b1, b2, eps, wd, t):
    p2, m2, v2 = ora.adamw_step(p, g, m, v, lr, b1, b2, eps, 0.0, t)
    return p2 * (1 - lr * wd), m2, v2


MUTANTS = [_mut_no_bias_correction, _mut_coupled_decay, _mut_eps_in_sqrt, _mut_swapped_corrections,
           _mut_decay_after_update]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__.strip("_") for m in MUTANTS])
def test_adamw_pins_catch_planted_mistake(mutant):
    assert not all(pin(mutant) for pin in PINS)
