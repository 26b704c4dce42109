"""Pins of the AdamW oracle (oracle/optim.py) against closed forms of Adam that
do not depend on the oracle's own code: the first step moves every parameter by
lr * g / (|g| + eps); a constant gradient keeps the bias-corrected moments at g
and g^2, so every step moves by the same amount; a zero gradient leaves only the
decoupled decay (1 - lr wd)^t; beta = 0 turns the moments into g and g^2."""
from __future__ import annotations

import numpy as np

import oracle

LR, B1, B2, EPS = 1e-3, 0.9, 0.999, 1e-8


def _f32(x):
    return float(np.float32(x))


def test_first_step_moves_by_lr_times_sign():
    rng = np.random.default_rng(0)
    g = rng.standard_normal(1000) * 1e-2
    p0 = rng.standard_normal(1000)
    p, m, v = oracle.adamw_step(p0, g, np.zeros(1000), np.zeros(1000), 1, LR, B1, B2, EPS, 0.0)
    lr, eps = _f32(LR), _f32(EPS)
    np.testing.assert_allclose(p, p0 - lr * g / (np.abs(g) + eps), rtol=0, atol=1e-15)
    np.testing.assert_allclose(m, (1 - _f32(B1)) * g, rtol=1e-15)
    np.testing.assert_allclose(v, (1 - _f32(B2)) * g * g, rtol=1e-15)


def test_constant_gradient_moves_by_the_same_amount_every_step():
    g = np.array([0.3, -2.0, 1e-3, -5e-7])
    p0 = np.array([1.0, -1.0, 0.5, 0.25])
    p, m, v = p0.copy(), np.zeros(4), np.zeros(4)
    for t in range(1, 21):
        p, m, v = oracle.adamw_step(p, g, m, v, t, LR, B1, B2, EPS, 0.0)
        step = _f32(LR) * g / (np.abs(g) + _f32(EPS))
        np.testing.assert_allclose(p, p0 - t * step, rtol=0, atol=1e-12)


def test_zero_gradient_leaves_the_decoupled_decay():
    p0 = np.array([1.0, -3.0, 0.125])
    wd = 0.01
    p, m, v = p0.copy(), np.zeros(3), np.zeros(3)
    for t in range(1, 11):
        p, m, v = oracle.adamw_step(p, np.zeros(3), m, v, t, LR, B1, B2, EPS, wd)
    np.testing.assert_allclose(p, p0 * (1 - _f32(LR) * _f32(wd)) ** 10, rtol=1e-14)
    assert np.all(m == 0) and np.all(v == 0)


def test_zero_betas_give_the_raw_moments():
    g = np.array([0.5, -0.25, 4.0])
    m_prev, v_prev = np.array([9.0, 9.0, 9.0]), np.array([7.0, 7.0, 7.0])
    p, m, v = oracle.adamw_step(np.zeros(3), g, m_prev, v_prev, 5, LR, 0.0, 0.0, EPS, 0.0)
    assert np.array_equal(m, g) and np.array_equal(v, g * g)
    np.testing.assert_allclose(p, -_f32(LR) * g / (np.abs(g) + _f32(EPS)), rtol=1e-15)
