"""Pins of the fp64 AdamW oracle: closed forms that do not come from the oracle."""

import json
import os

import numpy as np
import pytest

import oracle
from oracle import AdamWHParams

HP = AdamWHParams()

# The same pins hold the oracle of record (fp64 C++) and the numpy writing.
IMPLS = {"cpp": oracle.native, "numpy": oracle.adamw}


@pytest.fixture(params=sorted(IMPLS))
def impl(request):
    return IMPLS[request.param]


def test_first_step_from_zero_state_is_sign_like(impl):
    # t = 1, m = v = 0: m_hat = g, v_hat = g^2, so p <- p (1 - lr wd) - lr g / (|g| + eps).
    r = np.random.default_rng(1)
    p, g = r.standard_normal(64), r.standard_normal(64) * 1e-3
    pn, m, v = impl.adamw_step(p, g, np.zeros(64), np.zeros(64), 1, HP)
    assert np.allclose(pn, p * (1 - 0.02 * 0.01) - 0.02 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-15)
    assert np.allclose(m, 0.1 * g, rtol=1e-15, atol=0)
    assert np.allclose(v, 0.05 * g * g, rtol=1e-14, atol=0)


def test_constant_gradient_bias_correction_exact(impl):
    # With a constant g from zero state, m_t = (1 - beta1^t) g, so m_hat = g at
    # every t, and likewise v_hat = g^2: every step is the t = 1 step.
    r = np.random.default_rng(2)
    p0, g = r.standard_normal(32), r.standard_normal(32) * 1e-3
    p, m, v = p0.copy(), np.zeros(32), np.zeros(32)
    expect = p0.copy()
    for t in range(1, 6):
        p, m, v = impl.adamw_step(p, g, m, v, t, HP)
        expect = expect * (1 - 0.02 * 0.01) - 0.02 * g / (np.abs(g) + 1e-8)
        assert np.allclose(m, (1 - 0.9 ** t) * g, rtol=1e-13, atol=0)
        assert np.allclose(p, expect, rtol=1e-12, atol=0)


def test_zero_gradient_is_pure_decay(impl):
    p = np.linspace(-1, 1, 9)
    pn, m, v = impl.adamw_step(p, np.zeros(9), np.zeros(9), np.zeros(9), 1, HP)
    assert np.array_equal(pn, p * (1 - 0.02 * 0.01))
    assert np.all(m == 0) and np.all(v == 0)


def test_three_steps_against_unrolled_sums(impl):
    # Moments as closed sums: m_t = (1-b1) sum_k b1^(t-k) g_k, v_t = (1-b2) sum_k b2^(t-k) g_k^2.
    g = [0.3, -0.7, 0.2]
    p = 0.5
    b1, b2, lr, wd, eps = 0.9, 0.95, 0.02, 0.01, 1e-8
    expect = p
    for t in range(1, 4):
        mt = (1 - b1) * sum(b1 ** (t - k) * g[k - 1] for k in range(1, t + 1))
        vt = (1 - b2) * sum(b2 ** (t - k) * g[k - 1] ** 2 for k in range(1, t + 1))
        expect = expect * (1 - lr * wd) - lr * (mt / (1 - b1 ** t)) / (np.sqrt(vt / (1 - b2 ** t)) + eps)
    pp, m, v = np.array([p]), np.zeros(1), np.zeros(1)
    for t in range(1, 4):
        pp, m, v = impl.adamw_step(pp, np.array([g[t - 1]]), m, v, t, HP)
    assert abs(pp[0] - expect) < 1e-15


def test_step_count_starts_at_one(impl):
    with pytest.raises(ValueError):
        impl.adamw_step(np.zeros(1), np.zeros(1), np.zeros(1), np.zeros(1), 0, HP)


def test_golden_regression_fixture(impl):
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_adamw.json")
    with open(path) as f:
        gold = json.load(f)
    p, m, v = impl.adamw_step(np.array(gold["p"]), np.array(gold["g"]), np.array(gold["m"]),
                         np.array(gold["v"]), gold["t"], HP)
    assert np.allclose(p, gold["p_new"], rtol=0, atol=1e-16)
    assert np.allclose(m, gold["m_new"], rtol=0, atol=1e-18)
    assert np.allclose(v, gold["v_new"], rtol=0, atol=1e-20)
