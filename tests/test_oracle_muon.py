"""Pins of the fp64 Muon oracle against facts that do not come from the oracle.

Each test is chosen so that a plausible mistake in the oracle (a wrong
coefficient or sign, A = X^T X instead of X X^T, a missing normalisation, a
wrong iteration count, a transpose not undone, the scale on the wrong side,
weight decay not multiplied by lr, the plain-momentum form) fails at least one.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import MuonHParams

HP = MuonHParams()

# The same pins hold the oracle of record (fp64 C++) and the numpy writing.
IMPLS = {"cpp": oracle.native, "numpy": oracle.muon}


@pytest.fixture(params=sorted(IMPLS))
def impl(request):
    return IMPLS[request.param]


def p_fraction(s, steps=5):
    """Scalar quintic p(s) = a s + b s^3 + c s^5 composed ``steps`` times, exact rationals."""
    a, b, c = Fraction(34445, 10000), Fraction(-47750, 10000), Fraction(20315, 10000)
    s = Fraction(s)
    for _ in range(steps):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def p_float(s, steps=5):
    for _ in range(steps):
        s = 3.4445 * s - 4.7750 * s ** 3 + 2.0315 * s ** 5
    return s


def rng(seed):
    return np.random.default_rng(seed)


# --- worked scalar values of the five-fold quintic (exact rational arithmetic) ---

def test_quintic_worked_values():
    # p(1) = a + b + c = 0.701 exactly; five-fold values printed to 10 digits.
    assert p_fraction(1, 1) == Fraction(701, 1000)
    assert abs(float(p_fraction(1)) - 0.6964364095) < 1e-10
    assert abs(float(p_fraction(Fraction(1, 16))) - 1.0705244477) < 1e-10
    assert abs(p_float(2 ** -0.5) - 1.1081111157) < 1e-10
    assert abs(p_float(512 ** -0.5) - 0.8086068622) < 1e-10
    assert abs(p_float(1 / 64) - 0.9025257530) < 1e-10


# --- the singular-value closed form through an SVD (library routine) ---

@pytest.mark.parametrize("shape", [(24, 40), (40, 24), (17, 17), (1, 9), (9, 1), (64, 64), (33, 64)])
def test_newton_schulz_matches_svd_closed_form(shape, impl):
    g = rng(hash(shape) % 1000).standard_normal(shape)
    g += 3.0 * np.outer(rng(1).standard_normal(shape[0]), rng(2).standard_normal(shape[1]))
    ns = impl.newton_schulz(g, HP.a, HP.b, HP.c, 5, HP.eps)
    U, S, Vt = np.linalg.svd(g, full_matrices=False)
    norm = np.sqrt(np.sum(S ** 2))
    s0 = S / (norm + HP.eps)
    expect = (U * p_float(s0)) @ Vt
    assert ns.shape == g.shape
    assert np.linalg.norm(ns - expect) <= 1e-10 * max(1.0, np.linalg.norm(expect))


def test_newton_schulz_iteration_count_matters(impl):
    g = rng(5).standard_normal((8, 12))
    U, S, Vt = np.linalg.svd(g, full_matrices=False)
    s0 = S / (np.sqrt(np.sum(S ** 2)) + HP.eps)
    for k in (1, 3, 5, 7):
        ns = impl.newton_schulz(g, HP.a, HP.b, HP.c, k, HP.eps)
        assert np.allclose(ns, (U * p_float(s0, k)) @ Vt, rtol=0, atol=1e-12)


# --- closed forms of the whole update ---

def test_rank_one_update_closed_form(impl):
    # G = sigma u v^T, unit u, v, zero momentum: M = (1 - beta^2) G, so
    # O = p^5(s0) u v^T * scale with s0 = |M| / (|M| + eps), and
    # W_new = W (1 - lr wd) - lr O.
    m, n, sigma = 20, 30, 0.37
    u = rng(7).standard_normal(m); u /= np.linalg.norm(u)
    v = rng(8).standard_normal(n); v /= np.linalg.norm(v)
    G = sigma * np.outer(u, v)
    W = rng(9).standard_normal((m, n))
    Wn, O, buf = impl.muon_step(W, G, np.zeros((m, n)), HP)
    normM = (1 - HP.beta ** 2) * sigma
    s0 = normM / (normM + HP.eps)
    expect_O = p_float(s0) * np.outer(u, v)
    assert np.allclose(O, expect_O, rtol=0, atol=1e-13)
    assert np.allclose(Wn, W * (1 - 0.02 * 0.01) - 0.02 * expect_O, rtol=0, atol=1e-13)
    assert np.allclose(buf, 0.05 * G, rtol=0, atol=1e-16)


def test_orthonormal_rows_and_tall_scale(impl):
    # Wide G with orthonormal rows (256 x 512): every singular value of X_0 is
    # 1/(sqrt(256)+eps') ~ 1/16, so O = p^5(1/16) G_dir.
    q, _ = np.linalg.qr(rng(11).standard_normal((512, 256)))   # 512 x 256, orthonormal columns
    wide = q.T.copy()                                            # 256 x 512, orthonormal rows
    O, _ = impl.muon_update(wide / (1 - HP.beta ** 2), np.zeros_like(wide), HP)
    s0 = 16.0 / (16.0 + HP.eps)  # ||M||_F = sqrt(256) = 16
    assert np.allclose(O, p_float(s0 / 16.0) * wide, rtol=0, atol=1e-12)
    # Tall G (512 x 256) with orthonormal columns: transposed internally, then
    # scaled by sqrt(512/256) = sqrt(2) on the way out.
    O_t, _ = impl.muon_update(q / (1 - HP.beta ** 2), np.zeros_like(q), HP)
    assert np.allclose(O_t, np.sqrt(2.0) * p_float(s0 / 16.0) * q, rtol=0, atol=1e-12)
    assert abs(p_float(1 / 16) - 1.0705244477) < 1e-9


def test_shape_scale_values(impl):
    assert impl.shape_scale(256, 512) == 1.0
    assert impl.shape_scale(512, 512) == 1.0
    assert abs(impl.shape_scale(5504, 2048) - 1.6393596310755) < 1e-12
    assert abs(impl.shape_scale(27648, 5120) - 2.3237900077244) < 1e-12
    assert impl.shape_scale(16384, 64) == 16.0


# --- invariants ---

def test_transpose_equivariance(impl):
    G = rng(12).standard_normal((30, 50))
    a = impl.newton_schulz(G, HP.a, HP.b, HP.c, 5, HP.eps)
    b = impl.newton_schulz(G.T, HP.a, HP.b, HP.c, 5, HP.eps)
    assert np.allclose(a, b.T, rtol=0, atol=1e-13)


def test_orthogonal_equivariance(impl):
    G = rng(13).standard_normal((12, 20))
    Q, _ = np.linalg.qr(rng(14).standard_normal((12, 12)))
    P, _ = np.linalg.qr(rng(15).standard_normal((20, 20)))
    lhs = impl.newton_schulz(Q @ G @ P, HP.a, HP.b, HP.c, 5, HP.eps)
    rhs = Q @ impl.newton_schulz(G, HP.a, HP.b, HP.c, 5, HP.eps) @ P
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_positive_scale_invariance_up_to_eps(impl):
    G = rng(16).standard_normal((10, 14))
    a = impl.newton_schulz(G, HP.a, HP.b, HP.c, 5, 0.0)
    b = impl.newton_schulz(1e3 * G, HP.a, HP.b, HP.c, 5, 0.0)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_frobenius_normalise_unit_norm(impl):
    T = rng(17).standard_normal((7, 9))
    X = impl.frobenius_normalise(T, 0.0)
    assert abs(np.sqrt(np.sum(X * X)) - 1.0) < 1e-14


def test_constant_gradient_momentum_closed_form(impl):
    # EMA form from zero: buf_k = (1 - beta^k) G, M_k = ((1 - beta) + beta (1 - beta^k)) G.
    G = rng(18).standard_normal((5, 6))
    buf = np.zeros_like(G)
    for k in range(1, 4):
        M, buf = impl.nesterov_momentum(G, buf, 0.95, True)
        assert np.allclose(buf, (1 - 0.95 ** k) * G, rtol=0, atol=1e-15)
        assert np.allclose(M, (0.05 + 0.95 * (1 - 0.95 ** k)) * G, rtol=0, atol=1e-15)
    assert np.allclose(buf, 0.142625 * G, rtol=0, atol=1e-15)
    assert np.allclose(M, 0.18549375 * G, rtol=0, atol=1e-15)
    # plain momentum returns the buffer itself
    M2, b2 = impl.nesterov_momentum(G, np.zeros_like(G), 0.95, False)
    assert np.array_equal(M2, b2)


def test_zero_gradient_is_pure_decay(impl):
    W = rng(19).standard_normal((6, 4))
    Wn, O, buf = impl.muon_step(W, np.zeros((6, 4)), np.zeros((6, 4)), HP)
    assert np.all(O == 0.0)
    assert np.allclose(Wn, W * (1.0 - 0.02 * 0.01), rtol=0, atol=0)


def test_update_singular_values_in_quintic_range(impl):
    # p^5 maps [0.05, 1] into [0.6818, 1.1344]: singular values of O/scale of a
    # well-conditioned G stay in that band.
    G = rng(20).standard_normal((16, 64)) + 2.0 * np.eye(16, 64)
    X0 = impl.frobenius_normalise(G, HP.eps)
    s0 = np.linalg.svd(X0, compute_uv=False)
    assert s0.min() > 0.05
    O, _ = impl.muon_update(G / (1 - HP.beta ** 2), np.zeros_like(G), HP)
    s = np.linalg.svd(O, compute_uv=False)
    assert s.min() >= 0.6818 - 1e-4 and s.max() <= 1.1344 + 1e-4


def test_empty_matrix(impl):
    O, buf = impl.muon_update(np.zeros((0, 5)), np.zeros((0, 5)), HP)
    assert O.shape == (0, 5) and buf.shape == (0, 5)


def test_golden_regression_fixture(impl):
    """The oracle's own output for a tiny seeded case, stored by
    tests/golden/make_golden.py (which calls only oracle/ and synth/)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_step.json")
    with open(path) as f:
        gold = json.load(f)
    G = np.array(gold["G"]); W = np.array(gold["W"]); buf = np.array(gold["buf"])
    Wn, O, bn = impl.muon_step(W, G, buf, HP)
    assert np.allclose(O, np.array(gold["O"]), rtol=0, atol=1e-14)
    assert np.allclose(Wn, np.array(gold["W_new"]), rtol=0, atol=1e-15)
