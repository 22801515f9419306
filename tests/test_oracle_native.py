"""Pins of the fp64 C++ oracle's matrix product, and the C++ oracle against the
numpy oracle (two independent writings of the same definitions).

The matrix product is the oracle's one primitive.  Its definition: C[i][j] is
the sum over ascending k of op(A)[i][k] op(B)[k][j], each term added with one
fused multiply-add, starting from +0.  An exact-rational replay of that
definition (every fma is exact a*b+c rounded once, which Fraction arithmetic
followed by one float() conversion reproduces) must match it bit for bit, at
sizes that cross every blocking boundary of the C++ loops.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import AdamWHParams, MuonHParams
from oracle import adamw as np_adamw
from oracle import muon as np_muon
from oracle import native


def fma_replay(a_row, b_col):
    """sum_k a_k b_k, ascending k, each term by one correctly rounded fma."""
    acc = 0.0
    for a, b in zip(a_row, b_col):
        acc = float(Fraction(a) * Fraction(b) + Fraction(acc))
    return acc


def _operands(rng, M, N, K, ta, tb):
    A = rng.standard_normal((K, M) if ta else (M, K))
    B = rng.standard_normal((N, K) if tb else (K, N))
    opA = A.T if ta else A
    opB = B.T if tb else B
    return A, B, opA, opB


@pytest.mark.parametrize("ta", [False, True])
@pytest.mark.parametrize("tb", [False, True])
def test_matmul_bitwise_definition_small(ta, tb):
    rng = np.random.default_rng(3 + 2 * ta + tb)
    for M, N, K in [(1, 1, 1), (5, 7, 3), (6, 16, 9), (7, 17, 33)]:
        A, B, opA, opB = _operands(rng, M, N, K, ta, tb)
        C = native.matmul(A, B, ta, tb)
        for i in range(M):
            for j in range(N):
                assert C[i, j] == fma_replay(opA[i, :], opB[:, j]), (M, N, K, i, j)


@pytest.mark.parametrize("ta", [False, True])
@pytest.mark.parametrize("tb", [False, True])
def test_matmul_bitwise_definition_across_blocks(ta, tb):
    # 101 rows cross the 96-row task block and the 6-row register tile, 530
    # columns the 512-column block and the 16-column tile, 300 terms the
    # 256-term K block.  Sampled entries include every block's corners.
    rng = np.random.default_rng(11 + 2 * ta + tb)
    M, N, K = 101, 530, 300
    A, B, opA, opB = _operands(rng, M, N, K, ta, tb)
    C = native.matmul(A, B, ta, tb)
    rows = sorted({0, 5, 6, 95, 96, 100} | set(rng.integers(0, M, 4).tolist()))
    cols = sorted({0, 15, 16, 511, 512, 529} | set(rng.integers(0, N, 4).tolist()))
    for i in rows:
        for j in cols:
            assert C[i, j] == fma_replay(opA[i, :], opB[:, j]), (i, j)


def test_matmul_against_numpy_and_edges():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((200, 700))
    B = rng.standard_normal((700, 300))
    C = native.matmul(A, B)
    ref = A @ B
    assert np.max(np.abs(C - ref)) <= 1e-13 * np.max(np.abs(ref))
    assert np.array_equal(native.matmul(np.zeros((3, 0)), np.zeros((0, 4))), np.zeros((3, 4)))
    assert native.matmul(np.zeros((0, 5)), np.zeros((5, 4))).shape == (0, 4)


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(6)
    W, G, buf = (rng.standard_normal((150, 610)) for _ in range(3))
    hp = MuonHParams()
    before = native.threads()
    try:
        native.set_threads(1)
        one = native.muon_step(W, G, buf, hp)
        native.set_threads(max(2, before))
        many = native.muon_step(W, G, buf, hp)
    finally:
        native.set_threads(before)
    for x, y in zip(one, many):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("shape", [(1, 1), (1, 9), (9, 1), (24, 40), (40, 24), (64, 64), (130, 300), (300, 130)])
@pytest.mark.parametrize("nesterov", [True, False])
def test_native_matches_numpy_oracle(shape, nesterov):
    rng = np.random.default_rng(sum(shape) + nesterov)
    W, G = rng.standard_normal(shape), rng.standard_normal(shape) * 1e-2
    buf = rng.standard_normal(shape) * 1e-3
    hp = MuonHParams(nesterov=nesterov)
    Wn, O, bn = native.muon_step(W, G, buf, hp)
    Wr, Or, br = np_muon.muon_step(W, G, buf, hp)
    # elementwise steps are the same IEEE operations in the same order
    assert np.array_equal(bn, br)
    # the Newton-Schulz products accumulate in different orders (numpy: BLAS)
    assert np.linalg.norm(O - Or) <= 1e-12 * np.linalg.norm(Or)
    assert np.max(np.abs(Wn - Wr)) <= 1e-13 * max(1.0, np.max(np.abs(Wr)))


def test_native_adamw_matches_numpy_oracle_bitwise():
    rng = np.random.default_rng(9)
    p, g = rng.standard_normal(1000), rng.standard_normal(1000) * 1e-3
    m, v = rng.standard_normal(1000) * 1e-4, np.abs(rng.standard_normal(1000)) * 1e-7
    for t in (1, 2, 7):
        a = native.adamw_step(p, g, m, v, t, AdamWHParams())
        b = np_adamw.adamw_step(p, g, m, v, t, AdamWHParams())
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_parts_and_list_entry_points_validate():
    with pytest.raises(ValueError):
        native.muon_step_parts(np.zeros((2, 2)), [], np.zeros((2, 2)), MuonHParams())
    with pytest.raises(ValueError):
        native.adamw_step(np.zeros(1), np.zeros(1), np.zeros(1), np.zeros(1), 0, AdamWHParams())
