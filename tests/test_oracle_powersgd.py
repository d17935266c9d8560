"""Pins for the oracle's PowerSGD step with error feedback.

The pages name PowerSGD and its ranks (Accordion, Method and Key results;
On the Utility of Gradient Compression, Method and Key results) but do not
print its steps; the oracle takes the standard single power-iteration step
with a reused Q: P = M Q, orthonormalise P, Q' = M^T P, decompress P Q'^T,
memory = M - P Q'^T.  The pins below are linear-algebra facts of that step:
full rank reconstructs M, a rank-1 M is recovered at r = 1, P^T P = I, the
r = 1 closed form, the QR special case (numpy's Householder QR with a
positive diagonal), and the memory invariant.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import read_golden_rows


def rel(a, b):
    return np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-300)


def residual(m, g, eta):
    return (np.asarray(m, np.float32) + np.float32(eta) * np.asarray(g, np.float32)).astype(np.float64)


@pytest.mark.parametrize("shape", [(3, 7), (4, 4), (7, 3), (2, 9)])
def test_full_rank_reconstructs(shape):
    rows, cols = shape
    r = min(rows, cols)
    rng = np.random.default_rng(rows * 10 + cols)
    g = rng.standard_normal(shape).astype(np.float32)
    m = rng.standard_normal(shape).astype(np.float32)
    Q = rng.standard_normal((cols, 4)).astype(np.float32)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(g, m, Q, r, 0.5)
    M = residual(m, g, 0.5)
    assert rel(Mhat, M) < 1e-6          # stored in fp32
    assert np.max(np.abs(m_new)) < 1e-5 * np.max(np.abs(M))


def test_rank_one_recovered_at_r1():
    rng = np.random.default_rng(0)
    u = rng.standard_normal(40)
    w = rng.standard_normal(25)
    M = np.outer(u, w).astype(np.float32)
    Q = rng.standard_normal((25, 2)).astype(np.float32)   # q^T w != 0 a.s.
    P, Qn, m_new, Mhat = oracle.powersgd_unit(np.zeros_like(M), M, Q, 1, 1.0)
    assert rel(Mhat, M.astype(np.float64)) < 1e-6
    assert np.max(np.abs(m_new)) < 1e-5 * np.max(np.abs(M))
    # P is the unit vector along u, up to sign
    p = P[:, 0].astype(np.float64)
    assert abs(abs(p @ u) / np.linalg.norm(u) - 1) < 1e-6


@pytest.mark.parametrize("r", [1, 2, 3, 4])
def test_p_is_orthonormal(r):
    rng = np.random.default_rng(r)
    g = rng.standard_normal((64, 90)).astype(np.float32)
    m = np.zeros((64, 90), np.float32)
    Q = oracle.powersgd_init_q(90, 4, 1, 0, 0)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(g, m, Q, r, 1.0)
    Pr = P[:, :r].astype(np.float64)
    assert np.max(np.abs(Pr.T @ Pr - np.eye(r))) < 1e-6   # fp32 storage of an fp64 result
    assert not np.any(P[:, r:])


@pytest.mark.parametrize("r", [1, 2, 4])
def test_p_matches_qr_factor_and_q_matches_mtp(r):
    """Gram-Schmidt on P = MQ equals the thin-QR Q factor with a positive R
    diagonal; Q' equals M^T P; Mhat equals P Q'^T (numpy as independent check)."""
    rng = np.random.default_rng(10 + r)
    rows, cols = 33, 57
    g = rng.standard_normal((rows, cols)).astype(np.float32)
    m = rng.standard_normal((rows, cols)).astype(np.float32)
    Q = rng.uniform(-1, 1, (cols, 4)).astype(np.float32)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(g, m, Q, r, 0.25)
    M = residual(m, g, 0.25)
    Pq, R = np.linalg.qr(M @ Q[:, :r].astype(np.float64))
    Pq = Pq * np.sign(np.diag(R))
    assert np.max(np.abs(P[:, :r] - Pq)) < 1e-6
    assert rel(Qn[:, :r], M.T @ Pq) < 1e-6
    assert rel(Mhat, Pq @ (M.T @ Pq).T) < 1e-6
    assert np.array_equal(Qn[:, r:], Q[:, r:])          # unused columns untouched


def test_r1_closed_form():
    rng = np.random.default_rng(4)
    rows, cols = 20, 30
    g = rng.standard_normal((rows, cols)).astype(np.float32)
    m = np.zeros((rows, cols), np.float32)
    Q = rng.standard_normal((cols, 1)).astype(np.float32)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(g, m, Q, 1, 1.0)
    M = g.astype(np.float64)
    q = Q[:, 0].astype(np.float64)
    Mq = M @ q
    expect = np.outer(Mq, Mq @ M) / (Mq @ Mq)
    assert rel(Mhat, expect) < 1e-6


def test_memory_plus_decompressed_is_m():
    rng = np.random.default_rng(8)
    g = rng.standard_normal((48, 31)).astype(np.float32)
    m = rng.standard_normal((48, 31)).astype(np.float32)
    Q = oracle.powersgd_init_q(31, 2, 3, 0, 0)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(g, m, Q, 2, 0.05)
    M = residual(m, g, 0.05)
    assert np.max(np.abs(m_new.astype(np.float64) + Mhat - M)) < 1e-6 * np.max(np.abs(M))


def test_warm_start_converges_to_top_subspace():
    """Repeated steps on a fixed matrix with no memory feed (power iteration):
    the warm-started Q drives P Q^T to the best rank-r approximation."""
    rng = np.random.default_rng(9)
    U, _ = np.linalg.qr(rng.standard_normal((30, 30)))
    V, _ = np.linalg.qr(rng.standard_normal((20, 20)))
    s = np.array([10, 5, 1, 0.5] + [0.1] * 16)
    M = (U[:, :20] * s) @ V.T
    Q = oracle.powersgd_init_q(20, 2, 0, 0, 0)
    zero = np.zeros((30, 20), np.float32)
    for _ in range(30):
        P, Q, _, Mhat = oracle.powersgd_unit(zero, M.astype(np.float32), Q, 2, 1.0)
    best = (U[:, :2] * s[:2]) @ V[:, :2].T
    assert rel(Mhat, best) < 1e-4


def test_zero_matrix_gives_zero_columns():
    z = np.zeros((5, 6), np.float32)
    Q = oracle.powersgd_init_q(6, 2, 0, 0, 0)
    P, Qn, m_new, Mhat = oracle.powersgd_unit(z, z, Q, 2, 1.0)
    assert not np.any(P) and not np.any(Qn[:, :2]) and not np.any(Mhat) and not np.any(m_new)


def test_q_entry_hand_worked_values():
    """The [-1, 1) mapping of a generator output, against values worked by
    hand on the published SplitMix64 outputs and the two extreme words
    (tests/golden/powersgd_init_q_hand.txt)."""
    from fractions import Fraction
    rows = read_golden_rows("powersgd_init_q_hand.txt")
    assert len(rows) == 5
    for h, t, x in rows:
        h, t = int(h), int(t)
        assert h >> 40 == t
        assert Fraction(oracle.q_entry(h).item()) == Fraction(x)


def test_init_q_range_and_counter_order():
    Q = oracle.powersgd_init_q(1000, 4, 123, 0, 5)
    assert Q.min() >= -1.0 and Q.max() < 1.0
    assert abs(float(Q.mean())) < 0.05
    # entry (c, j) comes from output c*r_max + j + 1 of the stream-1 base
    base = oracle.randk_base(123, 1, 0, 5, 0)
    for c, j in [(0, 0), (0, 3), (3, 2), (999, 3)]:
        h = oracle.splitmix64_output(base, c * 4 + j + 1)
        assert Q[c, j] == oracle.q_entry(h)
    # and the base of seed 0, worker 0, layer 0 is the hand-worked case B
    golden = {r[0]: [int(x) for x in r[1:]] for r in read_golden_rows("randk_base_hand.txt")}
    Q0 = oracle.powersgd_init_q(2, 2, 0, 0, 0)
    assert Q0[1, 0] == oracle.q_entry(oracle.splitmix64_output(golden["B"][-1], 3))


def test_bad_rank_is_rejected():
    z = np.zeros((3, 5), np.float32)
    Q = np.zeros((5, 4), np.float32)
    for r in (0, 4):
        with pytest.raises(ValueError):
            oracle.powersgd_unit(z, z, Q, r, 1.0)
