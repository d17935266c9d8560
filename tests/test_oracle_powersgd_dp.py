"""Pins for the oracle's data-parallel PowerSGD step (or_powersgd_dp) and
the data-parallel uncompressed layer (or_dense_dp).

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Key results: PowerSGD is all-reduce compatible -- its payloads P
and Q are summed over the workers.  The steps are the standard single power
iteration with a shared warm start: P = sum_w M_w Q, orthonormalise P,
Q_w = M_w^T P, each worker's memory m_w = M_w - P Q_w^T, Q = mean_w Q_w.

Pins, none of which re-types the oracle's loops:
  - numpy: P spans the same columns as numpy's QR factor of sum_w M_w Q
    (signs fixed to a positive R diagonal), Q = mean_w M_w^T P, and P Q^T is
    the orthogonal projection of the mean M onto span(P);
  - one worker reduces to the single-worker oracle step (pinned elsewhere);
  - two identical workers give the single-worker result bit for bit (the sum
    doubles P exactly, and Gram-Schmidt is scale-free by powers of two);
  - the memories satisfy m_w + P Q_w^T = M_w, so sum_w m_w = W (M_mean -
    P Q^T) ; full rank empties every memory.
  - the dense layer: the mean of the residuals, memory to +0, and a sum
    whose worker order changes the rounding.
"""
import numpy as np
import pytest

import oracle


def residual(m, eta, g):
    return (m + np.float32(eta) * g).astype(np.float32)


def case(W, rows, cols, seed, r_max=4):
    rng = np.random.default_rng(seed)
    g = rng.standard_normal((W, rows, cols)).astype(np.float32)
    m = (0.3 * rng.standard_normal((W, rows, cols))).astype(np.float32)
    Q = rng.standard_normal((cols, r_max)).astype(np.float32)
    return g, m, Q


@pytest.mark.parametrize("W,r", [(3, 1), (4, 2), (5, 4)])
def test_against_numpy_qr_and_projection(W, r):
    g, m, Q = case(W, 40, 33, 10 * W + r)
    eta = 0.05
    P, Qn, mn = oracle.powersgd_dp_unit(g, m, Q, r, eta)
    M = residual(m, eta, g).astype(np.float64)
    Psum = sum(M[w] @ Q[:, :r].astype(np.float64) for w in range(W))
    Qf, R = np.linalg.qr(Psum)
    Qf = Qf * np.sign(np.diag(R))[None, :]
    assert np.allclose(P[:, :r], Qf, atol=1e-6)
    assert not P[:, r:].any()
    Pd = P[:, :r].astype(np.float64)
    Mbar = M.mean(axis=0)
    assert np.allclose(Qn[:, :r], Mbar.T @ Pd, rtol=1e-5, atol=1e-5)
    assert np.array_equal(Qn[:, r:], Q[:, r:])          # unused columns untouched
    proj = Pd @ Pd.T @ Mbar
    assert np.allclose(Pd @ Qn[:, :r].astype(np.float64).T, proj, atol=1e-5)
    for w in range(W):                                   # own error per worker
        Qw = M[w].T @ Pd
        assert np.allclose(mn[w], M[w] - Pd @ Qw.T, atol=1e-5)


def test_one_worker_is_the_single_worker_step():
    g, m, Q = case(1, 25, 17, 3)
    P1, Q1, m1 = oracle.powersgd_dp_unit(g, m, Q, 3, 0.05)
    P0, Q0, m0, _ = oracle.powersgd_unit(g[0], m[0], Q, 3, 0.05)
    assert np.array_equal(P1, P0)
    assert np.array_equal(Q1, Q0)
    assert np.array_equal(m1[0], m0)


def test_identical_workers_are_one_worker_bit_for_bit():
    g, m, Q = case(1, 30, 22, 4)
    g2, m2 = np.concatenate([g, g]), np.concatenate([m, m])
    P2, Q2, mn2 = oracle.powersgd_dp_unit(g2, m2, Q, 2, 0.05)
    P1, Q1, mn1, _ = oracle.powersgd_unit(g[0], m[0], Q, 2, 0.05)
    assert np.array_equal(P2, P1)
    assert np.array_equal(Q2, Q1)
    assert np.array_equal(mn2[0], mn1) and np.array_equal(mn2[1], mn1)


def test_full_rank_empties_every_memory():
    W, rows, cols = 3, 4, 9
    g, m, Q = case(W, rows, cols, 5)
    P, Qn, mn = oracle.powersgd_dp_unit(g, m, Q, rows, 0.05)
    M = residual(m, 0.05, g)
    assert np.abs(mn).max() <= 1e-5 * np.abs(M).max()
    # the decompressed mean is the mean residual
    assert np.allclose(P.astype(np.float64) @ Qn.astype(np.float64).T, M.mean(axis=0),
                       atol=1e-5)


def test_bad_arguments_are_rejected():
    g, m, Q = case(2, 5, 6, 6)
    with pytest.raises(Exception):
        oracle.powersgd_dp_unit(g, m, Q, 5, 0.05)   # r > r_max
    with pytest.raises(Exception):
        oracle.powersgd_dp_unit(g, m, Q, 0, 0.05)


def test_dense_dp_is_the_mean_and_clears_memory():
    W, n = 4, 101
    rng = np.random.default_rng(7)
    g = rng.standard_normal((W, n)).astype(np.float32)
    m = rng.standard_normal((W, n)).astype(np.float32)
    out, mn = oracle.dense_dp_unit(g, m, 0.5)
    v = residual(m, 0.5, g)
    s = np.zeros(n, np.float32)
    for w in range(W):
        s = (s + v[w]).astype(np.float32)
    assert np.array_equal(out, (s * np.float32(0.25)).astype(np.float32))
    assert not mn.any() and not np.signbit(mn).any()


def test_dense_dp_sums_in_worker_order():
    # (1e8 + 1) - 1e8 = 0 in fp32, (1e8 - 1e8) + 1 = 1
    g = np.zeros((3, 1), np.float32)
    for order, want in (([1e8, 1.0, -1e8], 0.0), ([1e8, -1e8, 1.0], 1.0)):
        m = np.array(order, np.float32).reshape(3, 1)
        out, _ = oracle.dense_dp_unit(g, m, 0.05)
        assert out[0] == np.float32(want) * np.float32(1.0 / 3.0)


def test_phases_compose_to_the_step():
    """The data-parallel step cut at its two all-reduces: per-worker P_w,
    their sum in worker order, Gram-Schmidt, per-worker Q_w and residual, the
    mean of Q_w -- bit for bit the one-call step (the cut an exchange between
    ranks makes), and P against numpy's QR of the summed P."""
    rng = np.random.default_rng(31)
    W, rows, cols, r = 3, 17, 23, 2
    g = rng.standard_normal((W, rows, cols)).astype(np.float32)
    m = rng.standard_normal((W, rows, cols)).astype(np.float32)
    Q = oracle.powersgd_init_q(cols, 4, 2, 0, 0)
    P_ref, Q_ref, m_ref = oracle.powersgd_dp_unit(g, m, Q, r, 0.05)
    Ms, Psum = [], np.zeros((rows, r))
    for w in range(W):
        M, Pw = oracle.powersgd_dp_p_unit(g[w], m[w], Q, r, 0.05)
        Ms.append(M)
        Psum = Psum + Pw
    Pd = oracle.mgs(Psum)
    q, rr = np.linalg.qr(Psum)
    assert np.allclose(Pd, q * np.sign(np.diag(rr)), atol=1e-12)
    Qsum = np.zeros((cols, r))
    for w in range(W):
        Qw, res = oracle.powersgd_dp_q_unit(Pd, Ms[w])
        Qsum = Qsum + Qw
        assert np.array_equal(res.view(np.uint32), m_ref[w].view(np.uint32))
    assert np.array_equal(Pd.astype(np.float32), P_ref[:, :r])
    assert np.array_equal((Qsum / W).astype(np.float32), Q_ref[:, :r])
