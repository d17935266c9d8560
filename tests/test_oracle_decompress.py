"""Pins for the oracle's decode side: the aggregate of W workers' payloads.

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Method / Key results: compressed payloads are combined across
data-parallel workers (all-reduce for PowerSGD, gather for sparse methods);
here the combination is an fp32 sum in worker order from +0.0, then a scale.
Pins: a single payload scatters to itself, disjoint payloads concatenate,
the sum order is the worker order (a case where order changes the result),
and the low-rank decode equals numpy's P Q^T.  The fused parameter update
("Sparsified SGD with Memory", Method: x_{t+1} = x_t - g_t) is pinned by a
hand-worked case and by x = 0 giving the negated aggregate; its step size
eta_t = 8 / (mu (a + t)) by values worked by hand.
"""
import numpy as np

import oracle
from oracle import steps


def test_single_payload_scatters():
    layers = [dict(rows=10, cols=1, kind="topk")]
    pay = {(0, 0): (np.array([1.5, -2.0], np.float32), np.array([3, 8], np.int32))}
    out = steps.decompress(layers, 1, pay, 1.0)
    expect = np.zeros(10, np.float32)
    expect[[3, 8]] = [1.5, -2.0]
    assert np.array_equal(out, expect)


def test_disjoint_payloads_concatenate():
    layers = [dict(rows=6, cols=1, kind="topk")]
    pay = {(0, 0): (np.array([1, 2], np.float32), np.array([0, 1], np.int32)),
           (1, 0): (np.array([3, 4], np.float32), np.array([2, 5], np.int32))}
    out = steps.decompress(layers, 2, pay, 0.5)
    assert out.tolist() == [0.5, 1.0, 1.5, 0.0, 0.0, 2.0]


def test_sum_is_in_worker_order():
    # (1e8 + -1e8) + 1 = 1, whereas (1e8 + 1) + -1e8 = 0 in fp32
    layers = [dict(rows=1, cols=1, kind="topk")]
    one = np.array([0], np.int32)
    vals = [1e8, -1e8, 1.0]
    pay = {(w, 0): (np.array([vals[w]], np.float32), one) for w in range(3)}
    assert steps.decompress(layers, 3, pay, 1.0)[0] == 1.0
    vals = [1e8, 1.0, -1e8]
    pay = {(w, 0): (np.array([vals[w]], np.float32), one) for w in range(3)}
    assert steps.decompress(layers, 3, pay, 1.0)[0] == 0.0


def test_scale_applies_after_sum():
    layers = [dict(rows=4, cols=1, kind="dense")]
    pay = {(w, 0): np.full(4, 1.0 + w, np.float32) for w in range(8)}
    out = steps.decompress(layers, 8, pay, 1.0 / 8)
    assert np.all(out == np.float32(36.0 / 8))


def test_lowrank_decode_is_p_qt():
    rng = np.random.default_rng(0)
    P = rng.standard_normal((7, 4)).astype(np.float32)
    Q = rng.standard_normal((5, 4)).astype(np.float32)
    layers = [dict(rows=7, cols=5, kind="powersgd")]
    out = steps.decompress(layers, 1, {(0, 0): (P, Q)}, 1.0, rank_per_layer=[3])
    expect = P[:, :3].astype(np.float64) @ Q[:, :3].astype(np.float64).T
    assert np.max(np.abs(out.reshape(7, 5) - expect)) < 1e-6


def test_topk_round_trip_recovers_sent_part():
    """decode(encode) + new memory == v: nothing is lost across the boundary."""
    rng = np.random.default_rng(3)
    n = 1000
    g = rng.standard_normal(n).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32)
    vals, idx, m_new = oracle.ef_topk_unit(g, m, 50, 0.05)
    layers = [dict(rows=n, cols=1, kind="topk")]
    out = steps.decompress(layers, 1, {(0, 0): (vals, idx)}, 1.0)
    v = m + np.float32(0.05) * g
    assert np.array_equal((out + m_new).view(np.uint32), (v + np.float32(0)).view(np.uint32))


def test_apply_hand_worked_case():
    # S = [0, 1.5, 0, -2 + 0.25]; x - 0.5 S = [1, 0.25, 1, 1.875]
    layers = [dict(rows=4, cols=1, kind="topk")]
    pay = {(0, 0): (np.array([1.5, -2.0], np.float32), np.array([1, 3], np.int32)),
           (1, 0): (np.array([0.25], np.float32), np.array([3], np.int32))}
    x = np.ones(4, np.float32)
    got = steps.apply_update(layers, 2, pay, 0.5, x)
    assert got.dtype == np.float32
    assert got.tolist() == [1.0, 0.25, 1.0, 1.875]
    assert x.tolist() == [1.0, 1.0, 1.0, 1.0]      # the input is not modified


def test_apply_from_zero_negates_the_aggregate():
    rng = np.random.default_rng(3)
    layers = [dict(rows=50, cols=1, kind="topk"), dict(rows=7, cols=1, kind="dense")]
    pay = {}
    for w in range(3):
        ix = np.sort(rng.choice(50, 9, replace=False)).astype(np.int32)
        pay[(w, 0)] = (rng.standard_normal(9).astype(np.float32), ix)
        pay[(w, 1)] = rng.standard_normal(7).astype(np.float32)
    agg = steps.decompress(layers, 3, pay, 0.25)
    got = steps.apply_update(layers, 3, pay, 0.25, np.zeros(57, np.float32))
    assert np.array_equal(got, -agg)
    assert not np.signbit(got[agg == 0]).any()     # 0 - (+0) is +0


def test_apply_rounds_once_per_element():
    # 1 - 2^-24 is exact in fp32; subtracting 2^-25 from 1 rounds to even (1.0)
    layers = [dict(rows=2, cols=1, kind="dense")]
    pay = {(0, 0): np.array([2.0 ** -24, 2.0 ** -25], np.float32)}
    got = steps.apply_update(layers, 1, pay, 1.0, np.ones(2, np.float32))
    assert got[0] == np.float32(1.0 - 2.0 ** -24)
    assert got[1] == np.float32(1.0)


def test_memsgd_eta_values():
    assert steps.memsgd_eta(0, 1.0, 8.0) == np.float32(1.0)
    assert steps.memsgd_eta(2, 0.5, 14.0) == np.float32(1.0)      # 8 / (0.5 * 16)
    assert steps.memsgd_eta(10, 4.0, 0.0) == np.float32(0.2)      # 8 / 40, rounded to fp32
    # decreasing in t, and mu * (a + t) * eta == 8 up to one fp32 rounding
    e = [steps.memsgd_eta(t, 0.1, 100.0) for t in range(50)]
    assert all(e[i] > e[i + 1] for i in range(49))
    for t in range(50):
        assert abs(float(e[t]) * 0.1 * (100.0 + t) - 8.0) <= 8.0 * 2.0 ** -24
