"""Pins for the oracle's Mem-SGD top-k / rand-k step.

Source: "Sparsified SGD with Memory", Method (g_t = comp_k(m_t + eta*grad),
m_{t+1} = m_t + eta*grad - g_t, comp_k a k-contraction) and Key results
(0 < k <= d).  Each test fixes the oracle against something other than its
own code: hand-worked values, brute force over all subsets, exact invariants,
the k = d special case (plain SGD) and the contraction inequality.
"""
import itertools

import numpy as np
import pytest

import oracle
from oracle import steps
from tests.conftest import read_golden


def f32(xs):
    return np.array([float(x) for x in xs], np.float32)


def bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def test_hand_worked_two_steps():
    g = read_golden("memsgd_topk_hand.txt")
    eta = float(g["eta"][0])
    m = f32(g["mem0"])
    for s in ("step1", "step2"):
        vals, idx, m = oracle.ef_topk_unit(f32(g[s + ".grad"]), m, int(g[s + ".k"][0]), eta)
        assert idx.tolist() == [int(x) for x in g[s + ".idx"]]
        assert np.array_equal(bits(vals), bits(f32(g[s + ".vals"])))
        assert np.array_equal(bits(m), bits(f32(g[s + ".mem"])))


def test_residual_uses_two_fp32_roundings():
    """v = fl32(m + fl32(eta*g)): matches numpy's IEEE fp32 ops bit for bit and
    differs from a single rounding of the exact value on some inputs."""
    rng = np.random.default_rng(1)
    n = 4096
    g = rng.standard_normal(n).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32)
    eta = np.float32(0.1)
    vals, idx, m_new = oracle.ef_topk_unit(g, m, n, eta)  # k = n sends all of v
    expect = m + eta * g                                   # numpy fp32: two roundings
    assert np.array_equal(bits(vals), bits(expect))
    once = (m.astype(np.float64) + np.float64(eta) * g.astype(np.float64)).astype(np.float32)
    assert np.any(bits(once) != bits(expect)), "inputs do not separate the readings"


def brute_force_topk_set(v, k):
    """The unique size-k set S with: i in S, j not in S  =>  |v_i| > |v_j|, or
    |v_i| == |v_j| and i < j.  Found by checking every subset."""
    key = np.abs(v.astype(np.float64))
    n = len(v)
    found = []
    for S in itertools.combinations(range(n), k):
        rest = [j for j in range(n) if j not in S]
        if all(key[i] > key[j] or (key[i] == key[j] and i < j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    return list(found[0])


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_subsets_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 9))
    pool = np.array([-2, -1, -0.0, 0.0, 1, 2, 0.5, -0.5], np.float32)
    g = rng.choice(pool, n).astype(np.float32)
    m = rng.choice(pool, n).astype(np.float32)
    eta = np.float32(1.0)
    v = m + eta * g
    for k in range(1, n + 1):
        vals, idx, m_new = oracle.ef_topk_unit(g, m, k, eta)
        S = brute_force_topk_set(v, k)
        assert idx.tolist() == S
        assert np.array_equal(bits(vals), bits(v[S]))


@pytest.mark.parametrize("method", ["topk", "randk"])
def test_memory_invariant_bit_exact(method):
    """m_{t+1} + g_t == m_t + eta*grad: for every coordinate one of the two
    terms is +0, the other carries v's bits exactly."""
    rng = np.random.default_rng(7)
    n, k, eta = 5000, 123, np.float32(0.05)
    m = rng.standard_normal(n).astype(np.float32)
    for t in range(4):
        g = rng.standard_normal(n).astype(np.float32)
        v = m + eta * g
        if method == "topk":
            vals, idx, m_new = oracle.ef_topk_unit(g, m, k, eta)
        else:
            vals, idx, m_new = oracle.ef_randk_unit(g, m, k, eta, 9, 0, 0, t)
        dense = np.zeros(n, np.float32)
        dense[idx] = vals
        assert len(set(idx.tolist())) == k and np.all(np.diff(idx) > 0)
        assert np.array_equal(bits(m_new + dense), bits(v + np.float32(0)))
        assert np.all(bits(m_new[idx]) == 0)           # +0.0 on the sent set
        sel = np.zeros(n, bool)
        sel[idx] = True
        assert np.array_equal(bits(m_new[~sel]), bits(v[~sel]))
        m = m_new


@pytest.mark.parametrize("method", ["topk", "randk"])
def test_k_equals_d_is_plain_sgd(method):
    """comp_d is the identity: with m_0 = 0 every step sends fl(eta*grad) and
    the memory stays zero (Key results: 0 < k <= d)."""
    rng = np.random.default_rng(3)
    n, eta = 777, np.float32(0.05)
    m = np.zeros(n, np.float32)
    for t in range(3):
        g = rng.standard_normal(n).astype(np.float32)
        if method == "topk":
            vals, idx, m = oracle.ef_topk_unit(g, m, n, eta)
        else:
            vals, idx, m = oracle.ef_randk_unit(g, m, n, eta, 1, 0, 0, t)
        assert idx.tolist() == list(range(n))
        assert np.array_equal(bits(vals), bits(eta * g))
        assert not np.any(m)


def test_k_one_is_argmax_lowest_index():
    rng = np.random.default_rng(5)
    for _ in range(50):
        n = int(rng.integers(1, 300))
        g = rng.integers(-4, 5, n).astype(np.float32)     # many ties, both signs
        m = np.zeros(n, np.float32)
        vals, idx, _ = oracle.ef_topk_unit(g, m, 1, 1.0)
        assert idx[0] == int(np.argmax(np.abs(g)))        # argmax returns the first
        assert vals[0] == g[idx[0]]


@pytest.mark.parametrize("k", [1, 10, 100, 999])
def test_topk_is_a_k_contraction(k):
    """||v - g||^2 <= (1 - k/d) ||v||^2 (the k-contraction of the Method)."""
    rng = np.random.default_rng(k)
    n = 1000
    g = (rng.standard_normal(n) * rng.exponential(1, n)).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32)
    v = (m + np.float32(0.3) * g).astype(np.float64)
    vals, idx, m_new = oracle.ef_topk_unit(g, m, k, 0.3)
    lhs = float(np.sum(m_new.astype(np.float64) ** 2))
    assert lhs <= (1 - k / n) * float(np.sum(v * v)) * (1 + 1e-12)
    # top-k leaves the smallest residual of all size-k sets: dropping the
    # k largest |v| is optimal, so any other set does no better
    other = np.sort(np.abs(v))[: n - k]
    assert lhs == pytest.approx(float(np.sum(other ** 2)), rel=1e-12)


def test_dense_layer_sends_everything():
    rng = np.random.default_rng(11)
    g = rng.standard_normal(300).astype(np.float32)
    m = rng.standard_normal(300).astype(np.float32)
    pay, m_new = oracle.dense_unit(g, m, 0.05)
    assert np.array_equal(bits(pay), bits(m + np.float32(0.05) * g))
    assert np.all(bits(m_new) == 0)


def test_k_from_ppm_is_integer_floor():
    assert oracle.k_from_ppm(30522 * 768, 10000) == 234408
    assert oracle.k_from_ppm(768, 10000) == 7
    assert oracle.k_from_ppm(50, 10000) == 1          # floor 0 -> clamped to 1
    assert oracle.k_from_ppm(1 << 20, 1000) == 1048
    assert oracle.k_from_ppm(1728, 100000) == 172


def test_bad_k_is_rejected():
    g = np.zeros(10, np.float32)
    for k in (0, 11):
        with pytest.raises(ValueError):
            oracle.ef_topk_unit(g, g, k, 1.0)


def test_table_loop_matches_units_and_thread_count():
    rng = np.random.default_rng(2)
    layers = [dict(rows=30, cols=7, kind="topk"), dict(rows=50, cols=1, kind="dense"),
              dict(rows=4, cols=100, kind="topk")]
    W = 3
    N = sum(l["rows"] * l["cols"] for l in layers)
    grad = rng.standard_normal((W, N)).astype(np.float32)
    mem1 = rng.standard_normal((W, N)).astype(np.float32)
    mem2 = mem1.copy()
    a = steps.sparse_step(layers, grad, mem1, 0.05, [5, 0, 40], threads=1)
    b = steps.sparse_step(layers, grad, mem2, 0.05, [5, 0, 40], threads=4)
    assert np.array_equal(bits(mem1), bits(mem2))
    for key in a:
        if isinstance(a[key], tuple):
            assert np.array_equal(a[key][1], b[key][1])
            assert np.array_equal(bits(a[key][0]), bits(b[key][0]))
        else:
            assert np.array_equal(bits(a[key]), bits(b[key]))
