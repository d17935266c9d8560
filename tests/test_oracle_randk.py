"""Pins for the oracle's rand-k selection and its counter-based generator.

Source: "Sparsified SGD with Memory", Abstract / Motivation / Research
questions: rand-k keeps k randomly chosen coordinates; Method: comp_k is a
k-contraction, so the chosen values are sent unscaled.  The generator is
SplitMix64 (Steele, Lea, Flood 2014), pinned by its published outputs; the
way (seed, stream, worker, layer, step) are folded into its state is this
library's reading, pinned by a chain worked by hand whose first fold is a
published output.
"""
import math

import numpy as np
import pytest

import oracle
from tests.conftest import read_golden_rows


def test_splitmix64_published_outputs():
    for row in read_golden_rows("splitmix64_published.txt"):
        state, *outs = (int(x) for x in row)
        assert [oracle.splitmix64_output(state, j) for j in (1, 2, 3)] == outs


def test_base_fold_chain_hand_worked():
    """The state of (seed, stream, worker, layer, step) against a chain worked
    by hand (tests/golden/randk_base_hand.txt): the first fold of each case is
    a published SplitMix64 output, which fixes the seed as the state and
    stream + 1 as the counter; the later folds fix the field order and the
    +1 offsets."""
    pub = {int(r[0]): [int(x) for x in r[1:]] for r in read_golden_rows("splitmix64_published.txt")}
    cases = read_golden_rows("randk_base_hand.txt")
    assert [c[0] for c in cases] == ["A", "B"]
    for name, *vals in cases:
        seed, stream, worker, layer, step, f1, f2, f3, f4 = (int(v) for v in vals)
        assert f1 == pub[seed][stream]          # output stream+1 of the seed state
        assert oracle.splitmix64_output(seed, stream + 1) == f1
        assert oracle.splitmix64_output(f1, worker + 1) == f2
        assert oracle.splitmix64_output(f2, layer + 1) == f3
        assert oracle.splitmix64_output(f3, step + 1) == f4
        assert oracle.randk_base(seed, stream, worker, layer, step) == f4, name


def test_key_is_high_half_of_output():
    base = oracle.randk_base(5, 0, 1, 2, 3)
    for i in (0, 1, 17, 123456):
        assert oracle.randk_key(base, i) == oracle.splitmix64_output(base, i + 1) >> 32


def test_base_depends_on_every_field():
    ref = oracle.randk_base(1, 0, 2, 3, 4)
    for args in [(2, 0, 2, 3, 4), (1, 1, 2, 3, 4), (1, 0, 3, 3, 4), (1, 0, 2, 4, 4),
                 (1, 0, 2, 3, 5)]:
        assert oracle.randk_base(*args) != ref


@pytest.mark.parametrize("seed", range(10))
def test_chosen_set_is_k_smallest_keys(seed):
    n, k = int(50 + 7 * seed), int(1 + 3 * seed)
    rng = np.random.default_rng(seed)
    g = rng.standard_normal(n).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32)
    vals, idx, m_new = oracle.ef_randk_unit(g, m, k, 0.5, 42 + seed, 1, 2, 3)
    base = oracle.randk_base(42 + seed, 0, 1, 2, 3)
    keys = [(oracle.randk_key(base, i), i) for i in range(n)]
    expect = sorted(i for _, i in sorted(keys)[:k])
    assert idx.tolist() == expect
    v = m + np.float32(0.5) * g
    assert np.array_equal(vals.view(np.uint32), v[idx].view(np.uint32))   # unscaled


def test_inclusion_is_uniform_and_unbiased():
    """Over S independent seeds every coordinate is kept with rate k/n (5 sigma)
    and the sent vector has mean (k/n) v."""
    n, k, S = 64, 8, 20000
    g = np.linspace(-1, 1, n).astype(np.float32)
    m = np.zeros(n, np.float32)
    counts = np.zeros(n)
    total = np.zeros(n)
    for s in range(S):
        vals, idx, _ = oracle.ef_randk_unit(g, m, k, 1.0, s, 0, 0, 0)
        assert len(idx) == k
        counts[idx] += 1
        total[idx] += vals
    p = k / n
    sigma = math.sqrt(S * p * (1 - p))
    assert np.all(np.abs(counts - S * p) < 5 * sigma)
    # mean of g_t: E[g_i] = p * v_i, within 5 sigma of the estimator
    sd = np.abs(g) * math.sqrt(p * (1 - p) / S)
    assert np.all(np.abs(total / S - p * g) <= 5 * sd + 1e-12)
    # chi-square of counts against uniform, 63 dof: 99.9999% quantile ~ 130
    chi2 = float(np.sum((counts - S * p) ** 2 / (S * p)))
    assert chi2 < 130


def test_steps_draw_independent_sets():
    n, k = 1000, 100
    g = np.ones(n, np.float32)
    m = np.zeros(n, np.float32)
    a = set(oracle.ef_randk_unit(g, m, k, 1.0, 7, 0, 0, 0)[1].tolist())
    b = set(oracle.ef_randk_unit(g, m, k, 1.0, 7, 0, 0, 1)[1].tolist())
    c = set(oracle.ef_randk_unit(g, m, k, 1.0, 7, 1, 0, 0)[1].tolist())
    # two independent uniform 100-subsets of 1000 share ~10 elements
    assert len(a & b) < 40 and len(a & c) < 40


def test_randk_contraction_in_expectation():
    """E||v - g||^2 = (1 - k/d) ||v||^2 for unscaled rand-k."""
    n, k, S = 200, 20, 3000
    rng = np.random.default_rng(0)
    v = rng.standard_normal(n).astype(np.float32)
    zero = np.zeros(n, np.float32)
    acc = 0.0
    for s in range(S):
        _, _, m_new = oracle.ef_randk_unit(v, zero, k, 1.0, s, 0, 0, 0)
        acc += float(np.sum(m_new.astype(np.float64) ** 2))
    vv = float(np.sum(v.astype(np.float64) ** 2))
    assert acc / S == pytest.approx((1 - k / n) * vv, rel=0.02)
