"""Pins for the oracle's Accordion detector.

Source: "Accordion: Adaptive Gradient Communication via Critical Learning
Regime Identification", Method: the rate of change of each layer's gradient
norm marks critical regimes; inside one the low-compression level l_low is
used, outside it l_high; Key results: the norm's rate of change is the
signal.  The 0.5 threshold and the 10-step interval are the VGG-19 workload's
parameters.  Pins: the scripted schedule (hand-derived golden), per-layer
independence, a rise, an exact tie, zero norms, and the norm itself against
numpy's fp64 norm.
"""
import numpy as np
import pytest

import oracle
from oracle import steps
from tests.conftest import read_golden_rows

LOW, HIGH = 0, 1


def expected_schedule():
    lv = {}
    for a, b, level in read_golden_rows("accordion_vgg19_schedule.txt"):
        for t in range(int(a), int(b) + 1):
            lv[t] = int(level)
    return lv


def small_vgg_like():
    # a few layers of VGG-19 shapes plus an uncompressed 1-D layer
    return [dict(rows=64, cols=27, kind="powersgd"), dict(rows=64, cols=576, kind="powersgd"),
            dict(rows=128, cols=1, kind="dense"), dict(rows=128, cols=1152, kind="powersgd"),
            dict(rows=100, cols=512, kind="powersgd")]


def scale_at(t):
    return 1.0 if t < 60 else (0.1 if t < 140 else 0.01)


def test_scripted_schedule():
    layers = small_vgg_like()
    offs, N = steps.layer_offsets(layers)
    st = steps.AccordionState(len(layers))
    expect = expected_schedule()
    rng = np.random.default_rng(0)
    for t in range(200):
        grad = np.empty(N, np.float32)
        for l, lay in enumerate(layers):
            n = lay["rows"] * lay["cols"]
            sig = scale_at(t) / np.sqrt(lay["cols"])
            grad[offs[l]:offs[l] + n] = (rng.standard_normal(n) * sig).astype(np.float32)
        out = steps.accordion_step(layers, grad, t, 10, 0.5, st, 4, 2)
        for l, lay in enumerate(layers):
            if lay["kind"] == "dense":
                assert out[l] == 0
                continue
            assert st.level[l] == expect[t], (t, l)
            assert out[l] == (4 if expect[t] == LOW else 2)


def test_topk_variant_levels_are_fractions():
    layers = [dict(rows=1000, cols=1, kind="topk"), dict(rows=64, cols=27, kind="topk")]
    st = steps.AccordionState(2)
    g = np.ones(1000 + 1728, np.float32)
    out = steps.accordion_step(layers, g, 0, 10, 0.5, st, 100000, 10000)
    assert out.tolist() == [100, 172]          # l_low = 10 % at the first check
    out = steps.accordion_step(layers, g, 10, 10, 0.5, st, 100000, 10000)
    assert out.tolist() == [10, 17]            # unchanged norm -> l_high = 1 %


def test_only_dropped_layers_switch():
    L = 10
    layers = [dict(rows=50, cols=20, kind="powersgd") for _ in range(L)]
    st = steps.AccordionState(L)
    rng = np.random.default_rng(1)
    base = rng.standard_normal(L * 1000).astype(np.float32)
    levels = {}
    for t in range(0, 80, 10):
        g = base.copy()
        if t >= 40:
            for l in (3, 7):
                g[l * 1000:(l + 1) * 1000] *= np.float32(0.1)
        steps.accordion_step(layers, g, t, 10, 0.5, st, 4, 2)
        levels[t] = st.level.copy()
    assert np.all(levels[0] == LOW)
    for t in (10, 20, 30, 50, 60, 70):
        assert np.all(levels[t] == HIGH), t
    assert [l for l in range(L) if levels[40][l] == LOW] == [3, 7]


def test_decision_rule_edges():
    d = oracle.accordion_decide
    assert d(-1.0, 3.0, 0.5) == LOW            # no earlier check
    assert d(1.0, 10.0, 0.5) == LOW            # rise x10: rel 9
    assert d(1.0, 0.5, 0.5) == LOW             # exact tie rel == 0.5 (>=)
    assert d(1.0, 1.5, 0.5) == LOW
    assert d(1.0, 0.5000001, 0.5) == HIGH
    assert d(1.0, 1.4999999, 0.5) == HIGH
    assert d(0.0, 0.0, 0.5) == HIGH            # both zero: no change
    assert d(0.0, 1e-30, 0.5) == LOW           # from zero: infinite change
    assert d(2.0, 0.0, 0.5) == LOW             # to zero: rel 1


def test_non_check_steps_keep_level():
    layers = [dict(rows=10, cols=10, kind="powersgd")]
    st = steps.AccordionState(1)
    g = np.ones(100, np.float32)
    steps.accordion_step(layers, g, 0, 10, 0.5, st, 4, 2)
    for t in range(1, 10):
        out = steps.accordion_step(layers, g * 100, t, 10, 0.5, st, 4, 2)
        assert out[0] == 4 and st.prev_norm[0] == pytest.approx(10.0)


def test_norm_matches_numpy():
    rng = np.random.default_rng(2)
    for n in (1, 7, 1000, 123457):
        g = (rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 3, n)).astype(np.float32)
        assert oracle.layer_norm(g) == pytest.approx(np.linalg.norm(g.astype(np.float64)),
                                                     rel=1e-13)
