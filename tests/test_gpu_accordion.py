"""GPU parity of accordion_select against the CPU oracle.

Source: "Accordion: Adaptive Gradient Communication via Critical Learning
Regime Identification", Method: per-layer gradient-norm rate of change picks
l_low inside critical regimes and l_high outside.  Levels and the k / rank
they map to must be identical to the oracle's at every step; norms agree to
1e-9 relative (fp64 sums in different orders).
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.conftest import read_golden_rows
from tests.helpers import gce, host, need_gpu, torch

pytestmark = pytest.mark.gpu


def schedule():
    lv = {}
    for a, b, level in read_golden_rows("accordion_vgg19_schedule.txt"):
        for t in range(int(a), int(b) + 1):
            lv[t] = int(level)
    return lv


def run_accordion(layers, grads_fn, T, interval, thr, lo, hi):
    g = gce()
    t = g.Table(workloads.table_layers(layers))
    L = len(layers)
    prev = torch.empty(L, dtype=torch.float64, device="cuda")
    level = torch.empty(L, dtype=torch.int32, device="cuda")
    cur = torch.zeros(L, dtype=torch.float64, device="cuda")
    kr = torch.zeros(L, dtype=torch.int32, device="cuda")
    ws = t.workspace(1, "accordion")
    g.accordion_init(t, prev, level)
    st = osteps.AccordionState(L)
    out = []
    for s in range(T):
        grad = grads_fn(s)
        g.accordion_select(t, grad, s, interval, thr, lo, hi, prev, level, cur, kr, ws)
        expect = osteps.accordion_step(layers, host(grad), s, interval, thr, st, lo, hi)
        assert np.array_equal(host(level), st.level), s
        assert np.array_equal(host(kr), expect.astype(np.int32)), s
        if s % interval == 0:
            for l, lay in enumerate(layers):
                if lay["kind"] != "dense":
                    assert abs(float(cur[l]) - st.norms[l]) <= 1e-9 * st.norms[l], (s, l)
        out.append(host(level).copy())
    return out


def test_vgg19_schedule_powersgd_levels():
    """VGG-19 shapes, 200 steps, scale drops x0.1 at 60 and 140, checks every
    10 steps, threshold 0.5, l_low = rank 4, l_high = rank 2."""
    need_gpu()
    layers = workloads.vgg19("powersgd", 4)
    assert workloads.total_elements(layers) == 20081188
    exp = schedule()
    levels = run_accordion(layers, lambda s: workloads.gradients(layers, 1, 3, s,
                                                                 scale=workloads.vgg19_scale(s))[0],
                           200, 10, 0.5, 4, 2)
    for s, lv in enumerate(levels):
        for l, lay in enumerate(layers):
            if lay["kind"] != "dense":
                assert lv[l] == exp[s], (s, l)


def test_vgg19_topk_variant_levels():
    need_gpu()
    layers = workloads.vgg19("topk", 100000)
    run_accordion(layers, lambda s: workloads.gradients(layers, 1, 3, s,
                                                        scale=workloads.vgg19_scale(s))[0],
                  80, 10, 0.5, 100000, 10000)


def test_per_layer_drop_and_rise():
    need_gpu()
    layers = [dict(rows=100, cols=300, kind="powersgd", cap=4, sigma=1.0) for _ in range(10)]

    def grads(s):
        g = workloads.gradients(layers, 1, 7, 0)[0].clone()
        if s >= 40:
            g[3 * 30000:4 * 30000] *= 0.1
            g[7 * 30000:8 * 30000] *= 10.0
        return g

    run_accordion(layers, grads, 60, 10, 0.5, 4, 2)
