"""Device-side checks and determinism of every step.

Non-finite inputs: the steps require finite gradients and memory; a NaN or
an infinity in the residual m + eta*grad sets GCE_STATUS_NONFINITE in the
workspace status word (read by gce_status), and a clean step leaves it clear.
The planted value is an ordinary input -- no fault, no invalid access.

Determinism: every reduction runs in a fixed order, so three runs of the same
step from the same inputs give the same bits (a race would show as a
difference between runs).
"""
import pytest

from gradient_compression_error_b200 import workloads
from tests.helpers import gce, need_gpu, torch

pytestmark = pytest.mark.gpu

LAYERS = {
    "topk": [dict(rows=300, cols=400, kind="topk", cap=1200, sigma=1.0),
             dict(rows=20000, cols=1, kind="topk", cap=200, sigma=1.0),
             dict(rows=70, cols=1, kind="dense", cap=0, sigma=1.0)],
    "randk": [dict(rows=300, cols=400, kind="randk", cap=1200, sigma=1.0),
              dict(rows=70, cols=1, kind="dense", cap=0, sigma=1.0)],
    "sign": [dict(rows=300, cols=400, kind="sign", cap=0, sigma=1.0),
             dict(rows=70, cols=1, kind="dense", cap=0, sigma=1.0)],
    "powersgd": [dict(rows=128, cols=576, kind="powersgd", cap=2, sigma=0.05),
                 dict(rows=70, cols=1, kind="dense", cap=0, sigma=1.0)],
    "powersgd_dp": [dict(rows=128, cols=576, kind="powersgd", cap=2, sigma=0.05),
                    dict(rows=70, cols=1, kind="dense", cap=0, sigma=1.0)],
}


def run_step(g, method, layers, W, grad, steps=1):
    """Run `steps` steps from zero memory; returns (status, output tensors)."""
    t = g.Table(workloads.table_layers(layers))
    mem = torch.zeros((W, t.N), device="cuda")
    ws = t.workspace(W, method)
    vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
    idx = torch.zeros((W, max(4, t.vals_per_worker)), dtype=torch.int32, device="cuda")
    P = torch.zeros((W, max(4, t.P_per_worker)), device="cuda")
    Q = torch.zeros((W, max(4, t.Q_per_worker)), device="cuda")
    if method in ("powersgd", "powersgd_dp"):
        g.powersgd_init_q(t, W, 3, Q)
    for s in range(steps):
        if method == "topk":
            g.ef_topk_step(t, W, grad, mem, 0.05, None, vals, idx, ws)
        elif method == "randk":
            g.ef_randk_step(t, W, grad, mem, 0.05, None, 11, s, vals, idx, ws)
        elif method == "sign":
            g.ef_sign_step(t, W, grad, mem, 0.05, vals, ws)
        elif method == "powersgd":
            g.powersgd_step(t, W, grad, mem, 0.05, None, P, Q, vals, None, ws)
        else:
            g.powersgd_dp_step(t, W, grad, mem, 0.05, None, P[0], Q[0], vals[0], ws)
    return g.status(ws), (mem, vals, idx, P, Q)


@pytest.mark.parametrize("method", sorted(LAYERS))
@pytest.mark.parametrize("where,value", [(0, float("nan")), (1, float("inf")),
                                         (-1, float("-inf"))])
def test_nonfinite_residual_is_flagged(method, where, value):
    """A NaN or infinity in one gradient element -- in the first compressed
    layer, its second element, or the last (dense) layer -- sets the bit; the
    same step on clean inputs does not."""
    need_gpu()
    g = gce()
    layers = LAYERS[method]
    W = 2
    grad = workloads.gradients(layers, W, 900, 0)
    clean, _ = run_step(g, method, layers, W, grad)
    assert not clean & g.STATUS_NONFINITE
    bad = grad.clone()
    bad[1, where] = value
    st, _ = run_step(g, method, layers, W, bad)
    assert st & g.STATUS_NONFINITE


@pytest.mark.parametrize("method", sorted(LAYERS))
def test_three_runs_give_the_same_bits(method):
    need_gpu()
    g = gce()
    layers = LAYERS[method]
    W = 3
    grad = workloads.gradients(layers, W, 901, 0)
    outs = [run_step(g, method, layers, W, grad, steps=3)[1] for _ in range(3)]
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), method
