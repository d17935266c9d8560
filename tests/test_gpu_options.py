"""Per-table settings: two tables driven from two threads, each on its own
stream, with different settings of the same option, give the oracle's
results bit for bit, and each table's status shows only its own setting.

Source: "Sparsified SGD with Memory", Method (the error-feedback top-k and
rand-k updates).  The settings only move work: the top-k candidate margin
(a negative one forces the exact fallback on every layer) and the rand-k
look-ahead.  Neither may change a result.
"""
import threading

import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, need_gpu, payload_slice, layer_slice, torch

pytestmark = pytest.mark.gpu

LAYERS = [dict(rows=400000, cols=1, kind="topk", cap=4000, sigma=1.0),
          dict(rows=300, cols=7, kind="dense", cap=0),
          dict(rows=65536, cols=3, kind="topk", cap=20000, sigma=1.0)]
W, STEPS = 2, 3


def run_table(table, method, grads, out, errors):
    """STEPS steps on `table` on a stream of its own; keeps the last payload."""
    g = gce()
    try:
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            t = table
            mem = torch.zeros((W, t.N), device="cuda")
            vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
            idx = torch.zeros((W, max(4, t.vals_per_worker)), dtype=torch.int32, device="cuda")
            ws = t.workspace(W, method)
            status = 0
            for s in range(STEPS):
                if method == "topk":
                    g.ef_topk_step(t, W, grads[s], mem, workloads.ETA, None, vals, idx, ws)
                else:
                    g.ef_randk_step(t, W, grads[s], mem, workloads.ETA, None, 77, s, vals, idx, ws)
                status |= g.status(ws)
            stream.synchronize()
        out["vals"], out["idx"], out["mem"], out["status"] = host(vals), host(idx), host(mem), status
    except Exception as e:  # surfaced by the main thread
        errors.append(e)


def oracle_run(method, grads):
    hmem = np.zeros((W, grads[0].shape[1]), np.float32)
    exp = None
    for s in range(STEPS):
        exp = osteps.sparse_step(LAYERS, host(grads[s]), hmem, workloads.ETA,
                                 [l["cap"] for l in LAYERS], method=method, seed=77, step=s,
                                 threads=8)
    return exp, hmem


def check(table, got, exp, hmem):
    for (w, l), e in exp.items():
        lay = LAYERS[l]
        if lay["kind"] == "dense":
            n = lay["rows"] * lay["cols"]
            assert np.array_equal(bits(got["vals"][w, payload_slice(table, 0, l, n)]), bits(e))
        else:
            ev, ei = e
            sl = payload_slice(table, 0, l, lay["cap"])
            assert np.array_equal(got["idx"][w, sl], ei), (w, l)
            assert np.array_equal(bits(got["vals"][w, sl]), bits(ev)), (w, l)
    assert np.array_equal(bits(got["mem"]), bits(hmem))


@pytest.mark.parametrize("method, option, values", [
    ("topk", "bracket_sigma", (-60.0, 6.0)),
    ("randk", "randk_ahead", (0.0, 1.0))])
def test_two_tables_two_threads_own_settings(method, option, values):
    need_gpu()
    g = gce()
    layers = workloads.table_layers(LAYERS)
    if method == "randk":
        layers = [dict(l, kind="randk") if l["kind"] == "topk" else l for l in layers]
    tables = [g.Table(layers), g.Table(layers)]
    for t, v in zip(tables, values):
        t.set_option(option, v)
        assert t.option(option) == v
    grads = [workloads.gradients(LAYERS, W, 120, s) for s in range(STEPS)]
    torch.cuda.synchronize()
    outs, errors = [{}, {}], []
    threads = [threading.Thread(target=run_table, args=(t, method, grads, o, errors))
               for t, o in zip(tables, outs)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    exp, hmem = oracle_run(method, grads)
    for t, o in zip(tables, outs):
        check(t, o, exp, hmem)
    if method == "topk":
        # only the table with the negative margin took the exact fallback
        assert outs[0]["status"] & g.STATUS_FALLBACK
        assert not outs[1]["status"] & g.STATUS_FALLBACK


def test_table_option_follows_the_process_value_until_set():
    need_gpu()
    g = gce()
    t = g.Table(workloads.table_layers(LAYERS))
    assert t.option("bracket_sigma") == 6.0
    try:
        g.set_bracket_sigma(3.5)
        assert t.option("bracket_sigma") == 3.5
        t.set_option("bracket_sigma", 9.0)
        g.set_bracket_sigma(2.0)
        assert t.option("bracket_sigma") == 9.0
        t.reset_option("bracket_sigma")
        assert t.option("bracket_sigma") == 2.0
    finally:
        g.set_bracket_sigma(6.0)
    with pytest.raises(g.GceError):
        t.set_option("sign_ahead", 0.5)        # tiles are whole numbers
    with pytest.raises(g.GceError):
        t.set_option("randk_ahead", 2)
