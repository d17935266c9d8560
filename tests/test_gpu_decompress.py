"""GPU parity of decompress_accumulate against the CPU oracle (bit-exact for
sparse and dense payloads, 1e-6 relative for low-rank ones).

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Method / Key results: the workers' compressed payloads are
combined across data-parallel workers; here W replicas in one GPU's HBM are
summed in worker order from +0.0, then scaled.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, need_gpu, torch

pytestmark = pytest.mark.gpu


def sparse_payloads(layers, W, seed, collide=True):
    """Random sorted unique index lists per (w, l) with k = cap entries."""
    rng = np.random.default_rng(seed)
    pay = {}
    for w in range(W):
        for l, lay in enumerate(layers):
            n = lay["rows"] * lay["cols"]
            if lay["kind"] == "dense":
                pay[(w, l)] = rng.standard_normal(n).astype(np.float32)
                continue
            k = lay["cap"]
            if collide:
                ix = np.sort(rng.choice(n, k, replace=False)).astype(np.int32)
            else:   # disjoint across workers
                ix = np.sort(rng.choice(np.arange(w, n, W), k, replace=False)).astype(np.int32)
            pay[(w, l)] = (rng.standard_normal(k).astype(np.float32) * 10.0 ** rng.uniform(-3, 3, k)
                           .astype(np.float32), ix)
    return pay


def upload(table, layers, W, pay):
    vals = np.zeros((W, max(table.vals_per_worker, 4)), np.float32)
    idx = np.zeros((W, max(table.vals_per_worker, 4)), np.int32)
    for (w, l), p in pay.items():
        o = table.info[l]["val_offset"]
        if layers[l]["kind"] == "dense":
            vals[w, o:o + len(p)] = p
        else:
            vals[w, o:o + len(p[0])] = p[0]
            idx[w, o:o + len(p[1])] = p[1]
    return torch.from_numpy(vals).cuda(), torch.from_numpy(idx).cuda()


@pytest.mark.parametrize("W,scale", [(1, 1.0), (3, 1.0), (8, 0.125), (8, 1.0)])
def test_sparse_and_dense_bit_exact(W, scale):
    need_gpu()
    g = gce()
    layers = [dict(rows=4096, cols=1, kind="topk", cap=100),
              dict(rows=10000, cols=7, kind="topk", cap=5000),     # many decode tiles
              dict(rows=333, cols=1, kind="dense", cap=0),
              dict(rows=1, cols=1, kind="topk", cap=1),
              dict(rows=300001, cols=1, kind="topk", cap=30000)]
    t = g.Table(layers)
    pay = sparse_payloads(layers, W, 11 + W)
    vals, idx = upload(t, layers, W, pay)
    out = torch.full((t.N,), float("nan"), device="cuda")
    ws = t.workspace(W, "decompress")
    g.decompress_accumulate(t, W, vals, idx, None, None, None, scale, out, ws)
    expect = osteps.decompress(layers, W, pay, scale)
    assert np.array_equal(bits(host(out)), bits(expect))


@pytest.mark.parametrize("W", [32, 33])
def test_many_workers_same_indices(W):
    """Every worker sends the same index set (every index collides W ways)
    with values spread over six decades, so any change of the worker order
    changes the rounding; 32 workers take the staged path, 33 the one-worker-
    at-a-time path.  Odd layer sizes put later layers off 16-byte alignment."""
    need_gpu()
    g = gce()
    layers = [dict(rows=12289, cols=1, kind="topk", cap=3001),
              dict(rows=4095, cols=3, kind="topk", cap=6000),
              dict(rows=9, cols=1, kind="topk", cap=9)]
    t = g.Table(layers)
    rng = np.random.default_rng(40 + W)
    pay = {}
    for l, lay in enumerate(layers):
        n = lay["rows"] * lay["cols"]
        ix = np.sort(rng.choice(n, lay["cap"], replace=False)).astype(np.int32)
        for w in range(W):
            v = (rng.standard_normal(lay["cap"]) * 10.0 ** rng.uniform(-3, 3, lay["cap"]))
            pay[(w, l)] = (v.astype(np.float32), ix)
    vals, idx = upload(t, layers, W, pay)
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate(t, W, vals, idx, None, None, None, 0.5, out, t.workspace(W, "decompress"))
    expect = osteps.decompress(layers, W, pay, 0.5)
    assert np.array_equal(bits(host(out)), bits(expect))


def test_dense_payloads_stage_in_several_chunks():
    """k = n / 2 over 8 workers: about 16 K entries per 4096-element decode
    tile, several times the shared-memory staging area."""
    need_gpu()
    g = gce()
    layers = [dict(rows=40000, cols=1, kind="topk", cap=20000),
              dict(rows=4096, cols=2, kind="topk", cap=8192)]
    t = g.Table(layers)
    pay = sparse_payloads(layers, 8, 77)
    vals, idx = upload(t, layers, 8, pay)
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate(t, 8, vals, idx, None, None, None, 1.0, out, t.workspace(8, "decompress"))
    expect = osteps.decompress(layers, 8, pay, 1.0)
    assert np.array_equal(bits(host(out)), bits(expect))


def test_worker_order_decides_rounding():
    need_gpu()
    g = gce()
    layers = [dict(rows=10, cols=1, kind="topk", cap=1)]
    t = g.Table(layers)
    for order, want in (([1e8, -1e8, 1.0], 1.0), ([1e8, 1.0, -1e8], 0.0)):
        pay = {(w, 0): (np.array([order[w]], np.float32), np.array([4], np.int32)) for w in range(3)}
        vals, idx = upload(t, layers, 3, pay)
        out = torch.zeros(t.N, device="cuda")
        g.decompress_accumulate(t, 3, vals, idx, None, None, None, 1.0, out, t.workspace(3, "decompress"))
        assert host(out)[4] == want


def test_k_per_layer_reads_prefix():
    need_gpu()
    g = gce()
    layers = [dict(rows=50000, cols=1, kind="topk", cap=5000)]
    t = g.Table(layers)
    pay = sparse_payloads(layers, 2, 5)
    vals, idx = upload(t, layers, 2, pay)
    k = torch.tensor([1234], dtype=torch.int32, device="cuda")
    out = torch.zeros(t.N, device="cuda")
    g.decompress_accumulate(t, 2, vals, idx, k, None, None, 1.0, out, t.workspace(2, "decompress"))
    expect = osteps.decompress(layers, 2, pay, 1.0, k_per_layer=[1234])
    assert np.array_equal(bits(host(out)), bits(expect))


def test_topk_step_round_trip_bert_w8():
    """Encode with ef_topk_step, decode with decompress_accumulate: the
    aggregate equals the oracle's sum of the same payloads bit for bit."""
    need_gpu()
    g = gce()
    layers = workloads.bert_base_topk()
    W = 8
    t = g.Table(workloads.table_layers(layers))
    grad = workloads.gradients(layers, W, 4, 0)
    mem = torch.zeros_like(grad)
    vals = torch.zeros((W, t.vals_per_worker), device="cuda")
    idx = torch.zeros((W, t.vals_per_worker), dtype=torch.int32, device="cuda")
    g.ef_topk_step(t, W, grad, mem, workloads.ETA, None, vals, idx, t.workspace(W, "topk"))
    del grad, mem
    out = torch.zeros(t.N, device="cuda")
    g.decompress_accumulate(t, W, vals, idx, None, None, None, 1.0, out, t.workspace(W, "decompress"))
    hv, hi = host(vals), host(idx)
    pay = {}
    for w in range(W):
        for l, lay in enumerate(layers):
            o, k = t.info[l]["val_offset"], lay["cap"]
            pay[(w, l)] = (hv[w, o:o + k], hi[w, o:o + k])
    expect = osteps.decompress(layers, W, pay, 1.0)
    assert np.array_equal(bits(host(out)), bits(expect))


APPLY_LAYERS = [dict(rows=4096, cols=1, kind="topk", cap=100),
                dict(rows=10000, cols=7, kind="topk", cap=5000),
                dict(rows=333, cols=1, kind="dense", cap=0),
                dict(rows=1, cols=1, kind="topk", cap=1),
                dict(rows=300001, cols=1, kind="topk", cap=30000)]


@pytest.mark.parametrize("W,scale", [(1, 1.0), (8, 0.125), (33, 0.5)])
def test_apply_sparse_and_dense_bit_exact(W, scale):
    """decompress_apply: x - fl(scale * S) in place, bit for bit the oracle's
    parameter update ("Sparsified SGD with Memory", Method)."""
    need_gpu()
    g = gce()
    layers = APPLY_LAYERS
    t = g.Table(layers)
    pay = sparse_payloads(layers, W, 90 + W)
    vals, idx = upload(t, layers, W, pay)
    x0 = np.random.default_rng(W).standard_normal(t.N).astype(np.float32)
    x = torch.from_numpy(x0.copy()).cuda()
    g.decompress_apply(t, W, vals, idx, None, None, None, scale, x, t.workspace(W, "decompress"))
    expect = osteps.apply_update(layers, W, pay, scale, x0)
    assert np.array_equal(bits(host(x)), bits(expect))


@pytest.mark.parametrize("W", [2, 9])
def test_apply_lowrank_matches_decode(W):
    """PowerSGD payloads: the fused update equals x minus this library's own
    decode bit for bit (2 workers: the tiled low-rank kernel; 9: the
    element-wise one), and the oracle's update within the low-rank decode's
    1e-6 relative bound."""
    need_gpu()
    g = gce()
    layers = [dict(rows=96, cols=1000, kind="powersgd", cap=4),
              dict(rows=37, cols=13, kind="powersgd", cap=2),
              dict(rows=50, cols=1, kind="dense", cap=0)]
    t = g.Table(layers)
    rng = np.random.default_rng(500 + W)
    P = rng.standard_normal((W, max(4, t.P_per_worker))).astype(np.float32)
    Q = rng.standard_normal((W, max(4, t.Q_per_worker))).astype(np.float32)
    vals = rng.standard_normal((W, max(4, t.vals_per_worker))).astype(np.float32)
    pay = {}
    for w in range(W):
        for l, lay in enumerate(layers):
            o = t.info[l]
            if lay["kind"] == "dense":
                pay[(w, l)] = vals[w, o["val_offset"]:o["val_offset"] + o["n"]]
            else:
                c = lay["cap"]
                pay[(w, l)] = (P[w, o["p_offset"]:o["p_offset"] + lay["rows"] * c].reshape(-1, c),
                               Q[w, o["q_offset"]:o["q_offset"] + lay["cols"] * c].reshape(-1, c))
    dP, dQ, dv = (torch.from_numpy(a).cuda() for a in (P, Q, vals))
    x0 = rng.standard_normal(t.N).astype(np.float32)
    x = torch.from_numpy(x0.copy()).cuda()
    ws = t.workspace(W, "decompress")
    g.decompress_apply(t, W, dv, None, None, dP, dQ, 0.5, x, ws)
    dec = torch.zeros(t.N, device="cuda")
    g.decompress_accumulate(t, W, dv, None, None, dP, dQ, 0.5, dec, ws)
    assert torch.equal(x.view(torch.int32), (torch.from_numpy(x0).cuda() - dec).view(torch.int32))
    ranks = [l["cap"] for l in layers]
    agg = osteps.decompress(layers, W, pay, 0.5, rank_per_layer=ranks)
    expect = osteps.apply_update(layers, W, pay, 0.5, x0, rank_per_layer=ranks)
    err = np.abs(host(x).astype(np.float64) - expect) - np.abs(np.spacing(expect))
    assert float(err.max()) <= 1e-6 * float(np.abs(agg).max())


def test_apply_reads_the_k_prefix():
    """With per-layer k, the fused update adds only the first k entries of
    every payload, like the decode."""
    need_gpu()
    g = gce()
    layers = [dict(rows=50000, cols=1, kind="topk", cap=5000), dict(rows=33, cols=1, kind="dense", cap=0)]
    t = g.Table(layers)
    pay = sparse_payloads(layers, 3, 6)
    vals, idx = upload(t, layers, 3, pay)
    k = torch.tensor([777, 0], dtype=torch.int32, device="cuda")
    x0 = np.random.default_rng(8).standard_normal(t.N).astype(np.float32)
    x = torch.from_numpy(x0.copy()).cuda()
    g.decompress_apply(t, 3, vals, idx, k, None, None, 1.0 / 3.0, x, t.workspace(3, "decompress"))
    expect = osteps.apply_update(layers, 3, pay, 1.0 / 3.0, x0, k_per_layer=[777, 0])
    assert np.array_equal(bits(host(x)), bits(expect))
