"""GPU parity of ef_randk_step against the CPU oracle (bit-exact).

Source: "Sparsified SGD with Memory", Abstract / Method: rand-k keeps k
random coordinates under the same error-feedback update; both sides draw
the coordinates from SplitMix64 keyed by (seed, worker, layer, step), each
implemented from the generator's published definition.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, layer_slice, need_gpu, payload_slice, torch

pytestmark = pytest.mark.gpu


def run_randk(layers, W, T, seed, make_grad, eta=0.05, k_fn=None, steps=None, between=None):
    """T steps (or the given step numbers) against the oracle; between(ws)
    runs after every step."""
    g = gce()
    t = g.Table(workloads.table_layers(layers))
    mem = torch.zeros((W, t.N), device="cuda")
    vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
    idx = torch.zeros((W, max(4, t.vals_per_worker)), dtype=torch.int32, device="cuda")
    ws = t.workspace(W, "randk")
    hmem = np.zeros((W, t.N), np.float32)
    for step in (range(T) if steps is None else steps):
        grad = make_grad(step)
        ks = [l["cap"] for l in layers] if k_fn is None else k_fn(step)
        kt = None if k_fn is None else torch.tensor(ks, dtype=torch.int32, device="cuda")
        expect = osteps.sparse_step(layers, host(grad), hmem, eta, ks, method="randk", seed=seed,
                                    step=step, threads=8)
        g.ef_randk_step(t, W, grad, mem, eta, kt, seed, step, vals, idx, ws)
        hv, hi, hm = host(vals), host(idx), host(mem)
        for (w, l), e in expect.items():
            if layers[l]["kind"] == "dense":
                n = layers[l]["rows"] * layers[l]["cols"]
                assert np.array_equal(bits(hv[w, payload_slice(t, 0, l, n)]), bits(e))
            else:
                sl = payload_slice(t, 0, l, ks[l])
                assert np.array_equal(hi[w, sl], e[1]), ("idx", step, w, l)
                assert np.array_equal(bits(hv[w, sl]), bits(e[0])), ("vals", step, w, l)
            ls = layer_slice(t, l)
            assert np.array_equal(bits(hm[w, ls]), bits(hmem[w, ls])), ("mem", step, w, l)
        if between is not None:
            between(ws)
    return g, ws


LAYERS = [dict(rows=1, cols=1, kind="randk", cap=1, sigma=1.0),
          dict(rows=8193, cols=1, kind="randk", cap=80, sigma=1.0),
          dict(rows=64, cols=1, kind="dense", cap=0, sigma=1.0),
          dict(rows=200, cols=500, kind="randk", cap=100000, sigma=1.0),   # k = n
          dict(rows=300017, cols=1, kind="randk", cap=3000, sigma=1.0),
          dict(rows=1 << 20, cols=1, kind="randk", cap=104857, sigma=1.0)]


def test_ragged_table_bit_exact():
    need_gpu()
    run_randk(LAYERS, 2, 3, 1234, lambda s: workloads.gradients(LAYERS, 2, 201, s))


def test_k_changes_between_steps():
    need_gpu()
    layers = [dict(rows=100000, cols=1, kind="randk", cap=10000, sigma=1.0)]
    ks = [[10000], [1000], [1]]
    run_randk(layers, 1, 3, 7, lambda s: workloads.gradients(layers, 1, 202, s),
              k_fn=lambda s: ks[s])


def test_look_ahead_on_and_off_and_skipped_steps():
    """The next step's key pass run inside this step's memory pass gives the
    same bits as running it in its own step: consecutive steps use it, a
    jump in the step number or a different seed does not."""
    need_gpu()
    g = gce()
    mk = lambda s: workloads.gradients(LAYERS, 2, 204, s)
    run_randk(LAYERS, 2, 0, 31, mk, steps=[0, 1, 2, 5, 6, 9])
    try:
        g.set_randk_ahead(False)
        run_randk(LAYERS, 2, 0, 31, mk, steps=[0, 1, 2, 5, 6, 9])
    finally:
        g.set_randk_ahead(True)


def test_look_ahead_survives_a_cleared_workspace():
    """A workspace wiped between two consecutive steps (as a fresh allocation at
    the same address would be) no longer holds the key pass: the tag check
    sends every layer to the exact fallback and the result stays exact."""
    need_gpu()
    g = gce()
    layers = [dict(rows=300017, cols=1, kind="randk", cap=3000, sigma=1.0),
              dict(rows=70000, cols=1, kind="randk", cap=700, sigma=1.0)]
    seen = []

    def wipe(ws):
        seen.append(g.status(ws))
        ws.zero_()

    run_randk(layers, 2, 3, 77, lambda s: workloads.gradients(layers, 2, 205, s), between=wipe)
    assert seen[1] & g.STATUS_FALLBACK and seen[2] & g.STATUS_FALLBACK


def test_forced_fallback_is_still_exact():
    need_gpu()
    g = gce()
    layers = [dict(rows=500000, cols=1, kind="randk", cap=5000, sigma=1.0),
              dict(rows=30000, cols=1, kind="randk", cap=300, sigma=1.0)]
    try:
        g.set_bracket_sigma(-50.0)    # empty band: every layer takes the exact fallback
        g2, ws = run_randk(layers, 2, 2, 99, lambda s: workloads.gradients(layers, 2, 203, s))
        assert g.status(ws) & g.STATUS_FALLBACK
    finally:
        g.set_bracket_sigma(6.0)


def test_bert_base_w8_sampled_units():
    """BERT-base shapes, rand-k 1 %, W = 8 at full size; oracle on sampled units."""
    need_gpu()
    g = gce()
    layers = workloads.bert_base_topk(kind="randk")
    W = 8
    t = g.Table(workloads.table_layers(layers))
    grad = workloads.gradients(layers, W, 4, 0)
    mem = torch.zeros_like(grad)
    vals = torch.zeros((W, t.vals_per_worker), device="cuda")
    idx = torch.zeros((W, t.vals_per_worker), dtype=torch.int32, device="cuda")
    g.ef_randk_step(t, W, grad, mem, 0.05, None, 5, 0, vals, idx, t.workspace(W, "randk"))
    import oracle
    hv, hi = host(vals), host(idx)
    for (w, l) in [(0, 0), (7, 5), (4, 3), (1, len(layers) - 1)]:
        ls = layer_slice(t, l)
        n = layers[l]["rows"] * layers[l]["cols"]
        ev, ei, em = oracle.ef_randk_unit(host(grad[w, ls]), np.zeros(n, np.float32),
                                          layers[l]["cap"], 0.05, 5, w, l, 0)
        sl = payload_slice(t, 0, l, layers[l]["cap"])
        assert np.array_equal(hi[w, sl], ei)
        assert np.array_equal(bits(hv[w, sl]), bits(ev))
        assert np.array_equal(bits(host(mem[w, ls])), bits(em))


def test_worker_offset_rows_equal_the_whole_job():
    """ef_randk_step_at: workers worker0 .. worker0+W-1 of a larger job give,
    row for row and bit for bit, what one ef_randk_step over the whole job
    gives those workers (the generator takes the job-wide worker index).
    Three steps, so the look-ahead record, keyed by worker0 too, is reused."""
    need_gpu()
    g = gce()
    layers = [dict(rows=300, cols=41, kind="randk", cap=123, sigma=1.0),
              dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=70000, cols=1, kind="randk", cap=700, sigma=0.5)]
    W = 4
    t = g.Table(workloads.table_layers(layers))

    def run(worker0, w_count, rows):
        mem = torch.zeros((w_count, t.N), device="cuda")
        vals = torch.zeros((w_count, max(4, t.vals_per_worker)), device="cuda")
        idx = torch.zeros((w_count, max(4, t.vals_per_worker)), dtype=torch.int32, device="cuda")
        ws = t.workspace(w_count, "randk")
        out = []
        for s in range(3):
            grad = workloads.gradients(layers, W, 960, s)[rows].clone()  # 16-byte aligned
            g.ef_randk_step_at(t, worker0, w_count, grad, mem, 0.05, None, 17, s, vals, idx, ws)
            out.append((mem.clone(), vals.clone(), idx.clone()))
        assert g.status(ws) & g.STATUS_K_RANGE == 0
        return out

    whole = run(0, W, slice(0, W))
    for worker0, w_count in [(1, 1), (3, 1), (1, 2)]:
        part = run(worker0, w_count, slice(worker0, worker0 + w_count))
        for (m, v, i), (mw, vw, iw) in zip(part, whole):
            rows = slice(worker0, worker0 + w_count)
            assert torch.equal(m.view(torch.int32), mw[rows].view(torch.int32)), worker0
            assert torch.equal(v.view(torch.int32), vw[rows].view(torch.int32)), worker0
            assert torch.equal(i, iw[rows]), worker0
    with pytest.raises(g.GceError):
        g.ef_randk_step_at(t, -1, 1, torch.zeros((1, t.N), device="cuda"),
                           torch.zeros((1, t.N), device="cuda"), 0.05, None, 17, 0,
                           torch.zeros((1, max(4, t.vals_per_worker)), device="cuda"),
                           torch.zeros((1, max(4, t.vals_per_worker)), dtype=torch.int32,
                                       device="cuda"),
                           t.workspace(1, "randk"))
