"""GPU parity of ef_topk_step against the CPU oracle (bit-exact).

Source: "Sparsified SGD with Memory", Method (the error-feedback top-k
update).  Every case compares vals, idx and the new memory of every
(worker, layer) bit for bit with oracle.steps.sparse_step on the same
seeded inputs, over several steps so that the memory carries.  At the
BERT-base size the oracle runs on sampled (worker, layer) units and every
unit is checked against properties that define the top-k set at any size.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
import oracle
from tests.helpers import HAS_GPU, bits, gce, host, need_gpu, payload_slice, layer_slice, torch

pytestmark = pytest.mark.gpu


class TopkRun:
    def __init__(self, layers, W):
        self.g = gce()
        self.layers = layers
        self.W = W
        self.table = self.g.Table(workloads.table_layers(layers))
        t = self.table
        dev = "cuda"
        self.mem = torch.zeros((W, t.N), dtype=torch.float32, device=dev)
        self.vals = torch.zeros((W, max(t.vals_per_worker, 4)), dtype=torch.float32, device=dev)
        self.idx = torch.zeros((W, max(t.vals_per_worker, 4)), dtype=torch.int32, device=dev)
        self.ws = t.workspace(W, "topk")
        self.host_mem = np.zeros((W, t.N), np.float32)

    def step(self, grad, eta, k_per_layer=None):
        kt = None
        if k_per_layer is not None:
            kt = torch.tensor(k_per_layer, dtype=torch.int32, device="cuda")
        self.g.ef_topk_step(self.table, self.W, grad, self.mem, eta, kt, self.vals, self.idx,
                            self.ws)
        torch.cuda.synchronize()

    def ks(self, k_per_layer=None):
        return [l["cap"] if k_per_layer is None else k_per_layer[i]
                for i, l in enumerate(self.layers)]

    def compare(self, expect, k_per_layer=None, units=None):
        """expect: oracle output {(w,l): (vals, idx) | payload}; host_mem updated."""
        vals, idx, mem = host(self.vals), host(self.idx), host(self.mem)
        ks = self.ks(k_per_layer)
        for (w, l), e in expect.items():
            lay = self.layers[l]
            if lay["kind"] == "dense":
                n = lay["rows"] * lay["cols"]
                got = vals[w, payload_slice(self.table, 0, l, n)]
                assert np.array_equal(bits(got), bits(e)), (w, l)
            else:
                ev, ei = e
                sl = payload_slice(self.table, 0, l, ks[l])
                assert np.array_equal(idx[w, sl], ei), ("idx", w, l)
                assert np.array_equal(bits(vals[w, sl]), bits(ev)), ("vals", w, l)
            ls = layer_slice(self.table, l)
            assert np.array_equal(bits(mem[w, ls]), bits(self.host_mem[w, ls])), ("mem", w, l)


def run_and_compare(layers, W, T, make_grad, eta=0.05, k_fn=None):
    run = TopkRun(layers, W)
    for t in range(T):
        grad = make_grad(t)
        kpl = k_fn(t) if k_fn else None
        hg = host(grad)
        expect = osteps.sparse_step(layers, hg, run.host_mem, eta, run.ks(kpl), method="topk",
                                    threads=8)
        run.step(grad, eta, kpl)
        run.compare(expect, kpl)
    return run


def randn_grad(layers, W, cfg):
    return lambda t: workloads.gradients(layers, W, cfg, t)


RAGGED = [dict(rows=1, cols=1, kind="topk", cap=1),
          dict(rows=7, cols=1, kind="topk", cap=3),
          dict(rows=100, cols=1, kind="dense", cap=0),
          dict(rows=8191, cols=1, kind="topk", cap=81),
          dict(rows=64, cols=128, kind="topk", cap=8192),      # k = n
          dict(rows=8193, cols=1, kind="topk", cap=1),
          dict(rows=350, cols=200, kind="topk", cap=700),       # sampled path, 1 %
          dict(rows=300017, cols=1, kind="topk", cap=30001),    # ragged tail, 10 %
          dict(rows=5, cols=3, kind="dense", cap=0)]


def test_ragged_table_bit_exact():
    need_gpu()
    for l in RAGGED:
        l["sigma"] = 1.0
    run_and_compare(RAGGED, 2, 3, randn_grad(RAGGED, 2, 101))


def test_per_layer_k_changes_between_steps():
    need_gpu()
    layers = [dict(rows=100000, cols=1, kind="topk", cap=10000, sigma=1.0),
              dict(rows=1728, cols=1, kind="topk", cap=172, sigma=1.0)]
    ks = [[10000, 172], [1000, 17], [10000, 17]]
    run_and_compare(layers, 1, 3, randn_grad(layers, 1, 102), k_fn=lambda t: ks[t])


def test_ties_integer_gradients():
    need_gpu()
    layers = [dict(rows=200000, cols=1, kind="topk", cap=2000, sigma=1.0),
              dict(rows=9000, cols=1, kind="topk", cap=4500, sigma=1.0)]
    W = 2
    N = workloads.total_elements(layers)

    def mk(t):
        g = torch.Generator(device="cuda")
        g.manual_seed(7000 + t)
        return torch.randint(-3, 4, (W, N), generator=g, device="cuda").float()

    run_and_compare(layers, W, 3, mk, eta=1.0)


def test_short_list_with_ties_at_T():
    """Gradients on a 1/64 grid: the value at the k-th place recurs a few hundred
    times, so the short list of keys in T's level-1 bin, from which the scan
    fixes T, holds ties at T that split across tiles.  Bit-exact, three steps."""
    need_gpu()
    layers = [dict(rows=300000, cols=1, kind="topk", cap=3000, sigma=1.0),
              dict(rows=700, cols=900, kind="topk", cap=6300, sigma=1.0),
              dict(rows=65536, cols=1, kind="topk", cap=655, sigma=1.0)]
    W = 2

    def mk(t):
        return torch.round(workloads.gradients(layers, W, 109, t) * 64.0) / 64.0

    run_and_compare(layers, W, 3, mk, eta=1.0)


def test_all_equal_magnitudes_and_zeros():
    need_gpu()
    layers = [dict(rows=100000, cols=1, kind="topk", cap=777, sigma=1.0),
              dict(rows=20000, cols=1, kind="topk", cap=20000, sigma=1.0),
              dict(rows=70000, cols=1, kind="topk", cap=5, sigma=1.0)]
    W = 1
    N = workloads.total_elements(layers)

    def mk(t):
        g = torch.Generator(device="cuda")
        g.manual_seed(8000 + t)
        sign = torch.randint(0, 2, (W, N), generator=g, device="cuda").float() * 2 - 1
        if t == 0:
            return torch.zeros((W, N), device="cuda")   # every |v| is 0: ties everywhere
        return sign * 0.5                               # |v| equal within each step

    run_and_compare(layers, W, 3, mk, eta=1.0)


def test_forced_fallback_is_still_exact():
    need_gpu()
    g = gce()
    layers = [dict(rows=400000, cols=1, kind="topk", cap=4000, sigma=1.0),
              dict(rows=65536, cols=3, kind="topk", cap=20000, sigma=1.0)]
    try:
        g.set_bracket_sigma(-60.0)   # candidate bound far too high: lists come out short
        run = run_and_compare(layers, 2, 2, randn_grad(layers, 2, 103))
        assert g.status(run.ws) & g.STATUS_FALLBACK
    finally:
        g.set_bracket_sigma(6.0)


def test_large_table_with_fallback_in_every_layer():
    """Ten 2.5 M-element top-k layers and a dense one over 4 workers (about
    1.2 GB of main-pass traffic), run once on the sampled bounds and once
    with every layer forced to the exact fallback.  Properties on every unit,
    the oracle on four units."""
    need_gpu()
    g = gce()
    layers = [dict(rows=2500, cols=1000, kind="topk", cap=25000, sigma=1.0) for _ in range(10)]
    layers.insert(5, dict(rows=300, cols=7, kind="dense", cap=0))
    W = 4
    units = [(3, 1), (0, 4), (1, 6), (2, 10)]
    for sigma in (6.0, -60.0):
        try:
            g.set_bracket_sigma(sigma)
            run = TopkRun(layers, W)
            host_mem = {u: np.zeros(2500 * 1000, np.float32) for u in units}
            for t in range(2):
                grad = workloads.gradients(layers, W, 106, t)
                mem_old = run.mem.clone()
                run.step(grad, workloads.ETA)
                check_topk_properties(run, grad, mem_old, workloads.ETA)
                del mem_old
                vals, idx = host(run.vals), host(run.idx)
                for (w, l) in units:
                    ls = layer_slice(run.table, l)
                    ev, ei, m_new = oracle.ef_topk_unit(host(grad[w, ls]), host_mem[(w, l)],
                                                        layers[l]["cap"], workloads.ETA)
                    host_mem[(w, l)] = m_new
                    sl = payload_slice(run.table, 0, l, layers[l]["cap"])
                    assert np.array_equal(idx[w, sl], ei), (sigma, w, l)
                    assert np.array_equal(bits(vals[w, sl]), bits(ev)), (sigma, w, l)
                    assert np.array_equal(bits(host(run.mem[w, ls])), bits(m_new)), (sigma, w, l)
            if sigma < 0:
                assert g.status(run.ws) & g.STATUS_FALLBACK
        finally:
            g.set_bracket_sigma(6.0)


def test_sample_blind_to_the_large_values_takes_the_coarse_levels():
    """The sample reads the first 32 elements of every 4096; here those are a
    thousand times smaller than the rest, so both sampled bounds come out far
    too low: nearly every element is a candidate (no fallback) and T lies above
    the upper bound, in one of level 1's coarse bins, so the selection takes all
    three radix levels.  Bit-exact against the oracle over two steps."""
    need_gpu()
    layers = [dict(rows=300000, cols=1, kind="topk", cap=3000, sigma=1.0),
              dict(rows=1000, cols=1000, kind="topk", cap=20000, sigma=1.0)]
    W = 2

    def mk(t):
        grad = workloads.gradients(layers, W, 108, t)
        pos = torch.arange(grad.shape[1], device="cuda")
        off = 0
        for l in layers:
            n = l["rows"] * l["cols"]
            seen = ((pos[off:off + n] - off) % 4096) < 32
            grad[:, off:off + n][:, seen] *= 1e-3
            off += n
        return grad

    run = run_and_compare(layers, W, 2, mk, eta=1.0)
    assert not run.g.status(run.ws) & run.g.STATUS_FALLBACK


def test_k_out_of_range_skips_layer_and_flags():
    need_gpu()
    g = gce()
    layers = [dict(rows=1000, cols=1, kind="topk", cap=10, sigma=1.0),
              dict(rows=2000, cols=1, kind="topk", cap=20, sigma=1.0)]
    run = TopkRun(layers, 1)
    grad = workloads.gradients(layers, 1, 104, 0)
    mem0 = run.mem.clone()
    run.step(grad, 0.05, [11, 20])                       # 11 > cap for layer 0
    assert g.status(run.ws) & g.STATUS_K_RANGE
    assert torch.equal(run.mem[:, :1000], mem0[:, :1000])
    expect = osteps.sparse_step(layers[1:], host(grad)[:, 1000:], run.host_mem[:, 1000:].copy(),
                                0.05, [20])
    ev, ei = expect[(0, 0)]
    assert np.array_equal(host(run.idx)[0, payload_slice(run.table, 0, 1, 20)], ei)


def test_repeated_step_is_deterministic():
    need_gpu()
    layers = workloads.memsgd_vector(1 << 20, 1024)
    g = gce()
    grad = workloads.gradients(layers, 1, 105, 0)
    outs = []
    for _ in range(3):
        run = TopkRun(layers, 1)
        run.mem.copy_(grad * 3)
        run.step(grad, 0.05)
        outs.append((host(run.vals).copy(), host(run.idx).copy(), host(run.mem).copy()))
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert np.array_equal(np.asarray(a).view(np.uint32), np.asarray(b).view(np.uint32))


def test_memsgd_vector_20_steps():
    """2^20-element vector, k = 1024, eta = 0.05, memory from 0, 20 steps."""
    need_gpu()
    layers = workloads.memsgd_vector()
    assert layers[0]["cap"] == 1024
    run_and_compare(layers, 1, 20, randn_grad(layers, 1, 1))


def check_topk_properties(run, grad, mem_old, eta, ks=None):
    """Properties that fix the top-k result at any size, checked with torch on
    the device: exactly k ascending unique indices per unit; sent values are
    v's bits; new memory + sent == v bit for bit; every sent |v| beats every
    kept one, ties going to the lower index.  ks: k per layer (default the
    caps).

    v = fl(m + fl(eta * g)) is formed by two separate torch kernels: the
    product is written to memory as an fp32 tensor before the sum reads it,
    so nothing can contract the two roundings into one FMA."""
    t = run.table
    W = run.W
    prod = grad * torch.tensor(eta, dtype=torch.float32, device="cuda")
    v = mem_old + prod
    del prod
    mem = run.mem
    sent = torch.zeros_like(mem)
    sel = torch.zeros(mem.shape, dtype=torch.bool, device="cuda")
    for l, lay in enumerate(run.layers):
        n = lay["rows"] * lay["cols"]
        off = t.info[l]["offset"]
        k = lay["cap"] if ks is None else int(ks[l])
        vo = t.info[l]["val_offset"]
        if lay["kind"] == "dense":     # sent whole; memory left at zero
            dv = run.vals[:, vo:vo + n]
            assert torch.equal(dv.view(torch.int32), v[:, off:off + n].view(torch.int32)), l
            sent[:, off:off + n] = dv
            continue
        ix = run.idx[:, vo:vo + k].long()
        vv = run.vals[:, vo:vo + k]
        assert bool((ix[:, 1:] > ix[:, :-1]).all()) if k > 1 else True, l
        assert int(ix.min()) >= 0 and int(ix.max()) < n
        vl = v[:, off:off + n]
        assert torch.equal(torch.gather(vl, 1, ix).view(torch.int32), vv.view(torch.int32))
        sent[:, off:off + n].scatter_(1, ix, vv)
        sel[:, off:off + n].scatter_(1, ix, True)
        key = vl.abs()
        s_l = sel[:, off:off + n]
        kmin = torch.where(s_l, key, torch.full_like(key, float("inf"))).min(dim=1).values
        kmax = torch.where(~s_l, key, torch.full_like(key, -1.0)).max(dim=1).values
        assert bool((kmin >= kmax).all()), l
        tie = (key == kmin[:, None])
        pos = torch.arange(n, device="cuda")[None, :].expand(W, n)
        sel_tie_max = torch.where(s_l & tie, pos, torch.full_like(pos, -1)).max(dim=1).values
        uns_tie_min = torch.where(~s_l & tie, pos, torch.full_like(pos, n)).min(dim=1).values
        assert bool((sel_tie_max < uns_tie_min).all()), l
    assert torch.equal((mem + sent).view(torch.int32), (v + 0.0).view(torch.int32))


def test_bert_base_w8_full_size():
    """BERT-base-shaped top-k 1 % over W = 8 replicas at full size (the bench
    workload): properties on every unit, oracle on sampled units, 2 steps."""
    need_gpu()
    layers = workloads.bert_base_topk()
    for l in layers:
        assert l["cap"] == oracle.k_from_ppm(l["rows"] * l["cols"], 10000)
    W = 8
    run = TopkRun(layers, W)
    sample_units = [(0, 0), (7, 4), (3, 3), (5, len(layers) - 1), (2, 8), (6, 9)]
    host_mem = {u: np.zeros(layers[u[1]]["rows"] * layers[u[1]]["cols"], np.float32)
                for u in sample_units}
    for t in range(2):
        grad = workloads.gradients(layers, W, 4, t)
        mem_old = run.mem.clone()
        run.step(grad, workloads.ETA)
        check_topk_properties(run, grad, mem_old, workloads.ETA)
        del mem_old
        vals, idx = host(run.vals), host(run.idx)
        for (w, l) in sample_units:
            ls = layer_slice(run.table, l)
            g_u = host(grad[w, ls])
            ev, ei, m_new = oracle.ef_topk_unit(g_u, host_mem[(w, l)], layers[l]["cap"],
                                                workloads.ETA)
            host_mem[(w, l)] = m_new
            sl = payload_slice(run.table, 0, l, layers[l]["cap"])
            assert np.array_equal(idx[w, sl], ei), (w, l)
            assert np.array_equal(bits(vals[w, sl]), bits(ev)), (w, l)
            assert np.array_equal(bits(host(run.mem[w, ls])), bits(m_new)), (w, l)
        del grad
    torch.cuda.empty_cache()
