"""End-to-end parity on the two workloads the other GPU tests cover only in
part: Accordion driving the compressors on the whole VGG-19 set for its 200
scripted steps, and single layers at the top of the bandwidth sweep.

Sources: "Accordion: Adaptive Gradient Communication via Critical Learning
Regime Identification", Method and Key results (the per-layer level switch
on VGG-19 between l_low = rank 4 / k 10 % and l_high = rank 2 / k 1 %);
"Sparsified SGD with Memory", Method (the error-feedback update, at any d).

Bars: top-k results bit-exact; PowerSGD outputs X in {P, Q, P Q^T, memory}
within ||X_gpu - X_ref||_F / max(||X_ref||_F, ||M||_F) <= 1e-4; Accordion
levels identical.  The oracle always follows its own trajectory.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
import oracle
from oracle import steps as osteps
from tests.helpers import bits, gce, host, layer_slice, need_gpu, payload_slice, torch
from tests.test_gpu_powersgd import PsRun, relerr
from tests.test_gpu_topk import TopkRun, check_topk_properties

pytestmark = pytest.mark.gpu

T_VGG = 200
INTERVAL, THRESHOLD = 10, 0.5
# steps around the scripted drops (60, 140), where the levels switch
SWITCH_STEPS = {0, 1, 9, 10, 59, 60, 61, 69, 70, 71, 139, 140, 141, 149, 150, 151, 199}


class AccordionPair:
    """accordion_select on the GPU next to the oracle's, levels compared."""

    def __init__(self, table, layers, lo, hi):
        self.g = gce()
        self.t, self.layers, self.lo, self.hi = table, layers, lo, hi
        L = len(layers)
        self.prev = torch.empty(L, dtype=torch.float64, device="cuda")
        self.level = torch.empty(L, dtype=torch.int32, device="cuda")
        self.cur = torch.zeros(L, dtype=torch.float64, device="cuda")
        self.kr = torch.zeros(L, dtype=torch.int32, device="cuda")
        self.ws = table.workspace(1, "accordion")
        self.g.accordion_init(table, self.prev, self.level)
        self.st = osteps.AccordionState(L)

    def select(self, grad0, s):
        self.g.accordion_select(self.t, grad0, s, INTERVAL, THRESHOLD, self.lo, self.hi,
                                self.prev, self.level, self.cur, self.kr, self.ws)
        expect = osteps.accordion_step(self.layers, host(grad0), s, INTERVAL, THRESHOLD,
                                       self.st, self.lo, self.hi)
        assert np.array_equal(host(self.level), self.st.level), s
        kr = host(self.kr)
        assert np.array_equal(kr, expect.astype(np.int32)), s
        return kr


def vgg_grad(layers, s):
    return workloads.gradients(layers, 1, 3, s, scale=workloads.vgg19_scale(s))


def test_vgg19_accordion_drives_powersgd_for_200_steps():
    """Accordion picks rank 4 or 2 per layer at every step; powersgd_step runs
    with those ranks on the whole VGG-19 set.  P and Q of every layer are
    compared every step, P Q^T and the memory of every layer every tenth step
    and around each switch."""
    need_gpu()
    layers = workloads.vgg19("powersgd", 4)
    run = PsRun(layers, 1, seed=11)
    acc = AccordionPair(run.t, layers, 4, 2)
    worst = 0.0
    seen = set()
    for s in range(T_VGG):
        grad = vgg_grad(layers, s)
        ranks = acc.select(grad[0], s)
        seen.add(int(ranks[0]))    # layer 0 (conv 1) is a PowerSGD layer
        full = s % 10 == 0 or s in SWITCH_STEPS
        worst = max(worst, run.step(grad, workloads.ETA, [int(r) for r in ranks], full=full))
    assert seen == {2, 4}          # both levels were driven through the compressor
    print("vgg19 powersgd: worst relative error over 200 steps %.3g" % worst)


# the oracle's own trajectory on these VGG-19 layers (w = 0), every step:
# every distinct compressed shape once (conv 1 is the exact-bounds path, the
# FC layer the smallest matrix) and every DENSE layer
def _vgg_oracle_units(layers):
    shapes, units = set(), []
    for l, lay in enumerate(layers):
        key = (lay["rows"], lay["cols"], lay["kind"])
        if lay["kind"] == "dense" or key not in shapes:
            shapes.add(key)
            units.append((0, l))
    return units


def test_vgg19_accordion_drives_topk_for_200_steps():
    """Accordion picks k = 10 % or 1 % of each layer at every step;
    ef_topk_step runs with those k on the whole VGG-19 set.  Every layer is
    checked every step against the properties that fix the top-k result
    (from the GPU's own previous memory); every distinct layer shape follows
    the oracle's own trajectory bit for bit at every step."""
    need_gpu()
    layers = workloads.vgg19("topk", 100000)
    run = TopkRun(layers, 1)
    acc = AccordionPair(run.table, layers, 100000, 10000)
    units = _vgg_oracle_units(layers)
    assert len(units) >= 12
    ks_seen = set()
    for s in range(T_VGG):
        grad = vgg_grad(layers, s)
        kr = acc.select(grad[0], s)
        ks = [int(k) if l["kind"] != "dense" else 0 for k, l in zip(kr, layers)]
        ks_seen.add(ks[0])
        expect = osteps.sparse_step(layers, host(grad), run.host_mem, workloads.ETA, ks,
                                    method="topk", units=units, threads=8)
        mem_old = run.mem.clone()
        run.step(grad, workloads.ETA, ks)
        check_topk_properties(run, grad, mem_old, workloads.ETA, ks=ks)
        del mem_old
        run.compare(expect, ks)
    l0 = layers[0]
    assert ks_seen == {oracle.k_from_ppm(l0["rows"] * l0["cols"], 100000),
                       oracle.k_from_ppm(l0["rows"] * l0["cols"], 10000)}


# ---- the top of the bandwidth sweep ---------------------------------------------------


def _one_layer_run(e, method, ppm):
    layers = workloads.sweep(e, method, ppm)
    return layers, TopkRun(layers, 1)


@pytest.mark.parametrize("ppm", [1000, 10000, 100000])
def test_sweep_top_2p30_topk_properties(ppm):
    """A single 2^30-element layer (131,072 main tiles, the bench's largest
    sweep point) at 0.1 / 1 / 10 %: two steps, every element checked against
    the properties that fix the top-k result."""
    need_gpu()
    layers, run = _one_layer_run(30, "topk", ppm)
    for s in range(2):
        grad = workloads.gradients(layers, 1, 5, s)
        mem_old = run.mem.clone()
        run.step(grad, workloads.ETA)
        check_topk_properties(run, grad, mem_old, workloads.ETA)
        del mem_old, grad
        torch.cuda.empty_cache()


def test_sweep_2p25_topk_oracle_whole_layer():
    """A single 2^25-element layer at 1 % (4096 main tiles): the oracle on the
    whole layer for two steps (its own memory), bit for bit.  The oracle's
    full sort takes tens of seconds per step at this size, so the larger
    sweep points are checked by properties."""
    need_gpu()
    layers, run = _one_layer_run(25, "topk", 10000)
    k = layers[0]["cap"]
    for s in range(2):
        grad = workloads.gradients(layers, 1, 5, 100 + s)
        ev, ei, m_new = oracle.ef_topk_unit(host(grad[0]), run.host_mem[0], k, workloads.ETA)
        run.host_mem[0] = m_new
        run.step(grad, workloads.ETA)
        run.compare({(0, 0): (ev, ei)})
        del grad


def test_sweep_2p25_randk_oracle_whole_layer():
    """rand-k 1 % on a single 2^25-element layer: the oracle on the whole
    layer for two steps, bit for bit (the second step uses the key pass the
    first one ran ahead)."""
    need_gpu()
    g = gce()
    layers = workloads.sweep(25, "randk", 10000)
    t = g.Table(workloads.table_layers(layers))
    n, k = t.N, layers[0]["cap"]
    mem = torch.zeros((1, n), device="cuda")
    vals = torch.zeros((1, t.vals_per_worker), device="cuda")
    idx = torch.zeros((1, t.vals_per_worker), dtype=torch.int32, device="cuda")
    ws = t.workspace(1, "randk")
    hmem = np.zeros(n, np.float32)
    for s in range(2):
        grad = workloads.gradients(layers, 1, 5, 200 + s)
        ev, ei, hmem = oracle.ef_randk_unit(host(grad[0]), hmem, k, workloads.ETA, 9, 0, 0, s)
        g.ef_randk_step(t, 1, grad, mem, workloads.ETA, None, 9, s, vals, idx, ws)
        torch.cuda.synchronize()
        assert np.array_equal(host(idx[0, :k]), ei), s
        assert np.array_equal(bits(host(vals[0, :k])), bits(ev)), s
        assert np.array_equal(bits(host(mem[0])), bits(hmem)), s
        del grad


def _lsr(z, s):
    """Logical right shift of int64 tensors (torch's >> is arithmetic)."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _as_i64(u):
    return u - (1 << 64) if u >= (1 << 63) else u


def _randk_keys(base, i0, i1):
    """rand-k keys of coordinates i0 .. i1-1 on the device: the high 32 bits of
    SplitMix64 output i+1 from the unit's base state (modular int64 arithmetic,
    logical shifts).  The test checks them against the oracle's key function."""
    i = torch.arange(i0, i1, device="cuda", dtype=torch.int64)
    z = _as_i64(base) + (i + 1) * _as_i64(0x9E3779B97F4A7C15)
    z = z ^ _lsr(z, 30)
    z = z * _as_i64(0xBF58476D1CE4E5B9)
    z = z ^ _lsr(z, 27)
    z = z * _as_i64(0x94D049BB133111EB)
    z = z ^ _lsr(z, 31)
    return _lsr(z, 32)


def test_sweep_top_2p30_randk_properties():
    """rand-k 1 % on a single 2^30-element layer (the bench's largest sweep
    point), two steps (the second on the key pass the first ran ahead), every
    element checked on the device: exactly k ascending indices; they are the k
    smallest (key, index) pairs, the keys recomputed from the oracle's base
    state; sent values are v's bits; memory is +0 on the sent set and v
    elsewhere.  v = fl(m + fl(eta * g)) by two torch kernels (no contraction)."""
    need_gpu()
    g = gce()
    layers = workloads.sweep(30, "randk", 10000)
    t = g.Table(workloads.table_layers(layers))
    n, k = t.N, layers[0]["cap"]
    mem = torch.zeros((1, n), device="cuda")
    vals = torch.zeros((1, t.vals_per_worker), device="cuda")
    idx = torch.zeros((1, t.vals_per_worker), dtype=torch.int32, device="cuda")
    ws = t.workspace(1, "randk")
    seed = 9
    for s in range(2):
        base = oracle.randk_base(seed, 0, 0, 0, s)
        probe = [0, 1, 12345, n // 2 + 7, n - 1]
        got = _randk_keys(base, 0, 2).tolist() + [int(_randk_keys(base, i, i + 1)) for i in probe[2:]]
        assert got == [oracle.randk_key(base, i) for i in probe], s
        grad = workloads.gradients(layers, 1, 5, 400 + s)
        mem_old = mem.clone()
        g.ef_randk_step(t, 1, grad, mem, workloads.ETA, None, seed, s, vals, idx, ws)
        torch.cuda.synchronize()
        ix = idx[0, :k].long()
        assert bool((ix[1:] > ix[:-1]).all()) and int(ix[0]) >= 0 and int(ix[-1]) < n
        prod = grad[0] * torch.tensor(workloads.ETA, dtype=torch.float32, device="cuda")
        v = mem_old[0] + prod
        del prod, grad, mem_old
        assert torch.equal(v[ix].view(torch.int32), vals[0, :k].view(torch.int32)), s
        sel = torch.zeros(n, dtype=torch.bool, device="cuda")
        sel[ix] = True
        expect_mem = torch.where(sel, torch.zeros_like(v), v)
        assert torch.equal(mem[0].view(torch.int32), expect_mem.view(torch.int32)), s
        del expect_mem, v
        # the chosen set is the k smallest (key, index): every chosen pair is
        # below every other one (key * 2^31 + index orders the pairs)
        top_chosen, low_other = -1, 1 << 64
        step = 1 << 26
        for i0 in range(0, n, step):
            comb = _randk_keys(base, i0, i0 + step) * (1 << 31) + torch.arange(
                i0, i0 + step, device="cuda", dtype=torch.int64)
            c = sel[i0:i0 + step]
            if bool(c.any()):
                top_chosen = max(top_chosen, int(comb[c].max()))
            if bool((~c).any()):
                low_other = min(low_other, int(comb[~c].min()))
            del comb
        assert top_chosen < low_other, s
        del sel
        torch.cuda.empty_cache()


@pytest.mark.parametrize("rank", [1, 2, 4])
def test_tall_2p26_powersgd_oracle_whole_matrix(rank):
    """PowerSGD rank 1 / 2 / 4 on a 32768 x 2048 matrix (2^26 elements; P is
    orthonormalised over several row chunks, as at the top of the sweep): two
    steps against the oracle's own trajectory, every output within 1e-4."""
    need_gpu()
    layers = [dict(rows=32768, cols=2048, kind="powersgd", cap=rank, sigma=1.0)]
    run = PsRun(layers, 1, seed=13)
    for s in range(2):
        worst = run.step(workloads.gradients(layers, 1, 5, 300 + s), workloads.ETA)
        assert worst <= 1e-4


@pytest.mark.parametrize("rank", [1, 2, 4])
def test_sweep_top_2p30_powersgd_properties(rank):
    """PowerSGD rank 1 / 2 / 4 on the 2^15 x 2^15 matrix (the bench's largest
    sweep point), checked in fp64 on the device from the step's own inputs: P
    has orthonormal columns, equal to the QR factor (positive diagonal) of
    M Q; Q' = M^T P; memory + P Q'^T = M."""
    need_gpu()
    g = gce()
    layers = workloads.sweep(30, "powersgd", rank=rank)
    rows, cols = layers[0]["rows"], layers[0]["cols"]
    t = g.Table(workloads.table_layers(layers))
    mem = torch.zeros((1, t.N), device="cuda")
    P = torch.zeros((1, t.P_per_worker), device="cuda")
    Q = torch.zeros((1, t.Q_per_worker), device="cuda")
    ws = t.workspace(1, "powersgd")
    g.powersgd_init_q(t, 1, 17, Q)
    for s in range(2):
        grad = workloads.gradients(layers, 1, 5, 400 + s)
        prod = grad * torch.tensor(workloads.ETA, device="cuda")
        M = (mem + prod).view(rows, cols)            # fl(m + fl(eta g)), two kernels
        del prod
        Q0 = Q[0].view(cols, rank).double()
        g.powersgd_step(t, 1, grad, mem, workloads.ETA, None, P, Q, None, None, ws)
        torch.cuda.synchronize()
        Md = M.double()
        Pg, Qg = P[0].view(rows, rank).double(), Q[0].view(cols, rank).double()
        eye = Pg.T @ Pg
        assert float((eye - torch.eye(rank, device="cuda", dtype=torch.float64)).abs().max()) < 1e-5
        # span: P is the orthonormal factor of M Q0 (column order, positive diagonal)
        Pref, R = torch.linalg.qr(Md @ Q0)
        Pref = Pref * torch.sign(torch.diagonal(R))[None, :]
        Mn = float(torch.linalg.norm(Md))
        assert float(torch.linalg.norm(Pg - Pref)) / max(float(torch.linalg.norm(Pref)), 1.0) < 1e-4
        Qref = Md.T @ Pg
        assert float(torch.linalg.norm(Qg - Qref)) / max(float(torch.linalg.norm(Qref)), Mn) < 1e-4
        resid = (mem[0].view(rows, cols).double() + Pg @ Qg.T - Md)
        assert float(torch.linalg.norm(resid)) / Mn < 1e-4
        del grad, M, Md, resid, Pref, R, Qref
        torch.cuda.empty_cache()
