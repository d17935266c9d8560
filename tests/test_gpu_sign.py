"""GPU parity of ef_sign_step (signSGD with error feedback), and of the sum
and majority-vote aggregates of its payloads, against the CPU oracle.

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Method / Key results: sign SGD, one bit per element, gathered;
"Sparsified SGD with Memory", Method: the memory.  The sign bits are
bit-exact.  The scale is an fp64 sum rounded once to fp32; the library adds
in its own fixed order, the oracle in index order, so the two may differ by
one fp32 step (never seen in practice): the test asserts equality within one
step and, where the scales are equal, the memory bit for bit.  The oracle
always follows its own trajectory and never takes the library's state.  Where
the scales differ, the memories of that step may differ by at most the scale
difference plus one rounding of the memory, and the two trajectories part:
from then on that unit is checked step by step against a separate oracle call
on the inputs the library's step had (its previous memory), with the same
rules.  Both aggregates, run on the library's own payload, are bit-exact.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
import oracle
from oracle import steps as osteps
from tests.helpers import bits, gce, host, layer_slice, need_gpu, torch

pytestmark = pytest.mark.gpu


def payload_of(table, layers, hv, W):
    """{(w, l): (scale, words)} for sign layers, {(w, l): floats} for dense."""
    out = {}
    for w in range(W):
        for l, lay in enumerate(layers):
            o = table.info[l]["val_offset"]
            n = lay["rows"] * lay["cols"]
            if lay["kind"] == "dense":
                out[(w, l)] = hv[w, o:o + n].copy()
            else:
                out[(w, l)] = (hv[w, o], hv[w, o + 4:o + 4 + (n + 31) // 32].view(np.uint32).copy())
    return out


class SignRun:
    def __init__(self, layers, W):
        self.g = gce()
        self.layers = layers
        self.W = W
        self.t = self.g.Table(workloads.table_layers(layers))
        t = self.t
        self.mem = torch.zeros((W, t.N), device="cuda")
        self.vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
        self.ws = t.workspace(W, "sign")
        self.hmem = np.zeros((W, t.N), np.float32)
        self.parted = set()   # units whose trajectories parted at a scale difference

    def step(self, grad, eta, check=True):
        hg = host(grad)
        gmem_old = host(self.mem) if check and self.parted else None
        expect = osteps.sparse_step(self.layers, hg, self.hmem, eta, None, method="sign",
                                    threads=8) if check else None
        self.g.ef_sign_step(self.t, self.W, grad, self.mem, eta, self.vals, self.ws)
        torch.cuda.synchronize()
        hv, hm = host(self.vals), host(self.mem)
        pay = payload_of(self.t, self.layers, hv, self.W)
        if not check:
            return pay
        for (w, l), e in expect.items():
            lay = self.layers[l]
            ls = layer_slice(self.t, l)
            if lay["kind"] == "dense":
                assert np.array_equal(bits(pay[(w, l)]), bits(e)), (w, l)
                assert np.array_equal(bits(hm[w, ls]), bits(self.hmem[w, ls])), (w, l)
                continue
            m_ref = self.hmem[w, ls]
            if (w, l) in self.parted:
                # single-step parity from the inputs this step had on the GPU
                m_ref = gmem_old[w, ls].copy()
                e = oracle.ef_sign_unit(hg[w, ls], m_ref, eta)
                e, m_ref = (e[0], e[1]), e[2]
            if not same_step(pay[(w, l)], hm[w, ls], e, m_ref, (w, l)):
                self.parted.add((w, l))
        return pay


def same_step(got, m_gpu, e, m_ref, unit):
    """Sign bits equal, scales within one fp32 step, memory bit for bit when
    the scales agree and within their difference plus one rounding when not.
    Returns whether the scales agreed."""
    sc, words = got
    e_sc, e_words = e
    assert np.array_equal(words, e_words), ("bits", unit)
    assert abs(int(bits(sc)) - int(bits(e_sc))) <= 1, ("scale", unit, sc, e_sc)
    if sc == e_sc:
        assert np.array_equal(bits(m_gpu), bits(m_ref)), ("mem", unit)
        return True
    mg, mr = m_gpu.astype(np.float64), m_ref.astype(np.float64)
    slack = np.spacing(np.maximum(np.abs(m_gpu), np.abs(m_ref)))
    assert np.all(np.abs(mg - mr) <= abs(float(sc) - float(e_sc)) + slack), ("mem", unit)
    return False


RAGGED = [dict(rows=1, cols=1, kind="sign", cap=0),
          dict(rows=31, cols=1, kind="sign", cap=0),
          dict(rows=33, cols=1, kind="sign", cap=0),
          dict(rows=7, cols=1, kind="dense", cap=0),        # later layers off 16 B alignment
          dict(rows=8191, cols=1, kind="sign", cap=0),
          dict(rows=64, cols=128, kind="sign", cap=0),      # exactly one tile
          dict(rows=8193, cols=1, kind="sign", cap=0),
          dict(rows=300017, cols=1, kind="sign", cap=0)]


def test_ragged_table_three_workers_three_steps():
    need_gpu()
    run = SignRun(RAGGED, 3)
    for s in range(3):
        run.step(workloads.gradients(RAGGED, 3, 700, s), 0.05)


def test_aligned_table_and_both_aggregates():
    need_gpu()
    g = gce()
    layers = [dict(rows=256, cols=1024, kind="sign", cap=0),
              dict(rows=100, cols=1, kind="dense", cap=0),
              dict(rows=4, cols=4096, kind="sign", cap=0)]
    W = 5
    run = SignRun(layers, W)
    for s in range(2):
        pay = run.step(workloads.gradients(layers, W, 701, s), 0.1)
    t = run.t
    ws = t.workspace(W, "decompress")
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate(t, W, run.vals, None, None, None, None, 0.2, out, ws)
    assert np.array_equal(bits(host(out)), bits(osteps.decompress(layers, W, pay, 0.2)))
    vote = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_vote(t, W, run.vals, 0.01, vote)
    assert np.array_equal(bits(host(vote)), bits(osteps.vote(layers, W, pay, 0.01)))
    x0 = np.random.default_rng(9).standard_normal(t.N).astype(np.float32)
    x = torch.from_numpy(x0.copy()).cuda()
    g.decompress_apply(t, W, run.vals, None, None, None, None, 0.2, x, ws)
    assert np.array_equal(bits(host(x)), bits(osteps.apply_update(layers, W, pay, 0.2, x0)))


def test_vote_ties_and_even_worker_count():
    """Two workers with opposite signs everywhere vote 0; equal signs vote
    +-scale."""
    need_gpu()
    g = gce()
    layers = [dict(rows=1000, cols=1, kind="sign", cap=0)]
    t = g.Table(workloads.table_layers(layers))
    W = 2
    grad = torch.randn(1, t.N, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    grad = torch.cat([grad, -grad])
    mem = torch.zeros((W, t.N), device="cuda")
    vals = torch.zeros((W, t.vals_per_worker), device="cuda")
    g.ef_sign_step(t, W, grad, mem, 1.0, vals, t.workspace(W, "sign"))
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_vote(t, W, vals, 1.0, out)
    ho = host(out)
    hg = host(grad)[0]
    assert (ho[hg != 0] == 0).all()


def test_bert_base_w8_full_size():
    """BERT-base-shaped sign layers over W = 8 replicas at full size: every
    unit's bits against torch's signbit on the device, the oracle on sampled
    units, two steps."""
    need_gpu()
    layers = workloads.bert_base_topk(kind="sign")
    W = 8
    run = SignRun(layers, W)
    units = [(0, 0), (7, 4), (3, len(layers) - 1), (5, 8)]
    host_mem = {u: np.zeros(layers[u[1]]["rows"] * layers[u[1]]["cols"], np.float32)
                for u in units}
    parted = set()   # units whose trajectories parted at a scale difference
    for s in range(2):
        grad = workloads.gradients(layers, W, 4, s)
        mem_old = run.mem.clone()
        # a parted unit is checked for one step from the inputs it had on the
        # GPU; the oracle's own trajectory is never overwritten
        gpu_in = {(w, l): host(mem_old[w, layer_slice(run.t, l)]) for (w, l) in parted}
        pay = run.step(grad, workloads.ETA, check=False)
        p = mem_old + grad * torch.tensor(workloads.ETA, dtype=torch.float32, device="cuda")
        hv = host(run.vals)
        for l in range(len(layers)):
            info = run.t.info[l]
            n, o = info["n"], info["val_offset"]
            neg = torch.signbit(p[:, info["offset"]:info["offset"] + n])
            pad = (-n) % 32
            negp = torch.nn.functional.pad(neg.to(torch.int64), (0, pad)).view(W, -1, 32)
            want = (negp << torch.arange(32, device="cuda")).sum(dim=2)
            got = torch.from_numpy(hv[:, o + 4:o + 4 + (n + 31) // 32].view(np.uint32)
                                   .astype(np.int64)).cuda()
            assert torch.equal(want, got), l
        del p, mem_old
        for (w, l) in units:
            ls = layer_slice(run.t, l)
            m_in = gpu_in[(w, l)] if (w, l) in parted else host_mem[(w, l)]
            sc, words, m_new = oracle.ef_sign_unit(host(grad[w, ls]), m_in, workloads.ETA)
            if (w, l) not in parted:
                host_mem[(w, l)] = m_new
            if not same_step(pay[(w, l)], host(run.mem[w, ls]), (sc, words), m_new, (w, l)):
                parted.add((w, l))
        del grad
    torch.cuda.empty_cache()


def test_thirty_three_workers_sum_vote_and_noalloc():
    """33 workers: the sum decode stages the sign words of 32 workers at a
    time (two chunks here); the vote counts all 33; the decode without a
    workspace gives the same bits as the one with."""
    need_gpu()
    g = gce()
    layers = [dict(rows=5000, cols=3, kind="sign", cap=0), dict(rows=9, cols=1, kind="dense", cap=0),
              dict(rows=4097, cols=1, kind="sign", cap=0)]
    W = 33
    run = SignRun(layers, W)
    pay = run.step(workloads.gradients(layers, W, 702, 0), 0.05)
    t = run.t
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate(t, W, run.vals, None, None, None, None, 0.75, out,
                            t.workspace(W, "decompress"))
    assert np.array_equal(bits(host(out)), bits(osteps.decompress(layers, W, pay, 0.75)))
    out2 = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate_noalloc(t, W, run.vals, None, None, None, None, 0.75, out2)
    assert torch.equal(out.view(torch.int32), out2.view(torch.int32))
    vote = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_vote(t, W, run.vals, 2.0, vote)
    assert np.array_equal(bits(host(vote)), bits(osteps.vote(layers, W, pay, 2.0)))


@pytest.mark.parametrize("W", [1, 8, 16, 17, 32])
def test_vote_and_sum_at_several_worker_counts(W):
    """Both aggregates on the ragged table, bit for bit against the oracle: one
    worker, 8 (the sum by its table of 256 worker-order sums; the vote with four
    words a lane group), 16 (the last transposed vote), 17 and 32 (the vote a
    thread per four outputs)."""
    need_gpu()
    g = gce()
    run = SignRun(RAGGED, W)
    pay = run.step(workloads.gradients(RAGGED, W, 703, 0), 0.05, check=False)
    t = run.t
    vote = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_vote(t, W, run.vals, 0.5, vote)
    assert np.array_equal(bits(host(vote)), bits(osteps.vote(RAGGED, W, pay, 0.5)))
    out = torch.full((t.N,), float("nan"), device="cuda")
    g.decompress_accumulate(t, W, run.vals, None, None, None, None, 0.25, out,
                            t.workspace(W, "decompress"))
    assert np.array_equal(bits(host(out)), bits(osteps.decompress(RAGGED, W, pay, 0.25)))


PIPE_LAYERS = [dict(rows=190000, cols=1, kind="sign", cap=0, sigma=1.0),
               dict(rows=33, cols=1, kind="dense", cap=0, sigma=1.0),
               dict(rows=5000, cols=3, kind="sign", cap=0, sigma=0.5),
               dict(rows=8192, cols=1, kind="sign", cap=0, sigma=2.0),
               dict(rows=300000, cols=1, kind="sign", cap=0, sigma=1.0),
               dict(rows=1, cols=1, kind="sign", cap=0, sigma=1.0)]


def _sign_steps(g, t, W, grad_seeds, ahead):
    """Two steps from the same memory under one schedule; (mem, vals, status)."""
    g.set_sign_ahead(ahead)
    mem = 0.1 * workloads.gradients(PIPE_LAYERS, W, 951, 0)
    vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
    ws = t.workspace(W, "sign")
    for s in grad_seeds:
        g.ef_sign_step(t, W, workloads.gradients(PIPE_LAYERS, W, 950, s), mem, 0.05, vals, ws)
    return mem, vals, g.status(ws)


@pytest.mark.parametrize("ahead", [1, 64, 300, 100000])
def test_pipelined_schedule_gives_the_two_pass_bits(ahead):
    """The one-launch schedule (norm tiles `ahead` tiles in front of the memory
    update) and the two passes give the same memory, scales and words: the
    partials, their order and the scale do not depend on the schedule.  The
    default schedule is checked against the oracle by the tests above."""
    need_gpu()
    g = gce()
    W = 3
    t = g.Table(workloads.table_layers(PIPE_LAYERS))
    try:
        m0, v0, st0 = _sign_steps(g, t, W, [0, 1], 0)
        m1, v1, st1 = _sign_steps(g, t, W, [0, 1], ahead)
    finally:
        g.set_sign_ahead(-1)
    assert st0 == 0 and st1 == 0
    assert torch.equal(m0.view(torch.int32), m1.view(torch.int32))
    assert torch.equal(v0.view(torch.int32), v1.view(torch.int32))


def test_wait_that_runs_out_sets_the_status():
    """Failure detection without a fault: with every memory-update tile placed
    before every norm tile, each update's wait for its layer scale runs out
    (about a second), the kernel sets GCE_STATUS_WAIT_TIMEOUT and returns; the
    context stays usable and the next step, in the normal order, is clean and
    matches the oracle.  One tile, one block: a single wait runs out."""
    need_gpu()
    g = gce()
    layers = [dict(rows=8192, cols=1, kind="sign", cap=0, sigma=1.0)]
    t = g.Table(workloads.table_layers(layers))
    mem = torch.zeros((1, t.N), device="cuda")
    vals = torch.zeros((1, max(4, t.vals_per_worker)), device="cuda")
    ws = t.workspace(1, "sign")
    grad = workloads.gradients(layers, 1, 952, 0)
    big = g.Table(workloads.table_layers([dict(rows=9 * 8192, cols=1, kind="sign", cap=0)]))
    try:
        g.set_sign_emit_first(True)
        g.ef_sign_step(t, 1, grad, mem, 0.05, vals, ws)
        st = g.status(ws)
        # more than 8 tiles: refused on the host, nothing launched
        with pytest.raises(g.GceError):
            g.ef_sign_step(big, 1, torch.zeros((1, big.N), device="cuda"),
                           torch.zeros((1, big.N), device="cuda"), 0.05,
                           torch.zeros((1, max(4, big.vals_per_worker)), device="cuda"),
                           big.workspace(1, "sign"))
    finally:
        g.set_sign_emit_first(False)
    assert st & g.STATUS_WAIT_TIMEOUT
    run = SignRun(layers, 1)
    run.step(grad, np.float32(0.05))
    assert g.status(run.ws) == 0
