"""powersgd_step_lazy against powersgd_step and the oracle.

The lazy step leaves M = m + eta*grad in the memory and takes the previous
step's P Q^T off when it next reads it; its payload (P, Q, DENSE values) and
the memory that gce_materialize_memory gives back must be those of the eager
step bit for bit, over steps that change ranks, skip a layer and
materialise in the middle.  The eager step is itself checked against the
oracle ("Accordion ...", Method: PowerSGD ranks; "Sparsified SGD with
Memory", Method: the memory); here P and Q of the lazy run are also compared
with the oracle's own trajectory within 1e-4.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, need_gpu, torch
from tests.test_gpu_powersgd import relerr

pytestmark = pytest.mark.gpu

LAYERS = [dict(rows=64, cols=27, kind="powersgd", cap=4, sigma=0.2),
          dict(rows=100, cols=1, kind="dense", cap=0, sigma=1.0),
          dict(rows=33, cols=2500, kind="powersgd", cap=3, sigma=0.05),    # 3 column chunks
          dict(rows=130, cols=1031, kind="powersgd", cap=2, sigma=0.1),    # unaligned rows
          dict(rows=9000, cols=40, kind="powersgd", cap=4, sigma=0.1)]     # tall: chunked P


class Pair:
    def __init__(self, layers, W):
        self.g = g = gce()
        self.t = t = g.Table(workloads.table_layers(layers))
        self.W = W
        self.bufs = {}
        for side in ("eager", "lazy"):
            b = dict(mem=torch.zeros((W, t.N), device="cuda"),
                     P=torch.zeros((W, max(4, t.P_per_worker)), device="cuda"),
                     Q=torch.zeros((W, max(4, t.Q_per_worker)), device="cuda"),
                     vals=torch.zeros((W, max(4, t.vals_per_worker)), device="cuda"),
                     ws=t.workspace(W, "powersgd"))
            g.powersgd_init_q(t, W, 5, b["Q"])
            self.bufs[side] = b
        self.lazy_rank = torch.zeros((W, t.L), dtype=torch.int32, device="cuda")

    def step(self, grad, ranks):
        kr = torch.tensor(ranks, dtype=torch.int32, device="cuda")
        e, z = self.bufs["eager"], self.bufs["lazy"]
        self.g.powersgd_step(self.t, self.W, grad, e["mem"], workloads.ETA, kr, e["P"], e["Q"],
                             e["vals"], None, e["ws"])
        self.g.powersgd_step_lazy(self.t, self.W, grad, z["mem"], workloads.ETA, kr, z["P"],
                                  z["Q"], z["vals"], self.lazy_rank, z["ws"])
        torch.cuda.synchronize()
        for name in ("P", "Q", "vals"):
            assert torch.equal(e[name].view(torch.int32), z[name].view(torch.int32)), name

    def materialize_and_compare(self):
        z = self.bufs["lazy"]
        self.g.materialize_memory(self.t, self.W, z["mem"], self.lazy_rank, z["ws"])
        torch.cuda.synchronize()
        assert torch.equal(self.bufs["eager"]["mem"].view(torch.int32), z["mem"].view(torch.int32))
        assert not torch.any(self.lazy_rank)


def test_lazy_equals_eager_bit_for_bit():
    need_gpu()
    W = 2
    pair = Pair(LAYERS, W)
    schedule = [[4, 0, 3, 2, 4], [2, 0, 3, 1, 4], [2, 0, 9, 2, 1],   # layer 2 skipped (9 > cap)
                [4, 0, 1, 2, 3], [1, 0, 3, 2, 4]]
    for s, ranks in enumerate(schedule):
        pair.step(workloads.gradients(LAYERS, W, 330, s), ranks)
        if s == 2:
            # the skipped layer kept its record; the others hold this step's rank
            lr = host(pair.lazy_rank)
            assert list(lr[0, [0, 2, 3, 4]]) == [2, 3, 2, 1]
            pair.materialize_and_compare()      # in the middle: the next step starts eager
    pair.materialize_and_compare()
    pair.materialize_and_compare()              # idempotent once materialised


def test_lazy_payload_follows_the_oracle():
    """Five lazy steps against the oracle's own trajectory: P and Q of every
    layer within 1e-4, DENSE payloads bit for bit, and the materialised
    memory within 1e-4 at the end."""
    need_gpu()
    g = gce()
    layers = LAYERS
    W = 1
    t = g.Table(workloads.table_layers(layers))
    mem = torch.zeros((W, t.N), device="cuda")
    P = torch.zeros((W, max(4, t.P_per_worker)), device="cuda")
    Q = torch.zeros((W, max(4, t.Q_per_worker)), device="cuda")
    vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
    ws = t.workspace(W, "powersgd")
    lazy = torch.zeros((W, t.L), dtype=torch.int32, device="cuda")
    g.powersgd_init_q(t, W, 7, Q)
    caps = [l["cap"] for l in layers]
    hQ = osteps.powersgd_init(layers, W, caps, 7)
    hmem = np.zeros((W, t.N), np.float32)
    for s in range(5):
        grad = workloads.gradients(layers, W, 331, s)
        expect = osteps.powersgd_step(layers, host(grad), hmem, workloads.ETA, caps, hQ,
                                      threads=4)
        g.powersgd_step_lazy(t, W, grad, mem, workloads.ETA, None, P, Q, vals, lazy, ws)
        torch.cuda.synchronize()
        hP, hQg, hv = host(P), host(Q), host(vals)
        for (w, l), e in expect.items():
            info = t.info[l]
            lay = layers[l]
            if lay["kind"] == "dense":
                o, n = info["val_offset"], info["n"]
                assert np.array_equal(bits(hv[w, o:o + n]), bits(e))
                continue
            rows, cols, cap = lay["rows"], lay["cols"], lay["cap"]
            P_ref, Mhat = e
            sl = slice(info["offset"], info["offset"] + info["n"])
            Mn = np.linalg.norm(hmem[w, sl].astype(np.float64) + Mhat.reshape(-1))
            Pg = hP[w, info["p_offset"]:info["p_offset"] + rows * cap].reshape(rows, cap)
            Qg = hQg[w, info["q_offset"]:info["q_offset"] + cols * cap].reshape(cols, cap)
            assert relerr(Pg, P_ref, 0.0) <= 1e-4, (s, l)
            assert relerr(Qg, hQ[(w, l)], Mn) <= 1e-4, (s, l)
    g.materialize_memory(t, W, mem, lazy, ws)
    torch.cuda.synchronize()
    hm = host(mem)
    for l, lay in enumerate(layers):
        info = t.info[l]
        sl = slice(info["offset"], info["offset"] + info["n"])
        if lay["kind"] == "dense":
            assert np.array_equal(bits(hm[0, sl]), bits(hmem[0, sl]))
        else:
            assert relerr(hm[0, sl], hmem[0, sl], np.linalg.norm(hmem[0, sl])) <= 1e-4, l


def test_lazy_equals_eager_on_a_large_layer():
    """A layer above 4 Mi elements (products in fp32 from the payload's
    factors, sums in fp64) next to a small one (fp64 products): the lazy
    step is the eager step bit for bit in both precisions."""
    need_gpu()
    layers = [dict(rows=4200, cols=1024, kind="powersgd", cap=4, sigma=0.03),
              dict(rows=64, cols=576, kind="powersgd", cap=2, sigma=0.04)]
    W = 1
    pair = Pair(layers, W)
    for s, ranks in enumerate([[4, 2], [2, 2], [3, 1]]):
        pair.step(workloads.gradients(layers, W, 332, s), ranks)
    pair.materialize_and_compare()
