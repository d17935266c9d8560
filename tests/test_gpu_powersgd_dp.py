"""GPU parity of powersgd_dp_step (data-parallel PowerSGD over the W
workers of one GPU) against the CPU oracle.

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Key results: PowerSGD is all-reduce compatible -- P and Q are
summed over the workers; the step is the single power iteration with a
shared warm start and each worker's own Mem-SGD memory ("Sparsified SGD
with Memory", Method).  Floating point: P, the shared Q, every worker's
memory and the decoded mean update satisfy ||X_gpu - X_ref||_F /
max(||X_ref||_F, ||M||_F) <= 1e-4 at every step; DENSE layers (the workers'
mean) are bit-exact.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, layer_slice, need_gpu, torch

pytestmark = pytest.mark.gpu
TOL = 1e-4


def relerr(a, b, scale):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), scale, 1e-30)


class DpRun:
    def __init__(self, layers, W, seed=0):
        self.g = gce()
        self.layers = layers
        self.W = W
        self.t = self.g.Table(workloads.table_layers(layers))
        t = self.t
        self.mem = torch.zeros((W, t.N), device="cuda")
        self.P = torch.zeros(max(4, t.P_per_worker), device="cuda")
        self.Q = torch.zeros(max(4, t.Q_per_worker), device="cuda")
        self.vals = torch.zeros(max(4, t.vals_per_worker), device="cuda")
        self.ws = t.workspace(W, "powersgd_dp")
        self.g.powersgd_init_q(t, 1, seed, self.Q)      # worker 0's start, shared
        self.hmem = np.zeros((W, t.N), np.float32)
        caps = [l["cap"] for l in layers]
        q0 = osteps.powersgd_init(layers, 1, caps, seed)
        self.hQ = {l: q for (w, l), q in q0.items()}

    def step(self, grad, eta, ranks=None):
        kt = None if ranks is None else torch.tensor(ranks, dtype=torch.int32, device="cuda")
        r = [l["cap"] for l in self.layers] if ranks is None else ranks
        hg = host(grad)
        M = (self.hmem + np.float32(eta) * hg).astype(np.float32)
        expect = osteps.powersgd_dp_step(self.layers, hg, self.hmem, eta, r, self.hQ, threads=8)
        Q_before = host(self.Q).copy()
        self.g.powersgd_dp_step(self.t, self.W, grad, self.mem, eta, kt, self.P, self.Q,
                                self.vals, self.ws)
        out = torch.zeros(self.t.N, device="cuda")
        self.g.decompress_accumulate(self.t, 1, self.vals, None, kt, self.P, self.Q, 1.0, out,
                                     self.t.workspace(1, "decompress"))
        torch.cuda.synchronize()
        hP, hQ, hm, hv, ho = (host(self.P), host(self.Q), host(self.mem), host(self.vals),
                              host(out))
        worst = 0.0
        for l, e in expect.items():
            lay = self.layers[l]
            ls = layer_slice(self.t, l)
            info = self.t.info[l]
            if lay["kind"] == "dense":
                n = info["n"]
                assert np.array_equal(bits(hv[info["val_offset"]:info["val_offset"] + n]),
                                      bits(e))
                assert np.array_equal(bits(hm[:, ls]), bits(self.hmem[:, ls]))
                assert np.array_equal(bits(ho[ls]), bits(e))
                continue
            rows, cols, cap = lay["rows"], lay["cols"], lay["cap"]
            rr = r[l]
            Mbar = np.linalg.norm(M[:, ls].astype(np.float64).mean(axis=0))
            P_gpu = hP[info["p_offset"]:info["p_offset"] + rows * cap].reshape(rows, cap)
            Q_gpu = hQ[info["q_offset"]:info["q_offset"] + cols * cap].reshape(cols, cap)
            Q_ref = self.hQ[l]
            upd = e[:, :rr].astype(np.float64) @ Q_ref[:, :rr].astype(np.float64).T
            errs = [relerr(P_gpu[:, :rr], e[:, :rr], 0.0),
                    relerr(Q_gpu[:, :rr], Q_ref[:, :rr], Mbar),
                    relerr(ho[ls], upd.reshape(-1), Mbar)]
            for w in range(self.W):
                errs.append(relerr(hm[w, ls], self.hmem[w, ls], np.linalg.norm(M[w, ls])))
            assert max(errs) <= TOL, (l, errs)
            worst = max(worst, max(errs))
            Q_prev = Q_before[info["q_offset"]:info["q_offset"] + cols * cap].reshape(cols, cap)
            assert np.array_equal(bits(Q_gpu[:, rr:]), bits(Q_prev[:, rr:]))
        return worst


def test_ragged_shapes_three_workers():
    need_gpu()
    layers = [dict(rows=64, cols=27, kind="powersgd", cap=4, sigma=0.2),
              dict(rows=7, cols=1500, kind="powersgd", cap=2, sigma=0.05),
              dict(rows=129, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=1025, cols=33, kind="powersgd", cap=4, sigma=0.1),
              dict(rows=5, cols=3, kind="powersgd", cap=1, sigma=1.0)]
    run = DpRun(layers, 3, seed=21)
    for s, ranks in enumerate([None, [2, 1, 0, 3, 1], [4, 2, 0, 1, 1]]):
        run.step(workloads.gradients(layers, 3, 600, s), 0.05, ranks)


def test_resnet18_rank2_four_workers():
    need_gpu()
    layers = workloads.resnet18_powersgd(2)
    run = DpRun(layers, 4, seed=22)
    for s in range(3):
        run.step(workloads.gradients(layers, 4, 2, s), workloads.ETA)


def test_tall_p_two_workers():
    need_gpu()
    layers = [dict(rows=20000, cols=96, kind="powersgd", cap=4, sigma=0.1),
              dict(rows=300, cols=40, kind="powersgd", cap=2, sigma=0.2)]
    run = DpRun(layers, 2, seed=23)
    for s in range(2):
        run.step(workloads.gradients(layers, 2, 601, s), 0.05)


def test_one_worker_is_the_replica_step_bit_for_bit():
    """W = 1: the data-parallel step and powersgd_step give the same bits."""
    need_gpu()
    g = gce()
    layers = [dict(rows=96, cols=200, kind="powersgd", cap=2, sigma=0.1),
              dict(rows=40, cols=1, kind="dense", cap=0, sigma=1.0)]
    t = g.Table(workloads.table_layers(layers))
    grad = workloads.gradients(layers, 1, 602, 0)
    mems = [torch.zeros((1, t.N), device="cuda") for _ in range(2)]
    Ps = [torch.zeros((1, t.P_per_worker), device="cuda") for _ in range(2)]
    Qs = [torch.zeros((1, t.Q_per_worker), device="cuda") for _ in range(2)]
    vs = [torch.zeros((1, t.vals_per_worker), device="cuda") for _ in range(2)]
    for Q in Qs:
        g.powersgd_init_q(t, 1, 3, Q)
    for s in range(2):
        g.powersgd_step(t, 1, grad, mems[0], 0.05, None, Ps[0], Qs[0], vs[0], None,
                        t.workspace(1, "powersgd"))
        g.powersgd_dp_step(t, 1, grad, mems[1], 0.05, None, Ps[1], Qs[1], vs[1],
                           t.workspace(1, "powersgd_dp"))
    torch.cuda.synchronize()
    for a, b in ((mems, "mem"), (Ps, "P"), (Qs, "Q"), (vs, "vals")):
        assert torch.equal(a[0].view(torch.int32), a[1].view(torch.int32)), b
