"""GPU parity of powersgd_step against the CPU oracle.

PowerSGD is named on the pages ("Accordion ...", Method / Key results; "On
the Utility of Gradient Compression ...", Method / Key results) with ranks
1, 2 and 4; the step is the single power iteration with a warm-started Q
and the Mem-SGD memory ("Sparsified SGD with Memory", Method).  Floating
point: every output X in {P, Q, P Q^T, memory} satisfies
||X_gpu - X_ref||_F / max(||X_ref||_F, ||M||_F) <= 1e-4, per step over the
whole trajectory; the uncompressed (DENSE) layers and the shared Q
initialisation are bit-exact.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
import oracle
from tests.helpers import bits, gce, host, layer_slice, need_gpu, torch

pytestmark = pytest.mark.gpu
TOL = 1e-4


def relerr(a, b, scale):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), scale, 1e-30)


class PsRun:
    def __init__(self, layers, W, seed=0):
        self.g = gce()
        self.layers = layers
        self.W = W
        self.t = self.g.Table(workloads.table_layers(layers))
        t = self.t
        self.mem = torch.zeros((W, t.N), device="cuda")
        self.P = torch.zeros((W, max(4, t.P_per_worker)), device="cuda")
        self.Q = torch.zeros((W, max(4, t.Q_per_worker)), device="cuda")
        self.vals = torch.zeros((W, max(4, t.vals_per_worker)), device="cuda")
        self.out = torch.zeros((W, t.N), device="cuda")
        self.ws = t.workspace(W, "powersgd")
        self.g.powersgd_init_q(t, W, seed, self.Q)
        self.hmem = np.zeros((W, t.N), np.float32)
        caps = [l["cap"] for l in layers]
        self.hQ = osteps.powersgd_init(layers, W, caps, seed)
        hq = host(self.Q)
        for (w, l), q in self.hQ.items():
            o = t.info[l]["q_offset"]
            assert np.array_equal(bits(hq[w, o:o + q.size]), bits(q.reshape(-1))), "Q init"

    def step(self, grad, eta, ranks=None, full=True):
        """One step on both sides; the oracle keeps its own trajectory.  P, Q
        and DENSE payloads are compared every step; the memory and P Q^T
        (whole-layer arrays) when `full`."""
        kt = None if ranks is None else torch.tensor(ranks, dtype=torch.int32, device="cuda")
        r = [l["cap"] for l in self.layers] if ranks is None else ranks
        expect = osteps.powersgd_step(self.layers, host(grad), self.hmem, eta, r, self.hQ,
                                      threads=8)
        Q_before = host(self.Q).copy()
        self.g.powersgd_step(self.t, self.W, grad, self.mem, eta, kt, self.P, self.Q, self.vals,
                             self.out, self.ws)
        torch.cuda.synchronize()
        hP, hQ, hv = host(self.P), host(self.Q), host(self.vals)
        hm, ho = (host(self.mem), host(self.out)) if full else (None, None)
        worst = 0.0
        for (w, l), e in expect.items():
            lay = self.layers[l]
            ls = layer_slice(self.t, l)
            info = self.t.info[l]
            if lay["kind"] == "dense":
                n = info["n"]
                assert np.array_equal(bits(hv[w, info["val_offset"]:info["val_offset"] + n]), bits(e))
                if full:
                    assert np.array_equal(bits(hm[w, ls]), bits(self.hmem[w, ls]))
                continue
            rows, cols, cap = lay["rows"], lay["cols"], lay["cap"]
            rr = r[l]
            P_ref, Mhat_ref = e
            Q_ref = self.hQ[(w, l)]
            Mfull = np.linalg.norm(self.hmem[w, ls].astype(np.float64) + Mhat_ref.reshape(-1))
            P_gpu = hP[w, info["p_offset"]:info["p_offset"] + rows * cap].reshape(rows, cap)
            Q_gpu = hQ[w, info["q_offset"]:info["q_offset"] + cols * cap].reshape(cols, cap)
            errs = [relerr(P_gpu[:, :rr], P_ref[:, :rr], 0.0),
                    relerr(Q_gpu[:, :rr], Q_ref[:, :rr], Mfull)]
            if full:
                errs += [relerr(ho[w, ls], Mhat_ref.reshape(-1), Mfull),
                         relerr(hm[w, ls], self.hmem[w, ls], Mfull)]
            assert max(errs) <= TOL, (w, l, errs)
            worst = max(worst, max(errs))
            # columns >= r are left as they were (the GPU's own previous values)
            Q_prev = Q_before[w, info["q_offset"]:info["q_offset"] + cols * cap].reshape(cols, cap)
            assert np.array_equal(bits(Q_gpu[:, rr:]), bits(Q_prev[:, rr:]))
        return worst


def test_ragged_shapes_single_and_multi_step():
    need_gpu()
    layers = [dict(rows=64, cols=27, kind="powersgd", cap=4, sigma=0.2),
              dict(rows=100, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=33, cols=2500, kind="powersgd", cap=3, sigma=0.05),   # 3 column chunks
              dict(rows=130, cols=1031, kind="powersgd", cap=1, sigma=0.1),   # unaligned rows
              dict(rows=4, cols=4, kind="powersgd", cap=4, sigma=1.0)]         # full rank
    run = PsRun(layers, 2, seed=3)
    for s in range(4):
        run.step(workloads.gradients(layers, 2, 301, s), 0.05)


def test_full_rank_reconstructs_and_memory_empties():
    need_gpu()
    layers = [dict(rows=3, cols=7, kind="powersgd", cap=3, sigma=1.0),
              dict(rows=4, cols=4, kind="powersgd", cap=4, sigma=1.0)]
    run = PsRun(layers, 1)
    run.step(workloads.gradients(layers, 1, 302, 0), 1.0)
    assert float(run.mem.abs().max()) < 1e-5


def test_rank_changes_between_steps():
    need_gpu()
    layers = [dict(rows=256, cols=2304, kind="powersgd", cap=4, sigma=0.02),
              dict(rows=64, cols=576, kind="powersgd", cap=4, sigma=0.04)]
    run = PsRun(layers, 1, seed=9)
    for s, ranks in enumerate([[4, 4], [2, 2], [2, 4], [4, 2]]):
        run.step(workloads.gradients(layers, 1, 303, s), 0.05, ranks)


def test_dense_out_equals_decoder():
    need_gpu()
    layers = [dict(rows=128, cols=1152, kind="powersgd", cap=2, sigma=0.03),
              dict(rows=256, cols=1, kind="dense", cap=0, sigma=1.0)]
    run = PsRun(layers, 1)
    run.step(workloads.gradients(layers, 1, 304, 0), 0.05)
    g = run.g
    dec = torch.zeros(run.t.N, device="cuda")
    g.decompress_accumulate(run.t, 1, run.vals, None, None, run.P, run.Q, 1.0, dec,
                            run.t.workspace(1, "decompress"))
    o = run.t.info[0]
    n0 = o["n"]
    assert torch.equal(dec[:n0].view(torch.int32), run.out[0, :n0].view(torch.int32))


def test_resnet18_rank2_ten_steps():
    """ResNet-18-shaped layers, rank 2, warm-started Q, 1-D layers sent whole,
    10 steps."""
    need_gpu()
    layers = workloads.resnet18_powersgd(2)
    assert workloads.total_elements(layers) == 12541440
    run = PsRun(layers, 1, seed=2)
    for s in range(10):
        run.step(workloads.gradients(layers, 1, 2, s), workloads.ETA)


def test_square_sweep_point_rank4():
    need_gpu()
    layers = workloads.sweep(22, "powersgd", rank=4)     # 2048 x 2048
    run = PsRun(layers, 1, seed=5)
    for s in range(2):
        run.step(workloads.gradients(layers, 1, 5, s), workloads.ETA)


def test_rank_one_matrix_recovered():
    need_gpu()
    g = gce()
    layers = [dict(rows=300, cols=200, kind="powersgd", cap=1, sigma=1.0)]
    t = g.Table(workloads.table_layers(layers))
    u = torch.randn(300, 1, device="cuda", generator=torch.Generator("cuda").manual_seed(1))
    v = torch.randn(1, 200, device="cuda", generator=torch.Generator("cuda").manual_seed(2))
    M = (u @ v).reshape(1, -1).contiguous()
    mem = M.clone()
    P = torch.zeros((1, t.P_per_worker), device="cuda")
    Q = torch.zeros((1, t.Q_per_worker), device="cuda")
    out = torch.zeros_like(M)
    g.powersgd_init_q(t, 1, 0, Q)
    g.powersgd_step(t, 1, torch.zeros_like(M), mem, 1.0, None, P, Q, None, out,
                    t.workspace(1, "powersgd"))
    torch.cuda.synchronize()
    assert float((out - M).norm() / M.norm()) < 1e-5
    assert float(mem.abs().max()) < 1e-5 * float(M.abs().max())


def test_tall_p_is_orthonormalised_over_many_blocks():
    """P taller than 8192 rows takes the multi-block Gram-Schmidt; ranks vary."""
    need_gpu()
    layers = [dict(rows=20000, cols=96, kind="powersgd", cap=4, sigma=0.1),
              dict(rows=16384, cols=1024, kind="powersgd", cap=2, sigma=0.03),
              dict(rows=300, cols=40, kind="powersgd", cap=4, sigma=0.2)]
    run = PsRun(layers, 2, seed=11)
    for s, ranks in enumerate([None, [2, 1, 3], [3, 2, 4]]):
        run.step(workloads.gradients(layers, 2, 305, s), 0.05, ranks)
