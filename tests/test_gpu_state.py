"""All step state is caller-owned buffers: checkpoint / resume and CUDA-graph
replay give the same bits as running straight through.

Top-k and decode are bit-exact operations, so the trajectories must match
bit for bit; PowerSGD and Accordion state (memory, Q, previous norm, level)
is saved and restored the same way.
"""
import io

import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from oracle import steps as osteps
from tests.helpers import bits, gce, host, need_gpu, torch

pytestmark = pytest.mark.gpu


def topk_buffers(g, t, W):
    return dict(mem=torch.zeros((W, t.N), device="cuda"),
                vals=torch.zeros((W, t.vals_per_worker), device="cuda"),
                idx=torch.zeros((W, t.vals_per_worker), dtype=torch.int32, device="cuda"),
                ws=t.workspace(W, "topk"), out=torch.zeros(t.N, device="cuda"),
                wsd=t.workspace(W, "decompress"))


def topk_step(g, t, W, b, grad):
    g.ef_topk_step(t, W, grad, b["mem"], 0.05, None, b["vals"], b["idx"], b["ws"])
    g.decompress_accumulate(t, W, b["vals"], b["idx"], None, None, None, 1.0, b["out"], b["wsd"])


def test_topk_checkpoint_resume_is_bit_identical():
    need_gpu()
    g = gce()
    layers = [dict(rows=300, cols=700, kind="topk", cap=2100, sigma=1.0),
              dict(rows=5000, cols=1, kind="topk", cap=50, sigma=1.0)]
    W, T, cut = 3, 6, 3
    t = g.Table(workloads.table_layers(layers))
    grads = [workloads.gradients(layers, W, 401, s) for s in range(T)]
    a = topk_buffers(g, t, W)
    for s in range(T):
        topk_step(g, t, W, a, grads[s])
    b = topk_buffers(g, t, W)
    for s in range(cut):
        topk_step(g, t, W, b, grads[s])
    buf = io.BytesIO()
    torch.save({"mem": b["mem"].cpu()}, buf)            # the memory is the only state
    buf.seek(0)
    c = topk_buffers(g, t, W)                            # fresh buffers and workspace
    c["mem"].copy_(torch.load(buf)["mem"].cuda())
    for s in range(cut, T):
        topk_step(g, t, W, c, grads[s])
    torch.cuda.synchronize()
    for key in ("mem", "vals", "idx", "out"):
        assert torch.equal(a[key].view(torch.int32), c[key].view(torch.int32)), key


def test_powersgd_and_accordion_checkpoint_resume():
    need_gpu()
    g = gce()
    layers = workloads.vgg19("powersgd", 4)[:6]
    W, T, cut = 1, 24, 11
    t = g.Table(workloads.table_layers(layers))
    L = len(layers)
    grads = [workloads.gradients(layers, W, 402, s, scale=workloads.vgg19_scale(6 * s))
             for s in range(T)]

    def fresh():
        st = dict(mem=torch.zeros((W, t.N), device="cuda"),
                  P=torch.zeros((W, t.P_per_worker), device="cuda"),
                  Q=torch.zeros((W, t.Q_per_worker), device="cuda"),
                  vals=torch.zeros((W, t.vals_per_worker), device="cuda"),
                  prev=torch.empty(L, dtype=torch.float64, device="cuda"),
                  level=torch.empty(L, dtype=torch.int32, device="cuda"),
                  kr=torch.zeros(L, dtype=torch.int32, device="cuda"))
        g.powersgd_init_q(t, W, 7, st["Q"])
        g.accordion_init(t, st["prev"], st["level"])
        return st

    def step(st, s, wsp, wsa):
        g.accordion_select(t, grads[s][0], s, 5, 0.5, 4, 2, st["prev"], st["level"], None,
                           st["kr"], wsa)
        g.powersgd_step(t, W, grads[s], st["mem"], 0.05, st["kr"], st["P"], st["Q"], st["vals"],
                        None, wsp)

    wsp, wsa = t.workspace(W, "powersgd"), t.workspace(1, "accordion")
    a = fresh()
    for s in range(T):
        step(a, s, wsp, wsa)
    b = fresh()
    for s in range(cut):
        step(b, s, wsp, wsa)
    buf = io.BytesIO()
    torch.save({k: v.cpu() for k, v in b.items() if k in ("mem", "Q", "prev", "level")}, buf)
    buf.seek(0)
    saved = torch.load(buf)
    c = fresh()
    for k, v in saved.items():
        c[k].copy_(v.cuda())
    for s in range(cut, T):
        step(c, s, t.workspace(W, "powersgd"), t.workspace(1, "accordion"))
    torch.cuda.synchronize()
    for key in ("mem", "P", "Q", "vals", "prev", "level", "kr"):
        x, y = a[key], c[key]
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), key


def test_cuda_graph_replay_matches_eager():
    """One top-k step + decode captured in a CUDA graph replays to the same
    bits as eager launches (the step allocates nothing and never syncs)."""
    need_gpu()
    g = gce()
    layers = workloads.bert_base_topk()[:20]
    W = 4
    t = g.Table(workloads.table_layers(layers))
    grads = [workloads.gradients(layers, W, 403, s) for s in range(3)]
    e = topk_buffers(g, t, W)
    for s in range(3):
        topk_step(g, t, W, e, grads[s])
    c = topk_buffers(g, t, W)
    static_grad = grads[0].clone()
    topk_step(g, t, W, c, static_grad)                    # warm-up outside the capture
    c["mem"].zero_()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        topk_step(g, t, W, c, static_grad)
    for s in range(3):
        static_grad.copy_(grads[s])
        graph.replay()
    torch.cuda.synchronize()
    for key in ("mem", "vals", "idx", "out"):
        assert torch.equal(e[key].view(torch.int32), c[key].view(torch.int32)), key
    del graph


def test_decode_of_many_workers_uses_the_general_path():
    """More than 8 PowerSGD workers: the element-wise decode path; checked
    against the oracle's low-rank sum."""
    need_gpu()
    g = gce()
    layers = [dict(rows=40, cols=300, kind="powersgd", cap=3),
              dict(rows=64, cols=1, kind="dense", cap=0)]
    W = 11
    t = g.Table(layers)
    rng = np.random.default_rng(0)
    P = rng.standard_normal((W, t.P_per_worker)).astype(np.float32)
    Q = rng.standard_normal((W, t.Q_per_worker)).astype(np.float32)
    vals = rng.standard_normal((W, t.vals_per_worker)).astype(np.float32)
    out = torch.zeros(t.N, device="cuda")
    g.decompress_accumulate(t, W, torch.from_numpy(vals).cuda(), None, None,
                            torch.from_numpy(P).cuda(), torch.from_numpy(Q).cuda(), 0.5, out,
                            t.workspace(W, "decompress"))
    pay = {}
    for w in range(W):
        i0, i1 = t.info[0], t.info[1]
        pay[(w, 0)] = (P[w, i0["p_offset"]:i0["p_offset"] + 40 * 3].reshape(40, 3),
                       Q[w, i0["q_offset"]:i0["q_offset"] + 300 * 3].reshape(300, 3))
        pay[(w, 1)] = vals[w, i1["val_offset"]:i1["val_offset"] + 64]
    expect = osteps.decompress(layers, W, pay, 0.5, rank_per_layer=[3, 0])
    got = host(out)
    assert np.array_equal(bits(got[12000:]), bits(expect[12000:]))     # dense: exact
    assert np.max(np.abs(got[:12000] - expect[:12000])) < 1e-5 * np.max(np.abs(expect[:12000]))
