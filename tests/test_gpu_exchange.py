"""DataParallelStep (gradient_compression_error_b200.exchange) on one GPU as a
one-rank NCCL group, against the oracle.

The rank encodes with the native one-worker step, gathers its row through
NCCL (all_gather_into_tensor into the [world, vals_per_worker] buffers) and
decodes with the native kernels; the oracle runs the same one-worker step and
decode on the CPU.  Two steps, so the memory carried between them is checked
too.  The many-rank gather itself is covered by the gloo tests on CPU: this run
has one GPU, and ranks sharing one GPU are not run.
"""
import datetime
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT
from tests.helpers import need_gpu

pytestmark = pytest.mark.gpu

LAYERS = {
    "topk": [dict(rows=300, cols=41, kind="topk", cap=123, sigma=1.0),
             dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=70000, cols=1, kind="topk", cap=700, sigma=0.5)],
    "randk": [dict(rows=300, cols=41, kind="randk", cap=123, sigma=1.0),
              dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=70000, cols=1, kind="randk", cap=700, sigma=0.5)],
    "sign": [dict(rows=40, cols=100, kind="sign", cap=0, sigma=1.0),
             dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=9000, cols=1, kind="sign", cap=0, sigma=2.0)],
}
ETA = 0.05
SEED = 23


def _bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def _rank(port, method, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        from tests.helpers import gce
        g = gce()
        from gradient_compression_error_b200 import workloads
        from gradient_compression_error_b200.exchange import DataParallelStep
        from oracle import steps as osteps
        layers = LAYERS[method]
        k = [l["cap"] for l in layers]
        t = g.Table(workloads.table_layers(layers))
        step = DataParallelStep(t, method)
        mem = (0.1 * workloads.gradients(layers, 1, 941, 0)).contiguous()
        mem_h = mem.cpu().numpy()
        x = workloads.gradients(layers, 1, 942, 0)[0].contiguous()
        x_h = x.cpu().numpy()
        out = torch.zeros(t.N, device="cuda")
        for s in range(2):
            grad = workloads.gradients(layers, 1, 940, s)
            pay = osteps.sparse_step(layers, grad.cpu().numpy(), mem_h, np.float32(ETA), k,
                                     method=method, seed=SEED, step=s)
            step(grad, mem, ETA, out, seed=SEED, step=s)       # scale 1/world = 1
            torch.cuda.synchronize()
            res["sum%d" % s] = np.array_equal(
                _bits(out.cpu().numpy()), _bits(osteps.decompress(layers, 1, pay, np.float32(1.0))))
            res["mem%d" % s] = np.array_equal(_bits(mem.cpu().numpy()), _bits(mem_h))
            step.decode(x, 0.5, apply=True)                    # x -= 0.5 * sum
            x_h = osteps.apply_update(layers, 1, pay, np.float32(0.5), x_h)
            torch.cuda.synchronize()
            res["apply%d" % s] = np.array_equal(_bits(x.cpu().numpy()), _bits(x_h))
            if method == "sign":
                step.decode(out, 2.0, vote=True)
                torch.cuda.synchronize()
                res["vote%d" % s] = np.array_equal(
                    _bits(out.cpu().numpy()), _bits(osteps.vote(layers, 1, pay, np.float32(2.0))))
        res["status_clear"] = g.status(step.ws_step) == 0
        # PowerSGD has its own class, and a table takes only its own kind's step:
        # both refused on the host before any call
        rk = g.Table(workloads.table_layers([dict(rows=1000, cols=1, kind="randk", cap=10,
                                                  sigma=1.0)]))
        try:
            DataParallelStep(rk, "powersgd")
            res["powersgd_refused"] = False
        except ValueError:
            res["powersgd_refused"] = True
        try:
            DataParallelStep(rk, "topk")
            res["kind_mismatch_refused"] = False
        except ValueError:
            res["kind_mismatch_refused"] = True
        t.close()
        rk.close()
        res["completed"] = True
    finally:
        dist.destroy_process_group()
        q.put(res)


@pytest.mark.parametrize("method,port", [("topk", 29531), ("sign", 29532), ("randk", 29533)])
def test_one_rank_nccl_step_matches_the_oracle(method, port):
    need_gpu()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_rank, args=(port, method, q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0
    assert res.get("completed") and all(res.values()), res


# ---- PowerSGD and Accordion between ranks -------------------------------------------------
PS_LAYERS = [dict(rows=64, cols=576, kind="powersgd", cap=4, sigma=0.04),
             dict(rows=128, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=9000, cols=40, kind="powersgd", cap=2, sigma=0.1),    # tall P
             dict(rows=130, cols=1031, kind="powersgd", cap=3, sigma=0.03)]


def test_powersgd_split_at_its_two_sums_is_the_dp_step():
    """Three ranks of one worker each, run one after the other on one GPU: the
    four calls of the cut step with the rows concatenated where ranks would
    gather them give powersgd_dp_step over the three workers bit for bit (P,
    Q, every worker's memory, the DENSE means), over steps that change ranks.
    Source: "On the Utility of Gradient Compression ...", Key results."""
    need_gpu()
    import torch
    from tests.helpers import gce
    from gradient_compression_error_b200 import workloads
    g = gce()
    R = 3
    t = g.Table(workloads.table_layers(PS_LAYERS))
    npart = g.powersgd_dp_partials(t)
    f = dict(device="cuda")
    # the one-GPU step over all R workers
    mem_a = torch.zeros((R, t.N), **f)
    P_a = torch.zeros(max(4, t.P_per_worker), **f)
    Q_a = torch.zeros(max(4, t.Q_per_worker), **f)
    v_a = torch.zeros(max(4, t.vals_per_worker), **f)
    ws_a = t.workspace(R, "powersgd_dp")
    g.powersgd_init_q(t, 1, 3, Q_a)
    # the cut step: one workspace, memory, P and Q per rank (a rank's buffers
    # are its own allocations, 16-byte aligned as the calls require)
    mem_b = [torch.zeros((1, t.N), **f) for _ in range(R)]
    Ps = [torch.zeros(max(4, t.P_per_worker), **f) for _ in range(R)]
    Qs = [Q_a.clone() for _ in range(R)]
    wss = [t.workspace(1, "powersgd_dp") for _ in range(R)]
    vals_b = torch.zeros(max(4, t.vals_per_worker), **f)
    for s, ranks in enumerate([[4, 0, 2, 3], [2, 0, 1, 3], [3, 0, 2, 1]]):
        kr = torch.tensor(ranks, dtype=torch.int32, **f)
        grad = workloads.gradients(PS_LAYERS, R, 350, s)
        g.powersgd_dp_step(t, R, grad, mem_a, workloads.ETA, kr, P_a, Q_a, v_a, ws_a)
        prow = [torch.zeros((1, npart), dtype=torch.float64, **f) for _ in range(R)]
        vrow = [torch.zeros((1, max(4, t.vals_per_worker)), **f) for _ in range(R)]
        for r in range(R):
            g.powersgd_dp_encode(t, 1, grad[r:r + 1].clone(), mem_b[r], workloads.ETA, kr, Qs[r],
                                 prow[r], vrow[r], wss[r])
        pall, vall = torch.cat(prow), torch.cat(vrow)          # the gathers
        qrow = [torch.zeros((1, max(4, t.Q_per_worker)), **f) for _ in range(R)]
        for r in range(R):
            g.powersgd_dp_orthogonalize(t, R, kr, pall, Ps[r], wss[r])
            g.powersgd_dp_project(t, 1, mem_b[r], kr, qrow[r], wss[r])
        qall = torch.cat(qrow)
        for r in range(R):
            g.powersgd_dp_mean(t, R, kr, qall, Qs[r], vall, vals_b)
        torch.cuda.synchronize()
        for r in range(R):
            assert torch.equal(Ps[r].view(torch.int32), P_a.view(torch.int32)), (s, r)
            assert torch.equal(Qs[r].view(torch.int32), Q_a.view(torch.int32)), (s, r)
        assert torch.equal(torch.cat(mem_b).view(torch.int32), mem_a.view(torch.int32)), s
        assert torch.equal(vals_b.view(torch.int32), v_a.view(torch.int32)), s


def test_accordion_sumsq_then_decide_is_select():
    """accordion_sumsq + accordion_decide on one gradient is accordion_select
    bit for bit (levels, norms, k), and with the sums of two gradients added
    (a two-rank all-reduce) the decision follows the oracle's on the norm of
    both gradients.  Source: "Accordion ...", Method."""
    need_gpu()
    import torch
    import oracle
    from tests.helpers import gce, host
    from gradient_compression_error_b200 import workloads
    g = gce()
    layers = workloads.vgg19("topk", 100000)
    t = g.Table(workloads.table_layers(layers))
    L = t.L
    f = dict(device="cuda")

    def state():
        st = dict(prev=torch.empty(L, dtype=torch.float64, **f),
                  level=torch.empty(L, dtype=torch.int32, **f),
                  cur=torch.zeros(L, dtype=torch.float64, **f),
                  k=torch.zeros(L, dtype=torch.int32, **f))
        g.accordion_init(t, st["prev"], st["level"])
        return st

    a, b, c = state(), state(), state()
    ws = t.workspace(1, "accordion")
    sumsq = torch.zeros(L, dtype=torch.float64, **f)
    sumsq2 = torch.zeros(L, dtype=torch.float64, **f)
    offs, _ = __import__("oracle.steps", fromlist=["layer_offsets"]).layer_offsets(layers)
    prev = [-1.0] * L
    for s in range(0, 200, 10):
        gr = workloads.gradients(layers, 2, 3, s, scale=workloads.vgg19_scale(s))
        g.accordion_select(t, gr[0], s, 10, 0.5, 100000, 10000, a["prev"], a["level"], a["cur"],
                           a["k"], ws)
        g.accordion_sumsq(t, gr[0], sumsq, ws)
        g.accordion_decide(t, sumsq, s, 10, 0.5, 100000, 10000, b["prev"], b["level"], b["cur"],
                           b["k"])
        g.accordion_sumsq(t, gr[1], sumsq2, ws)
        both = sumsq + sumsq2                                    # a two-rank all-reduce
        g.accordion_decide(t, both, s, 10, 0.5, 100000, 10000, c["prev"], c["level"], c["cur"],
                           c["k"])
        torch.cuda.synchronize()
        for name in ("prev", "level", "cur", "k"):
            assert torch.equal(a[name], b[name]), (s, name)
        hg = host(gr)
        lv = host(c["level"])
        for l, lay in enumerate(layers):
            if lay["kind"] == "dense":
                continue
            n = lay["rows"] * lay["cols"]
            s_all = oracle.layer_norm(np.concatenate([hg[0, offs[l]:offs[l] + n],
                                                      hg[1, offs[l]:offs[l] + n]]))
            assert lv[l] == oracle.accordion_decide(prev[l], s_all, 0.5), (s, l)
            prev[l] = s_all


def _ps_rank1(port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        from tests.helpers import gce
        g = gce()
        from gradient_compression_error_b200 import workloads
        from gradient_compression_error_b200.exchange import (AccordionAcrossRanks,
                                                              PowerSgdDataParallelStep)
        t = g.Table(workloads.table_layers(PS_LAYERS))
        step = PowerSgdDataParallelStep(t, seed=3)
        acc = AccordionAcrossRanks(t, 10, 0.5, 2, 1)
        mem = torch.zeros((1, t.N), device="cuda")
        mem_r = torch.zeros((1, t.N), device="cuda")
        P_r = torch.zeros_like(step.P)
        Q_r = torch.zeros_like(step.Q)
        g.powersgd_init_q(t, 1, 3, Q_r)
        v_r = torch.zeros_like(step.vals)
        ws_r = t.workspace(1, "powersgd_dp")
        prev = torch.empty(t.L, dtype=torch.float64, device="cuda")
        level = torch.empty(t.L, dtype=torch.int32, device="cuda")
        cur = torch.zeros(t.L, dtype=torch.float64, device="cuda")
        kr = torch.zeros(t.L, dtype=torch.int32, device="cuda")
        ws_a = t.workspace(1, "accordion")
        g.accordion_init(t, prev, level)
        out = torch.zeros(t.N, device="cuda")
        out_r = torch.zeros(t.N, device="cuda")
        ws_d = t.workspace(1, "decompress")
        ok = True
        for s in range(25):
            grad = workloads.gradients(PS_LAYERS, 1, 351, s, scale=0.1 if s >= 20 else 1.0)
            k = acc(grad[0], s)
            g.accordion_select(t, grad[0], s, 10, 0.5, 2, 1, prev, level, cur, kr, ws_a)
            step(grad, mem, workloads.ETA, k)
            step.decode(out, k)
            g.powersgd_dp_step(t, 1, grad, mem_r, workloads.ETA, kr, P_r, Q_r, v_r, ws_r)
            g.decompress_accumulate(t, 1, v_r, None, kr, P_r, Q_r, 1.0, out_r, ws_d)
            torch.cuda.synchronize()
            ok &= torch.equal(k, kr)
            for x, y in ((step.P, P_r), (step.Q, Q_r), (step.vals, v_r), (mem, mem_r), (out, out_r)):
                ok &= torch.equal(x.view(torch.int32), y.view(torch.int32))
        res["matches"] = bool(ok)
        res["completed"] = True
        t.close()
    finally:
        dist.destroy_process_group()
        q.put(res)


def test_one_rank_nccl_powersgd_and_accordion_between_ranks():
    """PowerSgdDataParallelStep and AccordionAcrossRanks as a one-rank NCCL
    group: the gathers and the all-reduce run through NCCL; P, Q, DENSE means,
    memory, decode and Accordion's k equal the one-GPU calls bit for bit."""
    need_gpu()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_ps_rank1, args=(29534, q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0
    assert res.get("completed") and all(res.values()), res


# ---- grouped exchange and rand-k with shared keys ------------------------------------------
GROUP_LAYERS = {
    "topk": [dict(rows=300, cols=40, kind="topk", cap=120, sigma=1.0),
             dict(rows=76, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=70000, cols=1, kind="topk", cap=700, sigma=0.5),
             dict(rows=64, cols=64, kind="topk", cap=41, sigma=2.0),
             dict(rows=5, cols=3, kind="dense", cap=0, sigma=1.0)],
    "sign": [dict(rows=40, cols=100, kind="sign", cap=0, sigma=1.0),
             dict(rows=76, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=9000, cols=1, kind="sign", cap=0, sigma=2.0),
             dict(rows=33, cols=1, kind="sign", cap=0, sigma=1.0)],
}


def _group_rank(port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        from tests.helpers import gce
        g = gce()
        from gradient_compression_error_b200 import workloads
        from gradient_compression_error_b200.exchange import (DataParallelStep,
                                                              GroupedDataParallelStep)
        for method, layers in GROUP_LAYERS.items():
            descs = workloads.table_layers(layers)
            t = g.Table(descs)
            whole = DataParallelStep(t, method)
            grouped = GroupedDataParallelStep(descs, method, cuts=[2, 3])
            mem_a = (0.1 * workloads.gradients(layers, 1, 951, 0)).contiguous()
            mem_b = mem_a.clone()
            out_a = torch.zeros(t.N, device="cuda")
            out_b = torch.full((t.N,), 3.0, device="cuda")
            k = None
            if method == "topk":
                k = torch.tensor([60, 0, 700, 20, 0], dtype=torch.int32, device="cuda")
            for s in range(2):
                grad = workloads.gradients(layers, 1, 950, s)
                whole(grad, mem_a, ETA, out_a, k=k)
                grouped(grad, mem_b, ETA, out_b, k=k)
                torch.cuda.synchronize()
                res["%s_out%d" % (method, s)] = torch.equal(out_a.view(torch.int32),
                                                            out_b.view(torch.int32))
                res["%s_mem%d" % (method, s)] = torch.equal(mem_a.view(torch.int32),
                                                            mem_b.view(torch.int32))
            try:   # a group must start at a multiple of 4 elements (here at element 7)
                odd = [dict(rows=7, cols=1, kind=method, cap=2 if method == "topk" else 0),
                       dict(rows=100, cols=1, kind=method, cap=5 if method == "topk" else 0)]
                GroupedDataParallelStep(workloads.table_layers(odd), method, cuts=[1])
                res["%s_misaligned_refused" % method] = False
            except ValueError:
                res["%s_misaligned_refused" % method] = True
            t.close()
        # rand-k with shared keys: worker 0's keys on every rank, values
        # alone gathered; the same as the native one-worker step as worker 0
        layers = LAYERS["randk"]
        t = g.Table(workloads.table_layers(layers))
        shared = DataParallelStep(t, "randk", shared_keys=True)
        mem_a = (0.1 * workloads.gradients(layers, 1, 953, 0)).contiguous()
        mem_b = mem_a.clone()
        vals = torch.zeros((1, max(4, t.vals_per_worker)), device="cuda")
        idx = torch.zeros((1, max(4, t.vals_per_worker)), dtype=torch.int32, device="cuda")
        ws, wsd = t.workspace(1, "randk"), t.workspace(1, "decompress")
        out_a = torch.zeros(t.N, device="cuda")
        out_b = torch.zeros(t.N, device="cuda")
        for s in range(2):
            grad = workloads.gradients(layers, 1, 952, s)
            shared(grad, mem_a, ETA, out_a, seed=SEED, step=s)
            g.ef_randk_step_at(t, 0, 1, grad, mem_b, ETA, None, SEED, s, vals, idx, ws)
            g.decompress_accumulate(t, 1, vals, idx, None, None, None, 1.0, out_b, wsd)
            torch.cuda.synchronize()
            res["shared_out%d" % s] = torch.equal(out_a.view(torch.int32), out_b.view(torch.int32))
            res["shared_mem%d" % s] = torch.equal(mem_a.view(torch.int32), mem_b.view(torch.int32))
        try:
            DataParallelStep(g.Table(workloads.table_layers(GROUP_LAYERS["topk"])), "topk",
                             shared_keys=True)
            res["shared_keys_topk_refused"] = False
        except ValueError:
            res["shared_keys_topk_refused"] = True
        t.close()
        res["completed"] = True
    finally:
        dist.destroy_process_group()
        q.put(res)


def test_one_rank_nccl_grouped_exchange_and_shared_randk_keys():
    """GroupedDataParallelStep (each layer group's gather started right after
    the group is encoded) gives the ungrouped step's aggregate and memory bit
    for bit, for top-k with per-layer k (one layer skipped) and for signSGD;
    misaligned groups are refused.  rand-k with shared keys equals the native
    step as worker 0 plus the decode ("On the Utility of Gradient
    Compression", Method: all-reduce-compatible exchange)."""
    need_gpu()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_group_rank, args=(29538, q))
    p.start()
    res = q.get(timeout=300)
    p.join(timeout=60)
    assert p.exitcode == 0
    assert res.get("completed") and all(res.values()), res
