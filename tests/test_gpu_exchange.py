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
        # PowerSGD is not exchanged, and a table takes only its own kind's step:
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
