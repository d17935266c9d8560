"""Payload exchange between data-parallel ranks (gradient_compression_error_b200.exchange),
run as gloo ranks on CPU.

Each rank encodes its own worker's gradient with the oracle (that worker's
units alone), packs the payload into one row, and gathers the rows through
PayloadExchange.  The gathered payloads must equal, bit for bit, those of the
oracle's W-worker step on one process, and so must their sum and (signSGD)
majority-vote aggregates.  This pins the claim the exchange rests on: one
worker per rank plus a rank-order gather is the W-replica step.  The packing
below is this test's own; PayloadExchange moves rows without reading them.
"""
import datetime
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT

LAYERS = {
    "topk": [dict(rows=300, cols=41, kind="topk", cap=123, sigma=1.0),
             dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=5000, cols=1, kind="topk", cap=50, sigma=0.5)],
    "randk": [dict(rows=300, cols=41, kind="randk", cap=123, sigma=1.0),
              dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=5000, cols=1, kind="randk", cap=50, sigma=0.5)],
    "sign": [dict(rows=40, cols=100, kind="sign", cap=0, sigma=1.0),
             dict(rows=77, cols=1, kind="dense", cap=0, sigma=1.0),
             dict(rows=1000, cols=1, kind="sign", cap=0, sigma=2.0)],
}
ETA = np.float32(0.05)
SEED, STEP = 41, 3


def _slots(lay):
    n = lay["rows"] * lay["cols"]
    if lay["kind"] == "dense":
        return n
    if lay["kind"] == "sign":
        return 1 + (n + 31) // 32
    return lay["cap"]


def _pack(layers, pay, w):
    """Worker w's payload as one float32 row and one int32 row."""
    n = sum(_slots(l) for l in layers)
    vals = np.zeros(n, np.float32)
    idx = np.zeros(n, np.int32)
    o = 0
    for l, lay in enumerate(layers):
        p = pay[(w, l)]
        if lay["kind"] == "dense":
            vals[o:o + len(p)] = p
        elif lay["kind"] == "sign":
            sc, words = p
            vals[o] = sc
            vals[o + 1:o + 1 + len(words)] = np.asarray(words, np.uint32).view(np.float32)
        else:
            v, i = p
            vals[o:o + len(v)] = v
            idx[o:o + len(i)] = i
        o += _slots(lay)
    return vals, idx


def _unpack(layers, vals, idx, w, out):
    o = 0
    for l, lay in enumerate(layers):
        s = _slots(lay)
        if lay["kind"] == "dense":
            out[(w, l)] = vals[o:o + s].copy()
        elif lay["kind"] == "sign":
            out[(w, l)] = (np.float32(vals[o]), vals[o + 1:o + s].view(np.uint32).copy())
        else:
            out[(w, l)] = (vals[o:o + s].copy(), idx[o:o + s].copy())
        o += s


def _same_bits(a, b):
    """Equal payloads: every array (or tuple member) equal bit for bit."""
    if isinstance(b, tuple):
        return len(a) == len(b) and all(_same_bits(x, y) for x, y in zip(a, b))
    a, b = np.atleast_1d(np.asarray(a)), np.atleast_1d(np.asarray(b))
    return a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))


def _inputs(layers, W):
    from gradient_compression_error_b200 import workloads
    grad = workloads.gradients(layers, W, 930, 0, device="cpu").numpy()
    mem = (0.1 * workloads.gradients(layers, W, 931, 0, device="cpu")).numpy()
    return grad, mem


def _rank(rank, world, port, method, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from gradient_compression_error_b200.exchange import PayloadExchange
    from oracle import steps as osteps
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        layers = LAYERS[method]
        k = [l["cap"] for l in layers]
        grad, mem = _inputs(layers, world)
        # this rank: worker `rank` alone (its units only; rand-k's generator
        # takes the job-wide worker index)
        m1 = mem.copy()
        pay1 = osteps.sparse_step(layers, grad, m1, ETA, k, method=method, seed=SEED, step=STEP,
                                  units=[(rank, l) for l in range(len(layers))])
        v, i = _pack(layers, pay1, rank)
        sparse = method != "sign"
        ex = PayloadExchange(len(v), sparse, "cpu")
        # a row of the wrong size is refused on every rank before any collective
        try:
            ex.gather(torch.zeros(len(v) + 1), torch.zeros(len(v) + 1, dtype=torch.int32))
            refused = False
        except ValueError:
            refused = True
        gv, gi = ex.gather(torch.from_numpy(v), torch.from_numpy(i) if sparse else None)
        gathered = {}
        for w in range(world):
            _unpack(layers, gv[w].numpy(), gi[w].numpy() if gi is not None else None, w, gathered)
        # the same W workers on one process
        mW = mem.copy()
        payW = osteps.sparse_step(layers, grad, mW, ETA, k, method=method, seed=SEED, step=STEP)
        same_payload = all(_same_bits(gathered[u], payW[u]) for u in payW)
        same_mem = np.array_equal(m1[rank].view(np.uint32), mW[rank].view(np.uint32))
        scale = np.float32(1.0 / world)
        s1 = osteps.decompress(layers, world, gathered, scale).view(np.uint32)
        sW = osteps.decompress(layers, world, payW, scale).view(np.uint32)
        same_sum = np.array_equal(s1, sW)
        same_vote = True
        if method == "sign":
            same_vote = np.array_equal(osteps.vote(layers, world, gathered, 1.0).view(np.uint32),
                                       osteps.vote(layers, world, payW, 1.0).view(np.uint32))
        rows_in_rank_order = all(np.array_equal(gv[w].numpy().view(np.uint32),
                                                _pack(layers, payW, w)[0].view(np.uint32))
                                 for w in range(world))
        dist.barrier()
        q.put((rank, dict(refused=refused, same_payload=same_payload, same_mem=same_mem,
                          same_sum=same_sum, same_vote=same_vote,
                          rows_in_rank_order=rows_in_rank_order)))
    finally:
        dist.destroy_process_group()


def _run(method, world, port):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, method, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


@pytest.mark.parametrize("method,world,port", [("topk", 2, 29521), ("sign", 3, 29522),
                                               ("randk", 2, 29523)])
def test_one_worker_per_rank_gathers_the_w_worker_step(method, world, port):
    out = _run(method, world, port)
    assert sorted(out) == list(range(world))
    for rank, r in out.items():
        assert all(r.values()), (rank, r)
