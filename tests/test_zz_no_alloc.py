"""decompress_accumulate_noalloc: the decoder for callers that cannot allocate.

Callers that run inside another allocator, whose device memory is reserved in
full by their framework, or that must not pay cudaMalloc's implicit device
synchronisation cannot hand the library a workspace.  This entry point keeps
its scratch in a fixed array inside the library instead; its output must be
the workspace decoder's, bit for bit (the tolerance the sparse decode tests
use), call after call -- the shared array keeps the previous call's contents.
Collected last on purpose (file name), so a stop-at-first-failure run has
already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

from tests.helpers import gce, need_gpu, torch

pytestmark = pytest.mark.gpu


def random_payload(table, layers, W, seed):
    rng = np.random.default_rng(seed)
    vals = np.zeros((W, table.vals_per_worker), np.float32)
    idx = np.zeros((W, table.vals_per_worker), np.int32)
    for w in range(W):
        for l, lay in enumerate(layers):
            o = table.info[l]["val_offset"]
            n = lay["rows"] * lay["cols"]
            if lay["kind"] == "dense":
                vals[w, o:o + n] = rng.standard_normal(n)
            else:
                k = lay["cap"]
                idx[w, o:o + k] = np.sort(rng.choice(n, k, replace=False))
                vals[w, o:o + k] = rng.standard_normal(k) * 10.0 ** rng.uniform(-3, 3, k)
    return torch.from_numpy(vals).cuda(), torch.from_numpy(idx).cuda()


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def call_noalloc(lib, table, W, vals, idx, scale, out, k=None, P=None, Q=None):
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.decompress_accumulate_noalloc(
        table.handle, W, _p(vals), _p(idx), _p(k), _p(P), _p(Q), C.c_float(scale), _p(out),
        stream)


def test_noalloc_decode_matches_workspace_decode_twice():
    need_gpu()
    g = gce()
    lib = g.lib()
    layers = [dict(rows=50000, cols=7, kind="topk", cap=3500),
              dict(rows=333, cols=1, kind="dense", cap=0),
              dict(rows=4096, cols=1, kind="topk", cap=4096),
              dict(rows=1, cols=1, kind="topk", cap=1),
              dict(rows=300001, cols=1, kind="topk", cap=30000)]
    W = 4
    table = g.Table(layers)
    ws = table.workspace(W, "decompress")
    for call, (seed, scale) in enumerate([(1, 1.0), (2, 0.25)]):
        vals, idx = random_payload(table, layers, W, seed)
        want = torch.full((table.N,), float("nan"), device="cuda")
        got = torch.full((table.N,), float("nan"), device="cuda")
        g.decompress_accumulate(table, W, vals, idx, None, None, None, scale, want, ws)
        assert call_noalloc(lib, table, W, vals, idx, scale, got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), call


def test_noalloc_per_layer_k_shrinks_and_skips_layers():
    """Call 1 decodes with large per-layer k; call 2 with smaller k, one layer
    at k = 0 and one above its cap (both contribute nothing).  Slots the first
    call filled and the second does not use must not leak into its output."""
    need_gpu()
    g = gce()
    lib = g.lib()
    layers = [dict(rows=50000, cols=7, kind="topk", cap=3500),
              dict(rows=333, cols=1, kind="dense", cap=0),
              dict(rows=4096, cols=1, kind="topk", cap=4096),
              dict(rows=1, cols=1, kind="topk", cap=1),
              dict(rows=300001, cols=1, kind="topk", cap=30000),
              dict(rows=9000, cols=3, kind="topk", cap=2000)]
    W = 3
    table = g.Table(layers)
    ws = table.workspace(W, "decompress")
    calls = [([3500, 0, 4096, 1, 30000, 2000], 1.0),
             ([17, 0, 0, 1, 29999, 2001], 0.5)]       # k = 0 and k > cap: layer skipped
    for call, (ks, scale) in enumerate(calls):
        vals, idx = random_payload(table, layers, W, 10 + call)
        k = torch.tensor(ks, dtype=torch.int32, device="cuda")
        want = torch.full((table.N,), float("nan"), device="cuda")
        got = torch.full((table.N,), float("nan"), device="cuda")
        g.decompress_accumulate(table, W, vals, idx, k, None, None, scale, want, ws)
        assert call_noalloc(lib, table, W, vals, idx, scale, got, k=k) == 0
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), call
    # the skipped layers decode to +0 (nothing summed), not to the first call's sums
    for l in (2, 5):
        o, n = table.info[l]["offset"], table.info[l]["n"]
        assert not torch.any(got[o:o + n].view(torch.int32))


def test_noalloc_low_rank_table_twice():
    """A PowerSGD table through the same entry point: P Q^T per layer, summed
    over the workers, equal to the workspace decoder bit for bit."""
    need_gpu()
    g = gce()
    lib = g.lib()
    layers = [dict(rows=64, cols=576, kind="powersgd", cap=4),
              dict(rows=128, cols=1, kind="dense", cap=0),
              dict(rows=513, cols=77, kind="powersgd", cap=2)]
    W = 2
    table = g.Table(layers)
    ws = table.workspace(W, "decompress")
    gen = torch.Generator(device="cuda").manual_seed(5)
    for call, (ks, scale) in enumerate([([4, 0, 2], 1.0), ([3, 0, 1], 0.5)]):
        P = torch.randn((W, table.P_per_worker), device="cuda", generator=gen)
        Q = torch.randn((W, table.Q_per_worker), device="cuda", generator=gen)
        vals = torch.randn((W, table.vals_per_worker), device="cuda", generator=gen)
        k = torch.tensor(ks, dtype=torch.int32, device="cuda")
        want = torch.full((table.N,), float("nan"), device="cuda")
        got = torch.full((table.N,), float("nan"), device="cuda")
        g.decompress_accumulate(table, W, vals, None, k, P, Q, scale, want, ws)
        assert call_noalloc(lib, table, W, vals, None, scale, got, k=k, P=P, Q=Q) == 0
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), call


def test_noalloc_rejects_tables_beyond_its_scratch():
    need_gpu()
    g = gce()
    lib = g.lib()
    layers = [dict(rows=1 << 24, cols=1, kind="topk", cap=10)]    # 16,385 bound slots per worker
    table = g.Table(layers)
    W = 64                                                         # 1,048,640 > 1,048,576
    vals = torch.zeros((1, 16), device="cuda")
    idx = torch.zeros((1, 16), dtype=torch.int32, device="cuda")
    out = torch.zeros(16, device="cuda")
    assert call_noalloc(lib, table, W, vals, idx, 1.0, out) == -3   # GCE_ERR_WORKSPACE
