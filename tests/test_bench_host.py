"""Host-side logic of bench.py: multi-rank timing aggregation (two gloo ranks
on CPU, as torchrun would launch them) and the CPU reference leg."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    t = bench.max_over_ranks_of(local_ms, world, "cpu")
    v = bench.job_throughput(world, 1000, 10, t)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, t, v))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29511
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in out:
        assert t == 20.0                          # max over ranks
        assert v == pytest.approx(2 * 1000 * 10 / 0.020)


def run_bench(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                       text=True, env=e, timeout=600, cwd=ROOT)
    return r


def test_reference_leg_prints_one_json_line():
    r = run_bench(["--impl", "reference", "--workload", "memsgd_vector_2p20", "--steps", "2",
                   "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "elements/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True


def test_reference_leg_is_silent_on_other_ranks():
    r = run_bench(["--impl", "reference", "--workload", "memsgd_vector_2p20", "--steps", "2",
                   "--warmup", "3"], env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0


def test_payload_bytes_per_worker():
    sys.path.insert(0, ROOT)
    import bench
    from gradient_compression_error_b200 import workloads as wl
    layers = [dict(rows=1000, cols=1, kind="topk", cap=10), dict(rows=7, cols=1, kind="dense")]
    assert bench.payload_bytes_per_worker(layers, "topk") == 80 + 28
    assert bench.payload_bytes_per_worker([dict(rows=33, cols=1, kind="sign")], "sign") == 12
    assert bench.payload_bytes_per_worker([dict(rows=64, cols=576, kind="powersgd", cap=2)],
                                          "powersgd") == 4 * 2 * (64 + 576)
    # BERT-base top-k 1 %: K = 1,094,775 pairs of 8 bytes against 437.9 MB of fp32
    bert = wl.bert_base_topk()
    b = bench.payload_bytes_per_worker(bert, "topk")
    assert b == 8 * 1094775
    assert 49 < 4 * 109482240 / b < 51


def test_workload_names():
    """The bench's workload names: the BERT-base sets, and the sweep points with
    an optional _w<W> worker count (the small W = 8 cases of the decoders)."""
    sys.path.insert(0, ROOT)
    import bench
    d = bench.workload_spec("bert_base_topk1pct_w8")
    assert (d["W"], d["method"], len(d["layers"])) == (8, "topk", 90)
    d = bench.workload_spec("sweep_topk_e24_ppm10000_w8")
    assert (d["W"], d["method"], d["layers"][0]["rows"], d["layers"][0]["cap"]) == \
        (8, "topk", 1 << 24, 167772)
    d = bench.workload_spec("sweep_randk_e30_ppm10000")
    assert (d["W"], d["method"], d["layers"][0]["rows"]) == (1, "randk", 1 << 30)
    d = bench.workload_spec("sweep_sign_e25_w8")
    assert (d["W"], d["method"], d["layers"][0]["kind"], d["layers"][0]["cap"]) == \
        (8, "sign", "sign", 0)
    d = bench.workload_spec("sweep_powersgd_e30_r2_lazy")
    assert (d["W"], d["method"], d["layers"][0]["rows"], d["layers"][0]["cols"]) == \
        (1, "powersgd_lazy", 1 << 15, 1 << 15)
    with pytest.raises(SystemExit):
        bench.workload_spec("no_such_workload")
