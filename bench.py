#!/usr/bin/env python
"""Benchmark of the gradient-compression hot path on B200: prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--profile]

Default workload (bert_base_topk1pct_w8): BERT-base-shaped fp32 gradients
(109,482,240 elements per worker, 90 tensors) compressed with error-feedback
top-k at 1 % of every tensor for W = 8 data-parallel worker replicas held in
one GPU's HBM, and the W sparse payloads summed on the device.  One step =
ef_topk_step (encode + memory update) + decompress_accumulate (decode), on
fresh seeded N(0, 1) gradients resident in HBM.  The metric is gradient
elements encoded+decoded per second (W * N per step); the roofline object
reports the dominant kernel (the fused residual / memory / candidate pass)
against the measured HBM copy bandwidth.

Under torchrun (N > 1) every rank runs its own independent replica of the
workload (the workload's W workers are simulated replicas; there is no data
exchange between GPUs): value = elements of all ranks / max time over ranks.
--impl reference times the CPU oracle (plain C, oracle/) on a bounded sample
of the same workload on the host cores.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gradient elements encoded+decoded per sec (GB/s vs HBM roofline); ms per step"
UNIT = "elements/s"
DEFAULT_WORKLOAD = "bert_base_topk1pct_w8"
MAIN_KERNEL = "tk_main_kernel"
MAIN_SOURCE = os.path.join(ROOT, "gradient_compression_error_b200", "csrc", "topk.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "tk_main_bert_base_w8_traffic.txt")
FALLBACK_HBM_GBS = 6650.0


def workload_spec(name):
    from gradient_compression_error_b200 import workloads as wl
    if name == "bert_base_topk1pct_w8":
        return dict(layers=wl.bert_base_topk(), W=8, cfg=4, method="topk")
    if name == "bert_base_topk1pct_w8_apply":    # decode fused with x -= mean update, eta_t
        return dict(layers=wl.bert_base_topk(), W=8, cfg=4, method="topk", apply=True)
    if name == "bert_base_sign_w8":              # signSGD with memory, 1 bit per element
        return dict(layers=wl.bert_base_topk(kind="sign"), W=8, cfg=4, method="sign")
    if name == "bert_base_sign_w1":              # one replica: a profiling-sized case
        return dict(layers=wl.bert_base_topk(kind="sign"), W=1, cfg=4, method="sign")
    if name == "bert_base_topk1pct_w1":          # one replica: a profiling-sized case
        return dict(layers=wl.bert_base_topk(), W=1, cfg=4, method="topk")
    if name == "bert_base_randk1pct_w8":
        return dict(layers=wl.bert_base_topk(kind="randk"), W=8, cfg=4, method="randk")
    if name == "memsgd_vector_2p20":
        return dict(layers=wl.memsgd_vector(), W=1, cfg=1, method="topk")
    if name == "resnet18_powersgd_r2":
        return dict(layers=wl.resnet18_powersgd(2), W=1, cfg=2, method="powersgd")
    if name == "resnet18_powersgd_r2_w8_dp":     # data-parallel: shared P and Q over 8 workers
        return dict(layers=wl.resnet18_powersgd(2), W=8, cfg=2, method="powersgd_dp")
    if name == "vgg19_accordion_powersgd":       # ranks 4 / 2 chosen by Accordion
        return dict(layers=wl.vgg19("powersgd", 4), W=1, cfg=3, method="powersgd",
                    accordion=(4, 2))
    if name == "vgg19_accordion_topk":           # k 10 % / 1 % chosen by Accordion
        return dict(layers=wl.vgg19("topk", 100000), W=1, cfg=3, method="topk",
                    accordion=(100000, 10000))
    # a sweep layer, one worker unless the name ends in _w<W> (e.g. the 2^24
    # layers at W = 8: a small case of the W = 8 decoders)
    base, sep, wsuf = name.rpartition("_w")
    W = int(wsuf) if name.startswith("sweep_") and sep and wsuf.isdigit() else 1
    if W > 1:
        name = base
    if name.startswith("sweep_topk_e"):          # e.g. sweep_topk_e28_ppm10000
        e, ppm = name[len("sweep_topk_e"):].split("_ppm")
        return dict(layers=wl.sweep(int(e), "topk", int(ppm)), W=W, cfg=5, method="topk")
    if name.startswith("sweep_randk_e"):
        e, ppm = name[len("sweep_randk_e"):].split("_ppm")
        return dict(layers=wl.sweep(int(e), "randk", int(ppm)), W=W, cfg=5, method="randk")
    if name.startswith("sweep_sign_e"):          # e.g. sweep_sign_e24
        e = name[len("sweep_sign_e"):]
        return dict(layers=wl.sweep(int(e), "sign"), W=W, cfg=5, method="sign")
    if name.startswith("sweep_powersgd_e"):      # e.g. sweep_powersgd_e28_r2[_lazy]
        lazy = name.endswith("_lazy")
        e, r = name[len("sweep_powersgd_e"):].replace("_lazy", "").split("_r")
        return dict(layers=wl.sweep(int(e), "powersgd", rank=int(r)), W=1, cfg=5,
                    method="powersgd_lazy" if lazy else "powersgd")
    raise SystemExit("unknown workload %s" % name)


MAIN_KERNELS = {"topk": "tk_main_kernel", "randk": "rk_emit_kernel", "powersgd": "ps_mq_kernel",
                "powersgd_lazy": "ps_mq_kernel",
                "powersgd_dp": "ps_mq_kernel", "sign": "sg_fused_kernel"}


def max_over_ranks_of(x, world, device):
    """The largest of the ranks' values (each rank times its own device)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def payload_bytes_per_worker(layers, method):
    """Bytes one worker sends per step (what its exchange would carry): sparse
    (value, index) pairs, a sign layer's words and scale, PowerSGD's P and Q,
    a dense layer's floats.  For the data-parallel PowerSGD step, a worker's
    share of the two all-reduces."""
    total = 0
    for l in layers:
        n = l["rows"] * l["cols"]
        if l["kind"] == "dense":
            total += 4 * n
        elif l["kind"] in ("topk", "randk"):
            total += 8 * l["cap"]
        elif l["kind"] == "sign":
            total += 4 * ((n + 31) // 32) + 4
        else:
            total += 4 * l["cap"] * (l["rows"] + l["cols"])
    return total


def job_throughput(world, elems_per_step, steps, t_ms_max):
    """Whole-job elements per second: every rank's elements over the slowest
    rank's time (each rank runs its own replica of the workload)."""
    return world * elems_per_step * steps / (t_ms_max / 1e3)


def measured_hbm_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def main_kernel_source_hash():
    """sha256 of the main kernel's source text (its definition in topk.cu),
    which is what the committed traffic capture was taken of."""
    src = open(MAIN_SOURCE).read()
    head = "tk_main_kernel("
    a = src.index("__global__ void __launch_bounds__(kTkThreads) " + head)
    b = src.index("\n}\n", a) + 3
    return hashlib.sha256(src[a:b].encode()).hexdigest()


def ncu_traffic_per_launch():
    """Per-launch DRAM bytes of the main kernel from the committed ncu summary,
    or None when the kernel's source changed since the capture."""
    try:
        src_hash = main_kernel_source_hash()
        fields = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("source_sha256") != src_hash:
            return None
        return float(fields["dram_bytes_per_launch_full_size"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def cpu_oracle_sample(spec, units, steps_seed, threads=None):
    """Run the oracle on `units` of the workload (host arrays from seeded
    gradients of worker w) on `threads` host threads (default: all cores);
    returns (elements, seconds, threads)."""
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from gradient_compression_error_b200 import workloads as wl
    import torch
    layers = spec["layers"]
    offs, o = [], 0
    for l in layers:
        offs.append(o)
        o += l["rows"] * l["cols"]
    threads = threads or os.cpu_count() or 1
    dp = spec["method"] == "powersgd_dp"   # a unit is one layer of every worker
    data = {}
    for (w, l) in units:
        n = layers[l]["rows"] * layers[l]["cols"]
        gs = []
        for ww in (range(spec["W"]) if dp else [w]):
            g = torch.Generator()
            g.manual_seed(wl.seed_for(spec["cfg"], ww, steps_seed) + l)
            gs.append(torch.randn(n, generator=g).numpy().astype(np.float32))
        data[(w, l)] = (np.stack(gs) if dp else gs[0],
                        np.zeros((len(gs), n) if dp else n, np.float32))

    def one(u):
        w, l = u
        lay = layers[l]
        gg, mm = data[u]
        out = np.zeros(gg.shape[-1], np.float32)
        if dp:
            if lay["kind"] == "dense":
                pay, m_new = oracle.dense_dp_unit(gg, mm, wl.ETA)
                oracle.accum_dense(out, pay)
            else:
                rows, cols = lay["rows"], lay["cols"]
                Q = oracle.powersgd_init_q(cols, lay["cap"], 1, 0, l)
                P, Qn, m_new = oracle.powersgd_dp_unit(gg.reshape(-1, rows, cols),
                                                       mm.reshape(-1, rows, cols), Q, lay["cap"],
                                                       wl.ETA)
                oracle.accum_lowrank(out, P, Qn, lay["cap"])
        elif lay["kind"] == "dense":
            pay, m_new = oracle.dense_unit(gg, mm, wl.ETA)
            oracle.accum_dense(out, pay)
        elif spec["method"] in ("powersgd", "powersgd_lazy"):
            rows, cols = lay["rows"], lay["cols"]
            Q = oracle.powersgd_init_q(cols, lay["cap"], 1, w, l)
            P, Qn, m_new, _ = oracle.powersgd_unit(gg.reshape(rows, cols), mm.reshape(rows, cols),
                                                   Q, lay["cap"], wl.ETA, want_mhat=False)
            oracle.accum_lowrank(out, P, Qn, lay["cap"])
        elif spec["method"] == "topk":
            vals, idx, m_new = oracle.ef_topk_unit(gg, mm, lay["cap"], wl.ETA)
            oracle.accum_sparse(out, vals, idx)
        elif spec["method"] == "sign":
            sc, words, m_new = oracle.ef_sign_unit(gg, mm, wl.ETA)
            oracle.accum_sign(out, sc, words)
        else:
            vals, idx, m_new = oracle.ef_randk_unit(gg, mm, lay["cap"], wl.ETA, 5, w, l, 0)
            oracle.accum_sparse(out, vals, idx)
        return gg.size

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        elems = sum(ex.map(one, units))
    dt = time.perf_counter() - t0
    return elems, dt, threads


# One step of every workload of the method's configurations, for the oracle
# timing table: the 2^20 vector, ResNet-18 PowerSGD, VGG-19 with Accordion's
# two levels (PowerSGD and top-k), one BERT-base worker, and the sweep (one
# step at 2^27, the largest point the oracle finishes in about a minute).
ORACLE_TABLE = ["memsgd_vector_2p20", "resnet18_powersgd_r2", "vgg19_accordion_powersgd",
                "vgg19_accordion_topk", "bert_base_topk1pct_w8", "sweep_topk_e27_ppm10000",
                "sweep_powersgd_e27_r2"]


def oracle_timing(threads_all):
    """{workload: (elements, s at 1 thread, s on all cores)} for one step of
    worker 0 of each workload in ORACLE_TABLE (encode + decode)."""
    rows = []
    for name in ORACLE_TABLE:
        spec = workload_spec(name)
        units = [(0, l) for l in range(len(spec["layers"]))]
        e1, t1, _ = cpu_oracle_sample(spec, units, 0, threads=1)
        en, tn, n = cpu_oracle_sample(spec, units, 0, threads=threads_all)
        rows.append({"workload": name, "elements": e1, "s_1thread": t1, "s_all": tn,
                     "threads": n})
    return rows


def run_reference(args, rank, world):
    if rank != 0:
        return
    spec = workload_spec(args.workload)
    L = len(spec["layers"])
    # bounded sample per step: one worker's tensors, rotating over workers,
    # capped near 6 M elements so a 13-step run stays within a few minutes
    samples = []
    for s in range(args.warmup + args.steps):
        w = s % spec["W"]
        units, tot = [], 0
        per_unit = spec["W"] if spec["method"] == "powersgd_dp" else 1
        for l in sorted(range(L), key=lambda l: -(spec["layers"][l]["rows"] * spec["layers"][l]["cols"])):
            n = spec["layers"][l]["rows"] * spec["layers"][l]["cols"] * per_unit
            if tot + n <= 6_000_000 or not units:
                units.append((w, l))
                tot += n
        samples.append(units)
    times, elems_tot, threads = [], 0, 1
    for s, units in enumerate(samples):
        elems, dt, threads = cpu_oracle_sample(spec, units, s)
        if s >= args.warmup:
            times.append(dt)
            elems_tot += elems
    t = sum(times)
    value = elems_tot / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded N(0,1) gradients)",
            "config": {"workload": args.workload, "W": spec["W"]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": "per step: the largest tensors of one worker (rotating; "
                                       "for the data-parallel PowerSGD workload, of every "
                                       "worker), about 6 M elements, %s encode + decode"
                                       % spec["method"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SECONDARY = ["sweep_powersgd_e30_r2", "sweep_powersgd_e30_r2_lazy", "bert_base_randk1pct_w8",
             "bert_base_sign_w8", "resnet18_powersgd_r2"]


def run_workload(name, args, world, rank, dev, primary):
    """Time `name` (args.steps steps after args.warmup warm-up steps) and
    return its measurement fields.  Inputs that fit twice in L2 are timed
    cold (L2 flushed between steps, each step between its own events) and
    hot (one event pair around the steps); larger ones with one event pair
    around the steps, the inputs themselves evicting L2."""
    import torch
    import torch.distributed as dist
    import gradient_compression_error_b200 as gce
    from gradient_compression_error_b200 import workloads as wl

    spec = workload_spec(name)
    layers, W = spec["layers"], spec["W"]
    table = gce.Table(wl.table_layers(layers))
    N = table.N
    K_total = sum(l["cap"] for l in layers)
    grads = [wl.gradients(layers, W, spec["cfg"], s) for s in range(2)]
    mem = torch.zeros((W, N), dtype=torch.float32, device=dev)
    vals = torch.zeros((W, table.vals_per_worker), dtype=torch.float32, device=dev)
    idx = torch.zeros((W, table.vals_per_worker), dtype=torch.int32, device=dev)
    ws = table.workspace(W, "powersgd" if spec["method"] == "powersgd_lazy" else spec["method"])
    ws_dc = table.workspace(W, "decompress")
    out = torch.zeros(N, dtype=torch.float32, device=dev)
    method = spec["method"]
    P = Q = lazy_rank = None
    if method == "powersgd_lazy":
        lazy_rank = torch.zeros((W, table.L), dtype=torch.int32, device=dev)
    if method in ("powersgd", "powersgd_lazy"):
        P = torch.zeros((W, max(4, table.P_per_worker)), dtype=torch.float32, device=dev)
        Q = torch.zeros((W, max(4, table.Q_per_worker)), dtype=torch.float32, device=dev)
        gce.powersgd_init_q(table, W, 1, Q)
    if method == "powersgd_dp":      # one shared P, Q and dense payload for all workers
        P = torch.zeros(max(4, table.P_per_worker), dtype=torch.float32, device=dev)
        Q = torch.zeros(max(4, table.Q_per_worker), dtype=torch.float32, device=dev)
        vals = torch.zeros(max(4, table.vals_per_worker), dtype=torch.float32, device=dev)
        gce.powersgd_init_q(table, 1, 1, Q)
    kr = None
    if "accordion" in spec:   # Accordion picks each layer's k or rank every step
        L = len(layers)
        prev = torch.empty(L, dtype=torch.float64, device=dev)
        level = torch.empty(L, dtype=torch.int32, device=dev)
        cur = torch.zeros(L, dtype=torch.float64, device=dev)
        kr = torch.zeros(L, dtype=torch.int32, device=dev)
        ws_ac = table.workspace(1, "accordion")
        gce.accordion_init(table, prev, level)
        lvl_low, lvl_high = spec["accordion"]

    apply = bool(spec.get("apply"))
    if apply:    # the parameters the mean update is applied to, in place
        out.normal_(generator=torch.Generator(device=dev).manual_seed(77))

    def step(s, grad):
        # the Mem-SGD step size eta_t = 8 / (mu (a + t)) with mu = 1, a = 160
        # (eta_0 = 0.05) when the update is applied; the fixed eta otherwise
        eta = gce.memsgd_eta(s, 1.0, 160.0) if apply else wl.ETA
        if kr is not None:
            gce.accordion_select(table, grad[0], s, 10, 0.5, lvl_low, lvl_high, prev, level, cur,
                                 kr, ws_ac)
        if method == "topk":
            gce.ef_topk_step(table, W, grad, mem, eta, kr, vals, idx, ws)
        elif method == "randk":
            gce.ef_randk_step(table, W, grad, mem, eta, kr, 5, s, vals, idx, ws)
        elif method == "sign":
            gce.ef_sign_step(table, W, grad, mem, eta, vals, ws)
        elif method == "powersgd_dp":
            gce.powersgd_dp_step(table, W, grad, mem, eta, kr, P, Q, vals, ws)
            # the shared payload is already the workers' mean: one decode
            gce.decompress_accumulate(table, 1, vals, None, kr, P, Q, 1.0, out, ws_dc)
            return
        elif method == "powersgd_lazy":
            gce.powersgd_step_lazy(table, W, grad, mem, eta, kr, P, Q, vals, lazy_rank, ws)
        else:
            gce.powersgd_step(table, W, grad, mem, eta, kr, P, Q, vals, None, ws)
        sparse = method in ("topk", "randk")
        if apply:
            gce.decompress_apply(table, W, vals, idx if sparse else None, kr, P, Q, 1.0 / W, out,
                                 ws_dc)
        else:
            gce.decompress_accumulate(table, W, vals, idx if sparse else None, kr, P, Q, 1.0,
                                      out, ws_dc)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return max_over_ranks_of(x, world, dev)

    for s in range(args.warmup):
        step(s, grads[s % 2])
    torch.cuda.synchronize()
    if gce.status(ws) & gce.STATUS_K_RANGE:
        raise SystemExit("device status reports an out-of-range k")

    # CUDA-graph replay: one graph per gradient buffer, captured after the
    # warm-up; the kernels and their arguments are those of the eager step
    graphs, launches_per_step = None, None
    graphable = not (method == "randk" or kr is not None or apply)
    if args.graph and primary and not graphable:
        raise SystemExit("--graph: this workload's step takes per-step host values")
    if args.graph and primary:
        graphs = []
        for b in range(2):
            gr = torch.cuda.CUDAGraph()
            l_before = gce.launch_count()
            with torch.cuda.graph(gr):
                step(0, grads[b])
            launches_per_step = gce.launch_count() - l_before
            graphs.append(gr)
        for s in range(3):
            graphs[s % 2].replay()
        torch.cuda.synchronize()

    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    input_bytes = 8 * W * N      # gradient and memory a step reads
    cold = input_bytes < 2 * l2_bytes
    flush = torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev) if cold else None

    def run_steps(k0, count, flushed):
        """count steps; returns their device time in ms (flushed: each step
        between its own events, L2 rewritten between steps)."""
        if not flushed:
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record()
            for s in range(count):
                if graphs:
                    graphs[s % 2].replay()
                else:
                    step(k0 + s, grads[s % 2])
            ev1.record()
            torch.cuda.synchronize()
            return ev0.elapsed_time(ev1)
        evs = []
        for s in range(count):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            if graphs:
                graphs[s % 2].replay()
            else:
                step(k0 + s, grads[s % 2])
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.2)
    l0 = gce.launch_count()
    main_kernel = MAIN_KERNELS[method]
    # events around the main pass only (every kernel with --profile)
    gce.profile_only(None if args.profile else main_kernel)
    gce.profile_start()
    t_local = run_steps(args.warmup, args.steps, cold)
    prof = gce.profile_stop()
    launches = gce.launch_count() - l0
    hot_ms = None
    if cold:   # the same steps with L2 left warm between them
        hot_ms = run_steps(args.warmup + args.steps, args.steps, False) / args.steps
    if graphs:
        # replays launch nothing from the host: the captured kernels per step;
        # the main-pass time comes from a short eager pass right after
        launches = launches_per_step * args.steps
        gce.profile_start()
        for s in range(min(args.steps, 20)):
            step(args.warmup + s, grads[s % 2])
        torch.cuda.synchronize()
        prof = gce.profile_stop()
        prof = {k: (v[0] * args.steps / min(args.steps, 20), v[1] * args.steps // min(args.steps, 20))
                for k, v in prof.items()}
    barrier()
    clk = clocks.stop()
    t_ms = max_over_ranks(t_local)
    fallback_seen = bool(gce.status(ws) & gce.STATUS_FALLBACK)

    elems_per_step = W * N
    value = job_throughput(world, elems_per_step, args.steps, t_ms)
    ms_step = t_ms / args.steps

    # the main pass, whichever template instance ran (rand-k's may carry the
    # next step's key pass)
    hits = [v for n, v in prof.items() if n == main_kernel or n.startswith(main_kernel + "<")]
    main_ms, main_n = sum(v[0] for v in hits), sum(v[1] for v in hits)
    peak, peak_kind = measured_hbm_gbs()
    # the main pass covers every compressed element once per step: bytes and
    # kernel time per step
    bytes_per_step_main = 12.0 * W * (N - sum(l["rows"] * l["cols"] for l in layers
                                             if l["kind"] == "dense"))
    main_ms_per_step = main_ms / args.steps
    achieved = (bytes_per_step_main / (main_ms_per_step / 1e3) / 1e9) if main_n else None
    traffic = ncu_traffic_per_launch() if name == DEFAULT_WORKLOAD else None
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                "kernel": main_kernel,
                "peak_source": peak_kind,
                "algorithmic_bytes_per_step": bytes_per_step_main,
                "launches_per_step": main_n / args.steps,
                "kernel_ms_per_step": main_ms_per_step if main_n else None}
    # whole-step algorithmic traffic: sparse W(12N + 8K) encode + 16 W K + 4N
    # decode; PowerSGD W * 12N encode + 4N decode (P and Q are negligible)
    if method in ("powersgd", "powersgd_dp", "powersgd_lazy"):
        step_bytes = W * 12.0 * N
    elif method == "sign":
        # grad and memory read once, memory written, words written (the
        # pipelined kernel's second visit reads L2); decode reads the words
        step_bytes = W * (12.0 * N + N / 8.0) + W * N / 8.0
    else:
        step_bytes = W * (12.0 * N + 8.0 * K_total) + 16.0 * W * K_total
    # the dense result: written (4 B), or read and written in place (8 B)
    step_bytes += (8.0 if apply else 4.0) * N
    step_gbs = step_bytes / (ms_step / 1e3) / 1e9

    # end to end through the public API with host buffers
    e2e = None
    if primary and not args.no_e2e:
        hgrad = torch.empty((W, N), dtype=torch.float32, pin_memory=True)
        hgrad.copy_(grads[0])
        hout = torch.empty(N, dtype=torch.float32, pin_memory=True)
        dgrad = grads[1]
        ke = max(3, min(args.steps, 20))
        step(0, dgrad)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(ke):
            dgrad.copy_(hgrad, non_blocking=True)
            step(s, dgrad)
            hout.copy_(out, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1))
        e2e = {"value": world * elems_per_step * ke / (te / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": W * N * 4, "d2h_bytes_per_step": N * 4, "steps": ke}
        del hgrad, hout

    if args.profile and rank == 0:
        tot = sum(v[0] for v in prof.values())
        for kname, (ms, n) in sorted(prof.items(), key=lambda x: -x[1][0]):
            print("%-32s %8d launches %10.3f ms %6.1f%%" % (kname, n, ms, 100 * ms / tot),
                  file=sys.stderr)

    l2_note = ("L2 flushed before every step (a %d MB write outside the step's events); "
               "hot (L2 warm) %.4f ms per step" % (2 * l2_bytes >> 20, hot_ms) if cold else
               "inputs larger than L2 (%.1f GB of grad+memory per step)" % (input_bytes / 1e9))
    return dict(spec=spec, layers=layers, W=W, N=N, K_total=K_total, apply=apply, value=value,
                ms_step=ms_step, hot_ms=hot_ms, cold=cold, roofline=roofline, step_gbs=step_gbs,
                peak=peak, launches=launches, clocks=clk, e2e=e2e, graphs=bool(graphs),
                fallback_seen=fallback_seen, l2_note=l2_note, method=method)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--profile", action="store_true", help="per-kernel table on stderr")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' short measurements")
    ap.add_argument("--oracle-timing", action="store_true",
                    help="time the CPU oracle on one step of every workload at 1 thread and "
                         "on all cores, print one JSON line, and exit")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step as a CUDA graph (workloads whose step takes no "
                         "per-step host values: top-k, sign, PowerSGD without Accordion)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.oracle_timing:
        if rank == 0:
            print(json.dumps({"oracle_timing": oracle_timing(os.cpu_count() or 1),
                              "cpu_model": cpu_model(), "cores": os.cpu_count()}), flush=True)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = "cuda"

    r = run_workload(args.workload, args, world, rank, dev, primary=True)
    spec, layers, W, N, method = r["spec"], r["layers"], r["W"], r["N"], r["method"]
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        units = [(0, l) for l in range(len(layers))]
        elems, dt, threads = cpu_oracle_sample(spec, units, 0)
        # the same sample on one thread, bounded to the largest tensors that
        # fit about 6 M elements (at one thread the full set takes minutes)
        sub, tot = [], 0
        for l in sorted(range(len(layers)), key=lambda l: -(layers[l]["rows"] * layers[l]["cols"])):
            n = layers[l]["rows"] * layers[l]["cols"]
            if tot + n <= 6_000_000 or not sub:
                sub.append((0, l))
                tot += n
        e1, t1, _ = cpu_oracle_sample(spec, sub, 0, threads=1)
        cpu = {"value": elems / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "worker 0: all %d tensors (%d elements), encode + decode, one step"
                         % (len(layers), elems), "seconds": dt,
               "value_1thread": e1 / t1,
               "sample_1thread": "worker 0: its largest tensors up to about 6 M elements "
                                 "(%d elements), encode + decode, one step, one thread" % e1,
               "cpu_model": cpu_model()}

    secondary = None
    if world == 1 and not args.no_secondary and args.workload == DEFAULT_WORKLOAD:
        import copy
        sargs = copy.copy(args)
        sargs.steps, sargs.warmup, sargs.graph, sargs.profile = min(args.steps, 30), 3, False, False
        secondary = []
        for name in SECONDARY:
            x = run_workload(name, sargs, world, rank, dev, primary=False)
            secondary.append({"workload": name, "value": x["value"], "unit": UNIT,
                              "ms_per_step": x["ms_step"], "steps": sargs.steps,
                              "warmup": sargs.warmup,
                              "timing": "cold (L2 flushed before every step)" if x["cold"]
                                        else "inputs larger than L2",
                              "ms_per_step_hot": x["hot_ms"],
                              "step_algorithmic_GBps": x["step_gbs"],
                              "step_frac_of_hbm": x["step_gbs"] / x["peak"],
                              "roofline": {k: x["roofline"][k] for k in
                                           ("kernel", "achieved", "frac", "kernel_ms_per_step")},
                              "gpu_launches": x["launches"], "clocks": x["clocks"]})
            del x
            torch.cuda.empty_cache()

    if rank == 0:
        K_total = r["K_total"]
        line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded N(0,1) gradients, resident in HBM)",
                "config": {"workload": args.workload, "W": W, "elements_per_worker": N,
                           "tensors": len(layers), "k_total_per_worker": K_total,
                           "eta": "8/(1*(160+t))" if r["apply"] else 0.05,
                           "update": "x -= mean of payloads (fused)" if r["apply"] else "decode only",
                           "parallelism": "replicas x%d" % world,
                           "launch": ("CUDA graph replay (main-pass time from 20 eager steps)"
                                      if r["graphs"] else "eager"),
                           "l2": r["l2_note"],
                           "payload_bytes_per_worker": payload_bytes_per_worker(layers, method),
                           "compression_ratio": 4.0 * N / payload_bytes_per_worker(layers, method),
                           "step_algorithmic_GBps": r["step_gbs"],
                           "step_frac_of_hbm": r["step_gbs"] / r["peak"],
                           "fallback_seen": r["fallback_seen"]},
                "roofline": r["roofline"], "cpu_baseline": cpu, "e2e": r["e2e"],
                "gpu_launches": r["launches"], "clocks": r["clocks"]}
        if secondary is not None:
            line["secondary"] = secondary
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
