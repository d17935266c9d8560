"""Exchange of compressed payloads between data-parallel ranks, one worker per rank.

The aggregation step of data-parallel training with compressed gradients
(Sparsified SGD with Memory, Method: the workers' sparse updates are summed;
On the Utility of Gradient Compression in Distributed Training Systems, the
evaluation of top-k and signSGD, whose payloads do not add up element by
element and so are gathered instead of all-reduced).  Every rank encodes its
own gradient as the single worker of a one-worker step; the ranks' payload
rows are then gathered in rank order, and every rank decodes the sum (or the
majority vote) of the gathered rows with the same kernels as W replicas on one
GPU.

Rank r's row lands where worker r's row sits in the one-GPU layout
([W, vals_per_worker] floats, and the same for the int32 indices of top-k and
rand-k), so the decode is bit for bit the decode of W replicas whose worker r
holds rank r's gradient and memory: each (worker, layer) encode is independent
of the other workers, and the decode adds the workers in index order.

Only torch.distributed moves bytes here (NCCL between GPUs, gloo on CPU); the
arithmetic of the method runs in the native library.  The ranks must agree on
the table and on k: with Accordion's per-layer levels, every rank passes the
same k tensor.

Payload kinds: top-k, rand-k, signSGD and dense layers.  rand-k's generator
takes the worker index, so rank r encodes as job-wide worker r
(ef_randk_step_at).  With shared keys every rank encodes as worker 0: all
ranks choose the same coordinates, only the values cross (half the bytes),
and the sum is the W-replica decode of rows that share one index row -- the
all-reduce-compatible form of rand-k.

GroupedDataParallelStep cuts the table into groups of consecutive layers and
starts each group's gather as soon as the group is encoded, so the exchange
of one group overlaps the encoding of the next (NCCL runs the collective on
its own stream after the work already queued on the caller's).

PowerSGD's data-parallel form sums P and Q over the workers between its
contractions (On the Utility of Gradient Compression, Key results: PowerSGD is
all-reduce compatible).  PowerSgdDataParallelStep runs it between ranks cut at
those two sums: each rank gathers the other ranks' rows (partial products of
M_w Q, then Q_w) and sums them in worker order itself, so every rank holds the
same P and Q and the step is bit for bit powersgd_dp_step over all workers.
AccordionAcrossRanks all-reduces the per-layer sums of squares, so every rank
takes Accordion's decision from the norm of all ranks' gradients.
"""
import torch
import torch.distributed as dist

METHODS = ("topk", "randk", "sign")


def gather_rows(out, row, group=None, async_op=False):
    """Row r of ``out`` [world, n] <- rank r's ``row`` (n elements of out's
    dtype and device), on every rank; every rank must call it, in the same
    order.  NCCL gathers into the buffer; gloo into a list of its row views.
    async_op: return the collective's work handle (wait() before reading out)
    instead of out."""
    if row is None or row.numel() != out.shape[1] or row.dtype != out.dtype \
            or row.device != out.device:
        raise ValueError("row must be %d %s elements on %s" % (out.shape[1], out.dtype,
                                                                out.device))
    row = row.reshape(-1)
    if not row.is_contiguous():
        raise ValueError("row must be contiguous")
    if dist.get_backend(group) == "nccl":
        work = dist.all_gather_into_tensor(out, row, group=group, async_op=async_op)
    else:
        work = dist.all_gather(list(out.unbind(0)), row, group=group, async_op=async_op)
    return work if async_op else out


class PayloadExchange:
    """Gathered payload rows of every rank: ``vals`` [world, vals_per_worker]
    float32 and, with ``with_idx``, ``idx`` of the same shape int32.

    ``gather`` takes this rank's row(s) and fills row r of each buffer with
    rank r's row; every rank must call it, in the same order.
    """

    def __init__(self, vals_per_worker, with_idx, device, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.n = max(1, int(vals_per_worker))
        self.vals = torch.zeros((self.world, self.n), dtype=torch.float32, device=device)
        self.idx = (torch.zeros((self.world, self.n), dtype=torch.int32, device=device)
                    if with_idx else None)

    def gather(self, vals_row, idx_row=None, async_op=False, values_only=False):
        """All ranks' rows, in rank order: (vals, idx); idx is None without
        indices.  values_only: idx_row is the same on every rank and is copied
        into every row locally instead of gathered.  async_op: start the
        collectives and return their work handles (wait() each before reading
        vals / idx)."""
        works = [gather_rows(self.vals, vals_row, self.group, async_op)]
        if self.idx is not None:
            if values_only:
                self.idx.copy_(idx_row.reshape(1, -1).expand_as(self.idx))
            else:
                works.append(gather_rows(self.idx, idx_row, self.group, async_op))
        return works if async_op else (self.vals, self.idx)


class DataParallelStep:
    """One data-parallel step over the ranks of ``group``, one worker per rank.

    ``encode`` runs this rank's one-worker step (ef_topk_step, ef_randk_step_at
    as worker ``rank`` -- worker 0 with ``shared_keys`` -- or ef_sign_step;
    W = 1) on grad / mem [1, N];
    ``exchange`` gathers every rank's payload (the values alone with
    ``shared_keys``: every rank chose the same indices);
    ``decode`` writes the aggregate of the gathered payloads.  ``__call__``
    runs the three in order.  The native calls run on the current CUDA stream,
    and torch.distributed orders its collectives after that stream's work.
    """

    def __init__(self, table, method, group=None, device="cuda", shared_keys=False):
        import gradient_compression_error_b200 as g
        if method not in METHODS:
            raise ValueError("method must be one of %s (PowerSGD: PowerSgdDataParallelStep)"
                             % (METHODS,))
        ck = table.compressed_kind
        if ck not in (-1, g.KIND[method]):
            raise ValueError("table of kind %s cannot take a %s step"
                             % (g.KIND_NAME.get(ck), method))
        if shared_keys and method != "randk":
            raise ValueError("shared keys are a rand-k mode")
        self.g = g
        self.table = table
        self.method = method
        self.shared_keys = bool(shared_keys)
        sparse = method in ("topk", "randk")
        self.ex = PayloadExchange(table.vals_per_worker, sparse, device, group)
        self.world = self.ex.world
        n = self.ex.n
        self.vals_row = torch.zeros((1, n), dtype=torch.float32, device=device)
        self.idx_row = (torch.zeros((1, n), dtype=torch.int32, device=device)
                        if sparse else None)
        self.ws_step = table.workspace(1, method, device)
        self.ws_dec = table.workspace(self.world, "decompress", device)

    def encode(self, grad, mem, eta, k=None, seed=0, step=0):
        """seed, step: rand-k's generator (the same on every rank)."""
        g = self.g
        if self.method == "topk":
            g.ef_topk_step(self.table, 1, grad, mem, eta, k, self.vals_row, self.idx_row,
                           self.ws_step)
        elif self.method == "randk":
            worker = 0 if self.shared_keys else self.ex.rank
            g.ef_randk_step_at(self.table, worker, 1, grad, mem, eta, k, seed, step,
                               self.vals_row, self.idx_row, self.ws_step)
        else:
            g.ef_sign_step(self.table, 1, grad, mem, eta, self.vals_row, self.ws_step)

    def exchange(self, async_op=False):
        return self.ex.gather(self.vals_row, self.idx_row, async_op=async_op,
                              values_only=self.shared_keys)

    def decode(self, out, scale, k=None, apply=False, vote=False):
        """out = scale * (rank-order sum of the payloads); with ``apply``,
        out -= that instead (the parameter update); with ``vote`` (signSGD),
        out = scale * the elementwise majority sign."""
        g = self.g
        vals, idx = self.ex.vals, self.ex.idx
        if vote:
            if self.method != "sign":
                raise ValueError("the majority vote needs sign payloads")
            g.decompress_vote(self.table, self.world, vals, scale, out)
        elif apply:
            g.decompress_apply(self.table, self.world, vals, idx, k, None, None, scale, out,
                               self.ws_dec)
        else:
            g.decompress_accumulate(self.table, self.world, vals, idx, k, None, None, scale, out,
                                    self.ws_dec)

    def __call__(self, grad, mem, eta, out, scale=None, k=None, apply=False, vote=False,
                 seed=0, step=0):
        """One step; scale defaults to 1/world (the mean)."""
        self.encode(grad, mem, eta, k, seed, step)
        self.exchange()
        self.decode(out, 1.0 / self.world if scale is None else scale, k, apply, vote)
        return out


class GroupedDataParallelStep:
    """DataParallelStep over groups of consecutive layers, with each group's
    exchange started as soon as the group is encoded: the gather of group g
    runs while group g + 1 encodes, and every group is decoded once all
    gathers have landed.  Results are those of the ungrouped step bit for bit
    (each (worker, layer) unit is encoded alone and decoded in worker order).

    ``layers``: the layer descriptors of the whole table (as for Table);
    ``cuts``: the indices of the layers that start a new group (ascending,
    each group starting at a multiple of 4 elements, the 16-byte alignment
    the kernels need).  top-k and signSGD (rand-k's keys depend on a layer's
    index within its table).
    """

    def __init__(self, layers, method, cuts, group=None, device="cuda"):
        import gradient_compression_error_b200 as g
        if method not in ("topk", "sign"):
            raise ValueError("grouped exchange: top-k or signSGD")
        bounds = [0] + [int(c) for c in cuts] + [len(layers)]
        if any(b1 <= b0 for b0, b1 in zip(bounds, bounds[1:])):
            raise ValueError("cuts must be ascending layer indices inside the table")
        self.g = g
        self.parts = []
        off = 0
        for b0, b1 in zip(bounds, bounds[1:]):
            if off % 4:
                raise ValueError("group at layer %d starts at element %d, not a multiple of 4"
                                 % (b0, off))
            t = g.Table(layers[b0:b1])
            self.parts.append(dict(lo=b0, hi=b1, off=off, n=t.N,
                                   step=DataParallelStep(t, method, group, device)))
            off += t.N
        self.N = off
        self.world = self.parts[0]["step"].world

    def __call__(self, grad, mem, eta, out, scale=None, k=None, apply=False, vote=False):
        """One step on this rank's grad / mem [1, N]; out [N] as in
        DataParallelStep; k: per-layer k for the whole table (or None)."""
        if grad.shape[-1] != self.N or mem.shape[-1] != self.N or out.numel() != self.N:
            raise ValueError("grad, mem and out must hold the table's %d elements" % self.N)
        scale = 1.0 / self.world if scale is None else scale
        works = []
        for p in self.parts:
            sl = slice(p["off"], p["off"] + p["n"])
            kp = None if k is None else k[p["lo"]:p["hi"]]
            p["step"].encode(grad[:, sl], mem[:, sl], eta, kp)
            works.append(p["step"].exchange(async_op=True))
        for p, ws in zip(self.parts, works):
            for w in ws:
                w.wait()
            kp = None if k is None else k[p["lo"]:p["hi"]]
            p["step"].decode(out[p["off"]:p["off"] + p["n"]], scale, kp, apply, vote)
        return out


class PowerSgdDataParallelStep:
    """Data-parallel PowerSGD over the ranks of ``group``, one worker per rank,
    cut at its two sums (include/gce.h, powersgd_dp_encode ... _mean).

    Every rank starts from the same warm start Q (``seed``) and ends each step
    with the same P, Q and DENSE mean; ``decode`` writes P Q^T plus the DENSE
    means (the workers' mean update) into a dense buffer.
    """

    def __init__(self, table, group=None, device="cuda", seed=0):
        import gradient_compression_error_b200 as g
        if table.compressed_kind not in (-1, g.KIND["powersgd"]):
            raise ValueError("PowerSgdDataParallelStep needs a PowerSGD table")
        self.g = g
        self.table = table
        self.group = group
        self.world = dist.get_world_size(group)
        f32, f64 = torch.float32, torch.float64
        npart = max(2, g.powersgd_dp_partials(table))
        nq, nv = max(4, table.Q_per_worker), max(4, table.vals_per_worker)
        self.P = torch.zeros(max(4, table.P_per_worker), dtype=f32, device=device)
        self.Q = torch.zeros(nq, dtype=f32, device=device)
        g.powersgd_init_q(table, 1, seed, self.Q)
        self.ppart_row = torch.zeros((1, npart), dtype=f64, device=device)
        self.ppart_all = torch.zeros((self.world, npart), dtype=f64, device=device)
        self.qw_row = torch.zeros((1, nq), dtype=f32, device=device)
        self.qw_all = torch.zeros((self.world, nq), dtype=f32, device=device)
        self.vals_row = torch.zeros((1, nv), dtype=f32, device=device)
        self.vals_all = torch.zeros((self.world, nv), dtype=f32, device=device)
        self.vals = torch.zeros(nv, dtype=f32, device=device)
        self.ws = table.workspace(1, "powersgd_dp", device)
        self.ws_dec = table.workspace(1, "decompress", device)

    def __call__(self, grad, mem, eta, k=None):
        """One step on this rank's gradient and memory [1, N]; returns (P, Q,
        DENSE means), the same on every rank."""
        g, t = self.g, self.table
        g.powersgd_dp_encode(t, 1, grad, mem, eta, k, self.Q, self.ppart_row, self.vals_row,
                             self.ws)
        gather_rows(self.ppart_all, self.ppart_row, self.group)
        gather_rows(self.vals_all, self.vals_row, self.group)
        g.powersgd_dp_orthogonalize(t, self.world, k, self.ppart_all, self.P, self.ws)
        g.powersgd_dp_project(t, 1, mem, k, self.qw_row, self.ws)
        gather_rows(self.qw_all, self.qw_row, self.group)
        g.powersgd_dp_mean(t, self.world, k, self.qw_all, self.Q, self.vals_all, self.vals)
        return self.P, self.Q, self.vals

    def decode(self, out, k=None, apply=False, scale=1.0):
        """out = P Q^T + DENSE means (scale times that); with ``apply``,
        out -= it instead."""
        fn = self.g.decompress_apply if apply else self.g.decompress_accumulate
        fn(self.table, 1, self.vals, None, k, self.P, self.Q, scale, out, self.ws_dec)


class AccordionAcrossRanks:
    """Accordion's per-layer level switch taken from the gradients of every
    rank of ``group``: on check steps the per-layer sums of squares are
    all-reduced before the decision, so all ranks hold the same levels and
    k / ranks (include/gce.h, accordion_sumsq / accordion_decide)."""

    def __init__(self, table, interval, threshold, lvl_low, lvl_high, group=None,
                 device="cuda"):
        import gradient_compression_error_b200 as g
        self.g = g
        self.table = table
        self.group = group
        self.args = (int(interval), float(threshold), int(lvl_low), int(lvl_high))
        L = table.L
        self.sumsq = torch.zeros(L, dtype=torch.float64, device=device)
        self.prev = torch.empty(L, dtype=torch.float64, device=device)
        self.level = torch.empty(L, dtype=torch.int32, device=device)
        self.cur = torch.zeros(L, dtype=torch.float64, device=device)
        self.k = torch.zeros(L, dtype=torch.int32, device=device)
        self.ws = table.workspace(1, "accordion", device)
        g.accordion_init(table, self.prev, self.level)

    def __call__(self, grad, step):
        """k (or rank) per layer for this step, from this rank's gradient [N]."""
        g = self.g
        interval, threshold, lo, hi = self.args
        if step % interval == 0:
            g.accordion_sumsq(self.table, grad, self.sumsq, self.ws)
            dist.all_reduce(self.sumsq, op=dist.ReduceOp.SUM, group=self.group)
        g.accordion_decide(self.table, self.sumsq, step, interval, threshold, lo, hi, self.prev,
                           self.level, self.cur, self.k)
        return self.k

