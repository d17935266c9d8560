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
(ef_randk_step_at).  Not exchanged here: PowerSGD, whose data-parallel form
sums P and Q over the workers inside the step, between its contractions.
"""
import torch
import torch.distributed as dist

METHODS = ("topk", "randk", "sign")


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
        # NCCL gathers straight into the [world, n] buffer; gloo takes a list
        # of its rows (views, written in place)
        self._into = dist.get_backend(group) == "nccl"

    def _gather(self, out, row):
        if row is None or row.numel() != self.n or row.dtype != out.dtype \
                or row.device != out.device:
            raise ValueError("payload row must be %d %s elements on %s"
                             % (self.n, out.dtype, out.device))
        row = row.reshape(-1)
        if not row.is_contiguous():
            raise ValueError("payload row must be contiguous")
        if self._into:
            dist.all_gather_into_tensor(out, row, group=self.group)
        else:
            dist.all_gather(list(out.unbind(0)), row, group=self.group)

    def gather(self, vals_row, idx_row=None):
        """All ranks' rows, in rank order: (vals, idx); idx is None without indices."""
        self._gather(self.vals, vals_row)
        if self.idx is not None:
            self._gather(self.idx, idx_row)
        return self.vals, self.idx


class DataParallelStep:
    """One data-parallel step over the ranks of ``group``, one worker per rank.

    ``encode`` runs this rank's one-worker step (ef_topk_step, ef_randk_step_at
    as worker ``rank`` or ef_sign_step; W = 1) on grad / mem [1, N];
    ``exchange`` gathers every rank's payload;
    ``decode`` writes the aggregate of the gathered payloads.  ``__call__``
    runs the three in order.  The native calls run on the current CUDA stream,
    and torch.distributed orders its collectives after that stream's work.
    """

    def __init__(self, table, method, group=None, device="cuda"):
        import gradient_compression_error_b200 as g
        if method not in METHODS:
            raise ValueError("method must be one of %s (PowerSGD is not exchanged here)"
                             % (METHODS,))
        ck = table.compressed_kind
        if ck not in (-1, g.KIND[method]):
            raise ValueError("table of kind %s cannot take a %s step"
                             % (g.KIND_NAME.get(ck), method))
        self.g = g
        self.table = table
        self.method = method
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
            g.ef_randk_step_at(self.table, self.ex.rank, 1, grad, mem, eta, k, seed, step,
                               self.vals_row, self.idx_row, self.ws_step)
        else:
            g.ef_sign_step(self.table, 1, grad, mem, eta, self.vals_row, self.ws_step)

    def exchange(self):
        return self.ex.gather(self.vals_row, self.idx_row)

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
