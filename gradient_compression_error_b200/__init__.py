"""Python binding of the gce C ABI (include/gce.h): argument marshalling only.

Every step of the gradient-compression path runs in the native library
libgce.so (CUDA C++ for sm_100a) built in-tree by
``python -m gradient_compression_error_b200.build``.  This module converts
torch CUDA tensors into device pointers and the current CUDA stream into a
``cudaStream_t``; it computes nothing itself.  If the library is missing the
first call raises -- there is no fallback.

The entry points keep the C names: ef_topk_step, ef_randk_step,
ef_randk_step_at, ef_sign_step, powersgd_init_q, powersgd_step,
powersgd_step_lazy (with materialize_memory), powersgd_dp_step and its four parts
for ranks (powersgd_dp_encode / _orthogonalize / _project / _mean), accordion_init, accordion_select, decompress_accumulate,
decompress_apply, decompress_accumulate_noalloc, decompress_vote, plus the
Table wrapper of gce_table_* and the workspace, status, schedule and profiling
helpers.  The exchange of payloads between data-parallel ranks sits on top of
these, in the ``exchange`` module.
"""
import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgce.so")

KIND = {"topk": 0, "randk": 1, "powersgd": 2, "dense": 3, "sign": 4}
KIND_NAME = {v: k for k, v in KIND.items()}
OP = {"topk": 0, "randk": 1, "powersgd": 2, "accordion": 3, "decompress": 4, "powersgd_dp": 5,
      "sign": 6}
OPT = {"bracket_sigma": 0, "randk_ahead": 1, "sign_ahead": 2, "sign_emit_first": 3}
STATUS_K_RANGE = 1
STATUS_FALLBACK = 2
STATUS_NONFINITE = 4
STATUS_WAIT_TIMEOUT = 8
LEVEL_LOW, LEVEL_HIGH = 0, 1
WS_HEADER_BYTES = 256

ERRORS = {-1: "invalid argument", -2: "CUDA runtime error", -3: "workspace missing or too small",
          -4: "device allocation failed", -5: "layer kinds do not fit this call"}


class GceError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s returned %d (%s)" % (fn, code, ERRORS.get(code, "unknown")))
        self.code = code


class LayerDesc(C.Structure):
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64), ("kind", C.c_int32), ("cap", C.c_int32)]


class LayerInfo(C.Structure):
    _fields_ = [("offset", C.c_int64), ("n", C.c_int64), ("rows", C.c_int64), ("cols", C.c_int64),
                ("kind", C.c_int32), ("cap", C.c_int32), ("val_offset", C.c_int64),
                ("p_offset", C.c_int64), ("q_offset", C.c_int64)]


class Totals(C.Structure):
    _fields_ = [("L", C.c_int64), ("N", C.c_int64), ("vals_per_worker", C.c_int64),
                ("P_per_worker", C.c_int64), ("Q_per_worker", C.c_int64),
                ("compressed_kind", C.c_int32)]


# exported symbol -> (restype, argtypes); the full list the header declares
_vp, _i32, _i64, _u64, _f32, _f64 = (C.c_void_p, C.c_int32, C.c_int64, C.c_uint64, C.c_float,
                                     C.c_double)
SIGNATURES = {
    "gce_table_create": (C.c_int, [C.POINTER(LayerDesc), _i32, C.POINTER(_vp)]),
    "gce_table_destroy": (C.c_int, [_vp]),
    "gce_table_get_totals": (C.c_int, [_vp, C.POINTER(Totals)]),
    "gce_table_get_layer": (C.c_int, [_vp, _i32, C.POINTER(LayerInfo)]),
    "gce_workspace_bytes": (C.c_int, [_vp, _i32, _i32, C.POINTER(C.c_size_t)]),
    "ef_topk_step": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "ef_randk_step": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _u64, _u64, _vp, _vp, _vp,
                                C.c_size_t, _vp]),
    "ef_randk_step_at": (C.c_int, [_vp, C.c_int64, _i32, _vp, _vp, _f32, _vp, _u64, _u64, _vp,
                                   _vp, _vp, C.c_size_t, _vp]),
    "powersgd_init_q": (C.c_int, [_vp, _i32, _u64, _vp, _vp]),
    "powersgd_step": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp,
                                C.c_size_t, _vp]),
    "powersgd_dp_step": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp,
                                   C.c_size_t, _vp]),
    "powersgd_step_lazy": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp,
                                     C.c_size_t, _vp]),
    "gce_materialize_memory": (C.c_int, [_vp, _i32, _vp, _vp, _vp, C.c_size_t, _vp]),
    "gce_powersgd_dp_partials": (C.c_int, [_vp, C.POINTER(_i64)]),
    "accordion_sumsq": (C.c_int, [_vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "accordion_decide": (C.c_int, [_vp, _vp, _i64, _i32, _f64, _i32, _i32, _vp, _vp, _vp, _vp,
                                   _vp]),
    "powersgd_dp_encode": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp,
                                     C.c_size_t, _vp]),
    "powersgd_dp_orthogonalize": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "powersgd_dp_project": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, C.c_size_t, _vp]),
    "powersgd_dp_mean": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ef_sign_step": (C.c_int, [_vp, _i32, _vp, _vp, _f32, _vp, _vp, C.c_size_t, _vp]),
    "decompress_vote": (C.c_int, [_vp, _i32, _vp, _f32, _vp, _vp]),
    "accordion_init": (C.c_int, [_vp, _vp, _vp, _vp]),
    "accordion_select": (C.c_int, [_vp, _vp, _i64, _i32, _f64, _i32, _i32, _vp, _vp, _vp, _vp,
                                   _vp, C.c_size_t, _vp]),
    "decompress_accumulate": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp,
                                        C.c_size_t, _vp]),
    "decompress_accumulate_noalloc": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _f32, _vp,
                                                _vp]),
    "decompress_apply": (C.c_int, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp,
                                   C.c_size_t, _vp]),
    "gce_memsgd_eta": (C.c_int, [_i64, _f64, _f64, C.POINTER(_f32)]),
    "gce_status": (C.c_int, [_vp, _vp, C.POINTER(_i32)]),
    "gce_launch_count": (_u64, []),
    "gce_error_string": (C.c_char_p, [C.c_int]),
    "gce_set_bracket_sigma": (C.c_int, [_f64]),
    "gce_table_set_option": (C.c_int, [_vp, _i32, _f64]),
    "gce_table_reset_option": (C.c_int, [_vp, _i32]),
    "gce_table_get_option": (C.c_int, [_vp, _i32, C.POINTER(_f64)]),
    "gce_set_randk_ahead": (C.c_int, [C.c_int32]),
    "gce_set_sign_ahead": (C.c_int, [C.c_int32]),
    "gce_set_sign_emit_first": (C.c_int, [C.c_int32]),
    "gce_sign_schedule": (C.c_int, [_vp, _i32, _i32, _i32, _vp, _i64, C.POINTER(_i64)]),
    "gce_profile_start": (C.c_int, []),
    "gce_profile_stop": (C.c_int, []),
    "gce_profile_only": (C.c_int, [C.c_char_p]),
    "gce_profile_count": (C.c_int, []),
    "gce_profile_get": (C.c_int, [_i32, C.c_char_p, _i32, C.POINTER(_f64), C.POINTER(_i64)]),
}

_lib = None


def lib():
    """Load libgce.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgce.so is not built; run "
                               "`python -m gradient_compression_error_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(fn, rc):
    if rc != 0:
        raise GceError(fn, rc)


def _ptr(t, dtype=None):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError("expected dtype %s, got %s" % (dtype, t.dtype))
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


class Table:
    """A gce_table: layers described by dicts {rows, cols, kind, cap}."""

    def __init__(self, layers):
        self.layers = [dict(l) for l in layers]
        arr = (LayerDesc * len(layers))()
        for i, l in enumerate(layers):
            arr[i] = LayerDesc(int(l["rows"]), int(l["cols"]), KIND[l["kind"]], int(l.get("cap", 0)))
        h = C.c_void_p()
        _check("gce_table_create", lib().gce_table_create(arr, len(layers), C.byref(h)))
        self.handle = h
        tot = Totals()
        _check("gce_table_get_totals", lib().gce_table_get_totals(h, C.byref(tot)))
        self.L, self.N = tot.L, tot.N
        self.vals_per_worker = tot.vals_per_worker
        self.P_per_worker, self.Q_per_worker = tot.P_per_worker, tot.Q_per_worker
        self.compressed_kind = tot.compressed_kind
        self.info = []
        for i in range(len(layers)):
            li = LayerInfo()
            _check("gce_table_get_layer", lib().gce_table_get_layer(h, i, C.byref(li)))
            self.info.append({f: getattr(li, f) for f, _ in LayerInfo._fields_})

    def close(self):
        if self.handle is not None and self.handle.value:
            lib().gce_table_destroy(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_option(self, name, value):
        """This table's own value of a setting (include/gce.h, GCE_OPT_*)."""
        _check("gce_table_set_option", lib().gce_table_set_option(self.handle, OPT[name],
                                                                  float(value)))

    def reset_option(self, name):
        """Follow the process-wide value of a setting again."""
        _check("gce_table_reset_option", lib().gce_table_reset_option(self.handle, OPT[name]))

    def option(self, name):
        """The value of a setting that a call on this table uses now."""
        v = C.c_double()
        _check("gce_table_get_option", lib().gce_table_get_option(self.handle, OPT[name],
                                                                  C.byref(v)))
        return v.value

    def workspace_bytes(self, W, op):
        n = C.c_size_t()
        _check("gce_workspace_bytes", lib().gce_workspace_bytes(self.handle, int(W), OP[op],
                                                                C.byref(n)))
        return n.value

    def workspace(self, W, op, device="cuda"):
        """A zero-filled uint8 CUDA tensor of the size the operation needs."""
        import torch
        return torch.zeros(max(self.workspace_bytes(W, op), WS_HEADER_BYTES), dtype=torch.uint8,
                           device=device)


def _f32():
    import torch
    return torch.float32


def _i32():
    import torch
    return torch.int32


def ef_topk_step(table, W, grad, mem, eta, k_or_rank, vals, idx, ws, stream=None):
    _check("ef_topk_step", lib().ef_topk_step(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), _ptr(vals, _f32()), _ptr(idx, _i32()), _ptr(ws), ws.numel(),
        _stream(stream)))


def ef_randk_step(table, W, grad, mem, eta, k_or_rank, seed, step, vals, idx, ws, stream=None):
    _check("ef_randk_step", lib().ef_randk_step(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), int(seed), int(step), _ptr(vals, _f32()), _ptr(idx, _i32()),
        _ptr(ws), ws.numel(), _stream(stream)))


def ef_randk_step_at(table, worker0, W, grad, mem, eta, k_or_rank, seed, step, vals, idx, ws,
                     stream=None):
    """ef_randk_step for job-wide workers worker0 .. worker0+W-1 (include/gce.h)."""
    _check("ef_randk_step_at", lib().ef_randk_step_at(
        table.handle, int(worker0), int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), int(seed), int(step), _ptr(vals, _f32()), _ptr(idx, _i32()),
        _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_init_q(table, W, seed, Q, stream=None):
    _check("powersgd_init_q", lib().powersgd_init_q(table.handle, int(W), int(seed),
                                                    _ptr(Q, _f32()), _stream(stream)))


def powersgd_step(table, W, grad, mem, eta, k_or_rank, P, Q, vals, dense_out, ws, stream=None):
    _check("powersgd_step", lib().powersgd_step(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), _ptr(P, _f32()), _ptr(Q, _f32()), _ptr(vals, _f32()),
        _ptr(dense_out, _f32()), _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_step_lazy(table, W, grad, mem, eta, k_or_rank, P, Q, vals, lazy_rank, ws,
                       stream=None):
    """powersgd_step leaving M in the memory; lazy_rank (int32 [W, L]) records
    the factors to take off (include/gce.h)."""
    _check("powersgd_step_lazy", lib().powersgd_step_lazy(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), _ptr(P, _f32()), _ptr(Q, _f32()), _ptr(vals, _f32()),
        _ptr(lazy_rank, _i32()), _ptr(ws), ws.numel(), _stream(stream)))


def materialize_memory(table, W, mem, lazy_rank, ws, stream=None):
    """mem <- M - P Q^T where lazy steps left M (their workspace ws holds the
    factors); lazy_rank -> 0."""
    _check("gce_materialize_memory", lib().gce_materialize_memory(
        table.handle, int(W), _ptr(mem, _f32()), _ptr(lazy_rank, _i32()), _ptr(ws), ws.numel(),
        _stream(stream)))


def powersgd_dp_step(table, W, grad, mem, eta, k_or_rank, P, Q, vals, ws, stream=None):
    """Data-parallel PowerSGD over the W workers: shared P and Q (the mean),
    per-worker memory (include/gce.h)."""
    _check("powersgd_dp_step", lib().powersgd_dp_step(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), _ptr(P, _f32()), _ptr(Q, _f32()), _ptr(vals, _f32()),
        _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_dp_partials(table):
    """fp64 partial products per worker that powersgd_dp_encode writes."""
    n = _i64()
    _check("gce_powersgd_dp_partials", lib().gce_powersgd_dp_partials(table.handle, C.byref(n)))
    return n.value


def powersgd_dp_encode(table, W, grad, mem, eta, k_or_rank, Q, Ppart, vals, ws, stream=None):
    """Data-parallel PowerSGD, first part: M into mem, partial M Q per worker
    (float64 [W, partials]), DENSE residual rows into vals (include/gce.h)."""
    import torch
    _check("powersgd_dp_encode", lib().powersgd_dp_encode(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(k_or_rank, _i32()), _ptr(Q, _f32()), _ptr(Ppart, torch.float64),
        _ptr(vals, _f32()), _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_dp_orthogonalize(table, W, k_or_rank, Ppart, P, ws, stream=None):
    """P from the gathered partials of all W workers."""
    import torch
    _check("powersgd_dp_orthogonalize", lib().powersgd_dp_orthogonalize(
        table.handle, int(W), _ptr(k_or_rank, _i32()), _ptr(Ppart, torch.float64),
        _ptr(P, _f32()), _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_dp_project(table, W, mem, k_or_rank, Qw, ws, stream=None):
    """Q_w = M_w^T P per worker into Qw, each worker's residual into mem."""
    _check("powersgd_dp_project", lib().powersgd_dp_project(
        table.handle, int(W), _ptr(mem, _f32()), _ptr(k_or_rank, _i32()), _ptr(Qw, _f32()),
        _ptr(ws), ws.numel(), _stream(stream)))


def powersgd_dp_mean(table, W, k_or_rank, Qw, Q, vals_all, vals, stream=None):
    """The workers' mean Q and DENSE payloads from the gathered rows."""
    _check("powersgd_dp_mean", lib().powersgd_dp_mean(
        table.handle, int(W), _ptr(k_or_rank, _i32()), _ptr(Qw, _f32()), _ptr(Q, _f32()),
        _ptr(vals_all, _f32()), _ptr(vals, _f32()), _stream(stream)))


def ef_sign_step(table, W, grad, mem, eta, vals, ws, stream=None):
    """signSGD with error feedback; vals holds each SIGN layer's scale (slot
    0) and sign words (slots 4..., uint32 bit patterns) (include/gce.h)."""
    _check("ef_sign_step", lib().ef_sign_step(
        table.handle, int(W), _ptr(grad, _f32()), _ptr(mem, _f32()), float(eta),
        _ptr(vals), _ptr(ws), ws.numel(), _stream(stream)))


def decompress_vote(table, W, vals, scale, out, stream=None):
    """sign SGD's majority vote over the workers' sign payloads."""
    _check("decompress_vote", lib().decompress_vote(
        table.handle, int(W), _ptr(vals), float(scale), _ptr(out, _f32()), _stream(stream)))


def accordion_init(table, prev_norm, level, stream=None):
    import torch
    _check("accordion_init", lib().accordion_init(table.handle, _ptr(prev_norm, torch.float64),
                                                  _ptr(level, _i32()), _stream(stream)))


def accordion_select(table, grad, step, interval, threshold, lvl_low, lvl_high, prev_norm, level,
                     cur_norm, k_or_rank_out, ws, stream=None):
    import torch
    _check("accordion_select", lib().accordion_select(
        table.handle, _ptr(grad, _f32()), int(step), int(interval), float(threshold),
        int(lvl_low), int(lvl_high), _ptr(prev_norm, torch.float64), _ptr(level, _i32()),
        _ptr(cur_norm, torch.float64), _ptr(k_or_rank_out, _i32()), _ptr(ws), ws.numel(),
        _stream(stream)))


def accordion_sumsq(table, grad, sumsq, ws, stream=None):
    """Per-layer sum of squares of grad (float64 [L]); see accordion_decide."""
    import torch
    _check("accordion_sumsq", lib().accordion_sumsq(
        table.handle, _ptr(grad, _f32()), _ptr(sumsq, torch.float64), _ptr(ws), ws.numel(),
        _stream(stream)))


def accordion_decide(table, sumsq, step, interval, threshold, lvl_low, lvl_high, prev_norm, level,
                     cur_norm, k_or_rank_out, stream=None):
    """accordion_select's decision from given per-layer sums of squares."""
    import torch
    _check("accordion_decide", lib().accordion_decide(
        table.handle, _ptr(sumsq, torch.float64), int(step), int(interval), float(threshold),
        int(lvl_low), int(lvl_high), _ptr(prev_norm, torch.float64), _ptr(level, _i32()),
        _ptr(cur_norm, torch.float64), _ptr(k_or_rank_out, _i32()), _stream(stream)))


def decompress_accumulate(table, W, vals, idx, k_or_rank, P, Q, scale, out, ws, stream=None):
    _check("decompress_accumulate", lib().decompress_accumulate(
        table.handle, int(W), _ptr(vals, _f32()), _ptr(idx, _i32()), _ptr(k_or_rank, _i32()),
        _ptr(P, _f32()), _ptr(Q, _f32()), float(scale), _ptr(out, _f32()), _ptr(ws), ws.numel(),
        _stream(stream)))


def decompress_apply(table, W, vals, idx, k_or_rank, P, Q, scale, x, ws, stream=None):
    """x -= scale * (worker-order sum of the payloads), in place (include/gce.h)."""
    _check("decompress_apply", lib().decompress_apply(
        table.handle, int(W), _ptr(vals, _f32()), _ptr(idx, _i32()), _ptr(k_or_rank, _i32()),
        _ptr(P, _f32()), _ptr(Q, _f32()), float(scale), _ptr(x, _f32()), _ptr(ws), ws.numel(),
        _stream(stream)))


def memsgd_eta(step, mu, a):
    """Step size 8 / (mu (a + t)) of the Mem-SGD method, as a float."""
    e = C.c_float()
    _check("gce_memsgd_eta", lib().gce_memsgd_eta(int(step), float(mu), float(a), C.byref(e)))
    return e.value


def decompress_accumulate_noalloc(table, W, vals, idx, k_or_rank, P, Q, scale, out, stream=None):
    """decompress_accumulate for callers that cannot allocate a workspace: the
    library's fixed 4 MiB scratch is used instead (see include/gce.h)."""
    _check("decompress_accumulate_noalloc", lib().decompress_accumulate_noalloc(
        table.handle, int(W), _ptr(vals, _f32()), _ptr(idx, _i32()), _ptr(k_or_rank, _i32()),
        _ptr(P, _f32()), _ptr(Q, _f32()), float(scale), _ptr(out, _f32()), _stream(stream)))


def status(ws, stream=None):
    """Wait for the stream, then read and clear the workspace status word."""
    st = C.c_int32()
    _check("gce_status", lib().gce_status(_ptr(ws), _stream(stream), C.byref(st)))
    return st.value


def launch_count():
    return int(lib().gce_launch_count())


def profile_start():
    _check("gce_profile_start", lib().gce_profile_start())


def profile_only(name_prefix=None):
    """Record only kernels whose name starts with name_prefix (None: all)."""
    _check("gce_profile_only", lib().gce_profile_only(
        None if name_prefix is None else name_prefix.encode()))


def profile_stop():
    """Stop timing launches; returns {kernel name: (total ms, launches)}."""
    _check("gce_profile_stop", lib().gce_profile_stop())
    out = {}
    for i in range(lib().gce_profile_count()):
        buf = C.create_string_buffer(256)
        ms, n = C.c_double(), C.c_int64()
        _check("gce_profile_get", lib().gce_profile_get(i, buf, 256, C.byref(ms), C.byref(n)))
        out[buf.value.decode()] = (ms.value, n.value)
    return out


def set_bracket_sigma(sigma):
    _check("gce_set_bracket_sigma", lib().gce_set_bracket_sigma(float(sigma)))


def set_randk_ahead(on):
    """Run the next rand-k step's key pass inside this one (include/gce.h)."""
    _check("gce_set_randk_ahead", lib().gce_set_randk_ahead(1 if on else 0))


def set_sign_ahead(tiles):
    """signSGD schedule: the norm runs `tiles` 8192-element tiles ahead of the
    memory update in one launch; 0 runs two passes; -1 (the default) sizes the
    look-ahead from the device's L2 (include/gce.h)."""
    _check("gce_set_sign_ahead", lib().gce_set_sign_ahead(int(tiles)))


def sign_schedule(layer_tiles, W, ahead):
    """The pipelined signSGD kernel's work-item order (host only): a list of
    runs (first item, lowest tile, kind, descending), kind 0 norm, 1 update,
    -1 the closing sentinel whose first item is the item count; descending 1:
    the run's tiles from the highest down (include/gce.h)."""
    tiles = (C.c_int32 * len(layer_tiles))(*[int(x) for x in layer_tiles])
    n = _i64()
    _check("gce_sign_schedule", lib().gce_sign_schedule(tiles, len(layer_tiles), int(W),
                                                        int(ahead), None, 0, C.byref(n)))
    runs = (C.c_int64 * (4 * n.value))()
    _check("gce_sign_schedule", lib().gce_sign_schedule(tiles, len(layer_tiles), int(W),
                                                        int(ahead), runs, n.value, C.byref(n)))
    return [tuple(runs[4 * i + j] for j in range(4)) for i in range(n.value)]


def set_sign_emit_first(on):
    """Test of the bounded wait: every memory-update tile before every norm
    tile, so the waits run out and GCE_STATUS_WAIT_TIMEOUT is set."""
    _check("gce_set_sign_emit_first", lib().gce_set_sign_emit_first(1 if on else 0))
