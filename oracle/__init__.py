"""Python face of the CPU oracle (oracle/gce_oracle.c).

TEST INFRASTRUCTURE ONLY: the parity tests, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may use this module; the product
library never imports it.  Every function handles one unit (one worker's
layer) with numpy arrays on the host; table-level loops live in
oracle/steps.py.

See oracle/gce_oracle.c for the definitions followed and their sources.
"""
import ctypes as C

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, u64, f32, f64, i32, u32 = (C.c_int64, C.c_uint64, C.c_float,
                                        C.c_double, C.c_int32, C.c_uint32)
        vp = C.c_void_p
        sig = {
            "or_k_from_ppm": (i64, [i64, i64]),
            "or_ef_topk": (C.c_int, [i64, i64, f32, vp, vp, vp, vp]),
            "or_splitmix64_output": (u64, [u64, u64]),
            "or_randk_base": (u64, [u64, u64, u64, u64, u64]),
            "or_randk_key": (u32, [u64, i64]),
            "or_ef_randk": (C.c_int, [i64, i64, f32, vp, vp, vp, vp, u64, u64, u64, u64]),
            "or_dense": (C.c_int, [i64, f32, vp, vp, vp]),
            "or_powersgd_init_q": (C.c_int, [i64, i64, u64, u64, u64, vp]),
            "or_q_entry": (f32, [u64]),
            "or_powersgd": (C.c_int, [i64, i64, i64, i64, f32, vp, vp, vp, vp, vp]),
            "or_powersgd_dp": (C.c_int, [i64, i64, i64, i64, i64, f32, vp, vp, vp, vp]),
            "or_dense_dp": (C.c_int, [i64, i64, f32, vp, vp, vp]),
            "or_powersgd_dp_p": (C.c_int, [i64, i64, i64, i64, f32, vp, vp, vp, vp]),
            "or_mgs": (None, [i64, i64, vp]),
            "or_powersgd_dp_q": (C.c_int, [i64, i64, i64, vp, vp, vp]),
            "or_ef_sign": (C.c_int, [i64, f32, vp, vp, vp, vp]),
            "or_accum_sign": (None, [i64, f32, vp, vp]),
            "or_vote_sign": (None, [i64, i64, i64, vp, f32, vp]),
            "or_layer_norm": (f64, [i64, vp]),
            "or_layer_sumsq": (f64, [i64, vp]),
            "or_accordion_decide": (i32, [f64, f64, f64]),
            "or_accum_sparse": (None, [i64, vp, vp, vp]),
            "or_accum_dense": (None, [i64, vp, vp]),
            "or_accum_lowrank": (None, [i64, i64, i64, i64, vp, vp, vp]),
            "or_scale": (None, [i64, f32, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with status %d" % (what, rc))


def k_from_ppm(n, ppm):
    return int(lib().or_k_from_ppm(int(n), int(ppm)))


def ef_topk_unit(g, m, k, eta):
    """Mem-SGD top-k step on one unit.  Returns (vals, idx, m_new)."""
    g = _f32(g)
    m = _f32(m).copy()
    n = g.size
    vals = np.empty(k, np.float32)
    idx = np.empty(k, np.int32)
    _check(lib().or_ef_topk(n, int(k), float(np.float32(eta)), _ptr(g), _ptr(m),
                            _ptr(vals), _ptr(idx)), "ef_topk")
    return vals, idx, m


def splitmix64_output(state, j):
    return int(lib().or_splitmix64_output(int(state) & (2**64 - 1), int(j)))


def randk_base(seed, stream, worker, layer, step):
    return int(lib().or_randk_base(seed, stream, worker, layer, step))


def randk_key(base, i):
    return int(lib().or_randk_key(int(base), int(i)))


def ef_randk_unit(g, m, k, eta, seed, worker, layer, step):
    """Mem-SGD rand-k step on one unit.  Returns (vals, idx, m_new)."""
    g = _f32(g)
    m = _f32(m).copy()
    n = g.size
    vals = np.empty(k, np.float32)
    idx = np.empty(k, np.int32)
    _check(lib().or_ef_randk(n, int(k), float(np.float32(eta)), _ptr(g), _ptr(m),
                             _ptr(vals), _ptr(idx), int(seed), int(worker),
                             int(layer), int(step)), "ef_randk")
    return vals, idx, m


def dense_unit(g, m, eta):
    """Uncompressed layer.  Returns (payload, m_new)."""
    g = _f32(g)
    m = _f32(m).copy()
    out = np.empty_like(g)
    _check(lib().or_dense(g.size, float(np.float32(eta)), _ptr(g), _ptr(m), _ptr(out)),
           "dense")
    return out, m


def q_entry(h):
    """The warm-start Q entry in [-1, 1) of one 64-bit generator output."""
    return np.float32(lib().or_q_entry(int(h) & (2**64 - 1)))


def powersgd_init_q(cols, r_max, seed, worker, layer):
    Q = np.empty((cols, r_max), np.float32)
    _check(lib().or_powersgd_init_q(cols, r_max, seed, worker, layer, _ptr(Q)),
           "powersgd_init_q")
    return Q


def powersgd_unit(g, m, Q, r, eta, want_mhat=True):
    """PowerSGD step on one rows x cols unit.

    g, m: (rows, cols) float32; Q: (cols, r_max) float32 warm start.
    Returns (P (rows, r_max), Q_new (cols, r_max), m_new, Mhat or None); columns
    >= r of P are zero and of Q_new are copied from Q.
    """
    g = _f32(g)
    rows, cols = g.shape
    m = _f32(m).copy()
    Q = _f32(Q).copy()
    r_max = Q.shape[1]
    P = np.zeros((rows, r_max), np.float32)
    Mhat = np.empty((rows, cols), np.float32) if want_mhat else None
    _check(lib().or_powersgd(rows, cols, int(r), r_max, float(np.float32(eta)), _ptr(g),
                             _ptr(m), _ptr(Q), _ptr(P),
                             _ptr(Mhat) if want_mhat else None), "powersgd")
    return P, Q, m, Mhat


def powersgd_dp_unit(g, m, Q, r, eta):
    """Data-parallel PowerSGD step on one matrix over W workers.

    g, m: (W, rows, cols) float32; Q: (cols, r_max) shared warm start.
    Returns (P (rows, r_max), Q_new (cols, r_max), m_new (W, rows, cols));
    columns >= r of P are zero and of Q_new are copied from Q.
    """
    g = _f32(g)
    W, rows, cols = g.shape
    m = _f32(m).copy()
    Q = _f32(Q).copy()
    r_max = Q.shape[1]
    P = np.zeros((rows, r_max), np.float32)
    _check(lib().or_powersgd_dp(W, rows, cols, int(r), r_max, float(np.float32(eta)), _ptr(g),
                                _ptr(m), _ptr(Q), _ptr(P)), "powersgd_dp")
    return P, Q, m


def powersgd_dp_p_unit(g, m, Q, r, eta):
    """Phase 1 of the data-parallel step for one worker's matrix: returns
    (M_w (rows, cols) float32, P_w = M_w Q (rows, r) float64)."""
    g = _f32(g)
    rows, cols = g.shape
    m = _f32(m).copy()
    Q = _f32(Q)
    Pw = np.zeros((rows, int(r)), np.float64)
    _check(lib().or_powersgd_dp_p(rows, cols, int(r), Q.shape[1], float(np.float32(eta)),
                                  _ptr(g), _ptr(m), _ptr(Q), _ptr(Pw)), "powersgd_dp_p")
    return m, Pw


def mgs(P):
    """Modified Gram-Schmidt of the columns of P (rows, r) float64, in order."""
    P = np.ascontiguousarray(P, np.float64).copy()
    lib().or_mgs(P.shape[0], P.shape[1], _ptr(P))
    return P


def powersgd_dp_q_unit(Pd, M):
    """Phase 2 for one worker: (Q_w = M^T P (cols, r) float64, residual
    M - P Q_w^T (rows, cols) float32)."""
    Pd = np.ascontiguousarray(Pd, np.float64)
    m = _f32(M).copy()
    rows, cols = m.shape
    Qw = np.zeros((cols, Pd.shape[1]), np.float64)
    _check(lib().or_powersgd_dp_q(rows, cols, Pd.shape[1], _ptr(Pd), _ptr(m), _ptr(Qw)),
           "powersgd_dp_q")
    return Qw, m


def dense_dp_unit(g, m, eta):
    """Data-parallel DENSE layer: g, m (W, n).  Returns (mean payload, m_new)."""
    g = _f32(g)
    W, n = g.shape
    m = _f32(m).copy()
    out = np.empty(n, np.float32)
    _check(lib().or_dense_dp(W, n, float(np.float32(eta)), _ptr(g), _ptr(m), _ptr(out)),
           "dense_dp")
    return out, m


def ef_sign_unit(g, m, eta):
    """signSGD with error feedback on one unit.  Returns (scale, words
    (uint32, ceil(n/32)), m_new)."""
    g = _f32(g)
    m = _f32(m).copy()
    n = g.size
    words = np.zeros((n + 31) // 32, np.uint32)
    sc = np.zeros(1, np.float32)
    _check(lib().or_ef_sign(n, float(np.float32(eta)), _ptr(g), _ptr(m), _ptr(sc), _ptr(words)),
           "ef_sign")
    return sc[0], words, m


def accum_sign(out, scale, words):
    words = np.ascontiguousarray(words, dtype=np.uint32)
    assert out.dtype == np.float32 and out.flags.c_contiguous
    assert words.size >= (out.size + 31) // 32
    lib().or_accum_sign(out.size, float(np.float32(scale)), _ptr(words), _ptr(out))


def vote_sign(words, n, out_scale):
    """words: (W, words_per_worker) uint32.  Returns the majority-vote
    update (n,) float32."""
    words = np.ascontiguousarray(words, dtype=np.uint32)
    W, wpw = words.shape
    assert wpw >= (n + 31) // 32
    out = np.empty(n, np.float32)
    lib().or_vote_sign(W, n, wpw, _ptr(words), float(np.float32(out_scale)), _ptr(out))
    return out


def layer_norm(g):
    g = _f32(g)
    return float(lib().or_layer_norm(g.size, _ptr(g)))


def layer_sumsq(g):
    g = _f32(g)
    return float(lib().or_layer_sumsq(g.size, _ptr(g)))


def accordion_decide(s_prev, s_cur, threshold):
    return int(lib().or_accordion_decide(float(s_prev), float(s_cur), float(threshold)))


def accum_sparse(out, vals, idx):
    vals = _f32(vals)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    assert out.dtype == np.float32 and out.flags.c_contiguous
    if idx.size and (idx.min() < 0 or idx.max() >= out.size):
        raise ValueError("index out of range")
    lib().or_accum_sparse(vals.size, _ptr(vals), _ptr(idx), _ptr(out))


def accum_dense(out, payload):
    payload = _f32(payload)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == payload.size
    lib().or_accum_dense(out.size, _ptr(payload), _ptr(out))


def accum_lowrank(out, P, Q, r):
    P = _f32(P)
    Q = _f32(Q)
    rows, r_max = P.shape
    cols = Q.shape[0]
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == rows * cols
    lib().or_accum_lowrank(rows, cols, int(r), r_max, _ptr(P), _ptr(Q), _ptr(out))


def scale(out, s):
    assert out.dtype == np.float32 and out.flags.c_contiguous
    lib().or_scale(out.size, float(np.float32(s)), _ptr(out))
