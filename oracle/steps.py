"""Table-level loops of the CPU oracle: one step over every (worker, layer).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  A layer is a dict with
keys rows, cols, kind ('topk' | 'randk' | 'powersgd' | 'dense'); layers sit
back to back in flat per-worker buffers of N = sum(rows*cols) floats.  The
units are independent, so the loops below may run them on a thread pool
(ctypes releases the GIL); results do not depend on the thread count.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import (accordion_decide, accum_dense, accum_lowrank, accum_sign, accum_sparse,
               dense_dp_unit, dense_unit, ef_randk_unit, ef_sign_unit, ef_topk_unit, k_from_ppm,
               layer_norm, powersgd_dp_unit, powersgd_init_q, powersgd_unit, scale, vote_sign)


def layer_offsets(layers):
    offs, o = [], 0
    for lay in layers:
        offs.append(o)
        o += lay["rows"] * lay["cols"]
    return offs, o


def _run(units, fn, threads):
    if threads <= 1:
        return [fn(u) for u in units]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, units))


def sparse_step(layers, grad, mem, eta, k_per_layer, method="topk", seed=0, step=0,
                units=None, threads=1):
    """Mem-SGD top-k / rand-k step (Sparsified SGD with Memory, Method), or
    with method="sign" signSGD with the same memory (On the Utility of
    Gradient Compression, Method: sign SGD).

    grad, mem: (W, N) float32; mem is updated in place.  Layers whose kind is
    'dense' are sent whole.  Returns {(w, l): (vals, idx)} for top-k / rand-k
    layers, {(w, l): (scale, words)} for sign layers and {(w, l): payload}
    for dense ones.  k_per_layer is unused for sign.
    """
    offs, N = layer_offsets(layers)
    W = grad.shape[0]
    if units is None:
        units = [(w, l) for w in range(W) for l in range(len(layers))]

    def one(u):
        w, l = u
        lay = layers[l]
        n = lay["rows"] * lay["cols"]
        sl = slice(offs[l], offs[l] + n)
        if lay["kind"] == "dense":
            pay, m_new = dense_unit(grad[w, sl], mem[w, sl], eta)
            return u, pay, None, m_new
        if method == "sign":
            sc, words, m_new = ef_sign_unit(grad[w, sl], mem[w, sl], eta)
            return u, sc, words, m_new
        k = int(k_per_layer[l])
        if method == "topk":
            vals, idx, m_new = ef_topk_unit(grad[w, sl], mem[w, sl], k, eta)
        else:
            vals, idx, m_new = ef_randk_unit(grad[w, sl], mem[w, sl], k, eta, seed,
                                             w, l, step)
        return u, vals, idx, m_new

    out = {}
    for u, a, b, m_new in _run(units, one, threads):
        w, l = u
        lay = layers[l]
        mem[w, offs[l]:offs[l] + lay["rows"] * lay["cols"]] = m_new
        out[u] = a if b is None else (a, b)
    return out


def powersgd_init(layers, W, r_max_per_layer, seed):
    """Warm-start Q for every (worker, PowerSGD layer)."""
    return {(w, l): powersgd_init_q(layers[l]["cols"], r_max_per_layer[l], seed, w, l)
            for w in range(W) for l, lay in enumerate(layers) if lay["kind"] == "powersgd"}


def powersgd_step(layers, grad, mem, eta, rank_per_layer, Qs, units=None, threads=1,
                  want_mhat=True):
    """PowerSGD step with error feedback; Qs {(w, l): Q} is updated in place.

    Returns {(w, l): (P, Mhat)} for PowerSGD layers and {(w, l): payload} for
    dense ones.
    """
    offs, N = layer_offsets(layers)
    W = grad.shape[0]
    if units is None:
        units = [(w, l) for w in range(W) for l in range(len(layers))]

    def one(u):
        w, l = u
        lay = layers[l]
        rows, cols = lay["rows"], lay["cols"]
        sl = slice(offs[l], offs[l] + rows * cols)
        if lay["kind"] == "dense":
            pay, m_new = dense_unit(grad[w, sl], mem[w, sl], eta)
            return u, pay, None, None, m_new
        P, Qn, m_new, Mhat = powersgd_unit(grad[w, sl].reshape(rows, cols),
                                           mem[w, sl].reshape(rows, cols), Qs[u],
                                           int(rank_per_layer[l]), eta, want_mhat)
        return u, P, Qn, Mhat, m_new.reshape(-1)

    out = {}
    for u, a, Qn, Mhat, m_new in _run(units, one, threads):
        w, l = u
        lay = layers[l]
        mem[w, offs[l]:offs[l] + lay["rows"] * lay["cols"]] = m_new
        if Qn is None:
            out[u] = a
        else:
            Qs[u] = Qn
            out[u] = (a, Mhat)
    return out


def powersgd_dp_step(layers, grad, mem, eta, rank_per_layer, Qs, units=None, threads=1):
    """Data-parallel PowerSGD step over all W workers of grad / mem (W, N):
    P summed over the workers, one orthonormal P, each worker's own Q_w and
    residual, Q the workers' mean ("On the Utility of Gradient Compression",
    Key results: PowerSGD is all-reduce compatible).  Qs {l: Q} (shared per
    layer) is updated in place; mem is updated in place.

    Returns {l: P} for PowerSGD layers and {l: mean payload} for dense ones.
    units: the layer ids to run (default all).
    """
    offs, N = layer_offsets(layers)
    W = grad.shape[0]
    if units is None:
        units = list(range(len(layers)))

    def one(l):
        lay = layers[l]
        rows, cols = lay["rows"], lay["cols"]
        sl = slice(offs[l], offs[l] + rows * cols)
        if lay["kind"] == "dense":
            pay, m_new = dense_dp_unit(grad[:, sl], mem[:, sl], eta)
            return l, pay, None, m_new
        P, Qn, m_new = powersgd_dp_unit(grad[:, sl].reshape(W, rows, cols),
                                        mem[:, sl].reshape(W, rows, cols), Qs[l],
                                        int(rank_per_layer[l]), eta)
        return l, P, Qn, m_new.reshape(W, -1)

    out = {}
    for l, a, Qn, m_new in _run(units, one, threads):
        lay = layers[l]
        mem[:, offs[l]:offs[l] + lay["rows"] * lay["cols"]] = m_new
        if Qn is not None:
            Qs[l] = Qn
        out[l] = a
    return out


class AccordionState:
    """Per-layer Accordion state: previous check's norm (-1 = none) and level.

    Levels: 0 = LOW (l_low, less compression), 1 = HIGH (l_high).
    """

    def __init__(self, L):
        self.prev_norm = np.full(L, -1.0)
        self.level = np.zeros(L, np.int32)
        self.norms = np.zeros(L)


def accordion_step(layers, grad, step, interval, threshold, state, lvl_low, lvl_high):
    """One Accordion select (Accordion, Method).

    grad: (N,) float32 raw gradient.  On a check step (step % interval == 0)
    every compressed layer's norm is taken and its level decided; other steps
    keep the levels.  lvl_low / lvl_high are ranks for PowerSGD layers and k
    fractions in ppm for top-k / rand-k layers.  Returns k_or_rank per layer
    (0 for dense layers).
    """
    offs, N = layer_offsets(layers)
    check = (step % interval) == 0
    out = np.zeros(len(layers), np.int64)
    for l, lay in enumerate(layers):
        n = lay["rows"] * lay["cols"]
        if lay["kind"] == "dense":
            continue
        if check:
            s = layer_norm(grad[offs[l]:offs[l] + n])
            state.norms[l] = s
            state.level[l] = accordion_decide(state.prev_norm[l], s, threshold)
            state.prev_norm[l] = s
        p = lvl_low if state.level[l] == 0 else lvl_high
        out[l] = p if lay["kind"] == "powersgd" else k_from_ppm(n, p)
    return out


def decompress(layers, W, payload, scale_factor, rank_per_layer=None, k_per_layer=None):
    """Dense aggregate of the W workers' payloads (On the Utility of Gradient
    Compression, Key results: payloads are summed across workers).

    payload {(w, l): (vals, idx) | (P, Q) | dense}; sparse payloads use the
    first k_per_layer[l] entries, low-rank ones the first rank_per_layer[l]
    columns.  Sum in worker order from +0.0 in fp32, then times the scale.
    """
    offs, N = layer_offsets(layers)
    out = np.zeros(N, np.float32)
    for w in range(W):
        for l, lay in enumerate(layers):
            rows, cols = lay["rows"], lay["cols"]
            view = out[offs[l]:offs[l] + rows * cols]
            p = payload[(w, l)]
            if lay["kind"] == "dense":
                accum_dense(view, p)
            elif lay["kind"] == "powersgd":
                P, Q = p
                accum_lowrank(view, P, Q, int(rank_per_layer[l]))
            elif lay["kind"] == "sign":
                sc, words = p
                accum_sign(view, sc, words)
            else:
                vals, idx = p
                k = int(k_per_layer[l]) if k_per_layer is not None else len(vals)
                accum_sparse(view, vals[:k], idx[:k])
    scale(out, scale_factor)
    return out


def apply_update(layers, W, payload, scale_factor, x, rank_per_layer=None, k_per_layer=None):
    """Parameter update of "Sparsified SGD with Memory", Method: x_{t+1} =
    x_t - g_t, with the W workers' updates combined as `decompress` combines
    them: x - fl(scale * S), one fp32 round-to-nearest subtraction per
    element.  Returns the new x (float32)."""
    u = decompress(layers, W, payload, scale_factor, rank_per_layer, k_per_layer)
    return np.subtract(np.asarray(x, np.float32), u, dtype=np.float32)


def memsgd_eta(t, mu, a):
    """Step size eta_t = 8 / (mu (a + t)) of "Sparsified SGD with Memory",
    Method, in fp64, rounded once to fp32."""
    return np.float32(8.0 / (float(mu) * (float(a) + float(t))))


def vote(layers, W, payload, scale_factor):
    """Majority-vote aggregate of sign payloads (sign SGD's aggregation, On
    the Utility of Gradient Compression, Method): per element scale *
    sign(#positive - #negative) over the workers, 0 on a tie; dense layers
    are summed as `decompress` sums them."""
    offs, N = layer_offsets(layers)
    out = np.zeros(N, np.float32)
    for l, lay in enumerate(layers):
        n = lay["rows"] * lay["cols"]
        view = out[offs[l]:offs[l] + n]
        if lay["kind"] == "dense":
            for w in range(W):
                accum_dense(view, payload[(w, l)])
            scale(view, scale_factor)
        else:
            words = np.stack([payload[(w, l)][1] for w in range(W)])
            view[:] = vote_sign(words, n, scale_factor)
    return out
