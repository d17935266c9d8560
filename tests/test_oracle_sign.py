"""Pins for the oracle's signSGD with error feedback (or_ef_sign) and its
two aggregates (worker-order sum, majority vote).

Source: "On the Utility of Gradient Compression in Distributed Training
Systems", Method / Key results: sign SGD sends one bit per element and,
lacking an all-reduce, is gathered; "Sparsified SGD with Memory", Method:
the memory keeps what was not sent.  The compressor sends s * sign(p) with
s the layer's mean |p|, so the memory keeps p - s sign(p).

Pins: a hand-worked layer; the bits equal numpy's signbit (negative zero
included) packed little-endian; n s equals the L1 norm of p within one fp32
rounding; m + s sign(p) gives back p; the sum decode against values worked by
hand; the vote against a counted example with a tie.
"""
import numpy as np

import oracle
from oracle import steps


def test_hand_worked_layer():
    sc, words, m = oracle.ef_sign_unit(np.zeros(4, np.float32),
                                       np.array([1, -2, 3, -4], np.float32), 0.05)
    assert sc == np.float32(2.5)                       # (1 + 2 + 3 + 4) / 4
    assert words.tolist() == [0b1010]
    assert m.tolist() == [-1.5, 0.5, 0.5, -1.5]


def test_bits_are_numpy_signbits_packed_little_endian():
    rng = np.random.default_rng(1)
    n = 1000
    g = rng.standard_normal(n).astype(np.float32)
    m = rng.standard_normal(n).astype(np.float32)
    g[7], m[7] = np.float32(0.0), np.float32(-0.0)     # p = -0.0 + 0.0 = +0.0
    g[8], m[8] = np.float32(-0.0), np.float32(-0.0)    # p = -0.0
    sc, words, m_new = oracle.ef_sign_unit(g, m, 0.5)
    p = (m + np.float32(0.5) * g).astype(np.float32)
    want = np.packbits(np.signbit(p).astype(np.uint8), bitorder="little")
    want = np.pad(want, (0, (-want.size) % 4)).view("<u4")
    assert np.array_equal(words, want)
    assert not (words[-1] >> np.uint32(n % 32)).any()   # unused high bits are 0
    assert np.signbit(p[8]) and not np.signbit(p[7])


def test_scale_is_the_mean_magnitude_and_memory_closes():
    rng = np.random.default_rng(2)
    n = 4097
    g = rng.standard_normal(n).astype(np.float32)
    m = (0.1 * rng.standard_normal(n)).astype(np.float32)
    sc, words, m_new = oracle.ef_sign_unit(g, m, 0.05)
    p = (m + np.float32(0.05) * g).astype(np.float32)
    l1 = np.abs(p.astype(np.float64)).sum()
    assert abs(float(sc) * n - l1) <= l1 * 2.0 ** -23
    sgn = np.where(np.signbit(p), -1.0, 1.0)
    back = m_new.astype(np.float64) + float(sc) * sgn
    assert np.allclose(back, p, rtol=0, atol=float(np.spacing(np.float32(np.abs(p).max()))))


def test_sum_and_vote_aggregates():
    layers = [dict(rows=5, cols=1, kind="sign"), dict(rows=2, cols=1, kind="dense")]
    # worker bits (1 = negative) on 5 elements
    bits = [[0, 1, 1, 0, 1], [0, 0, 1, 1, 0], [1, 0, 1, 1, 0]]
    scales = [np.float32(0.5), np.float32(0.25), np.float32(2.0)]
    pay = {}
    for w in range(3):
        word = np.array([sum(b << i for i, b in enumerate(bits[w]))], np.uint32)
        pay[(w, 0)] = (scales[w], word)
        pay[(w, 1)] = np.array([w, -w], np.float32)
    out = steps.decompress(layers, 3, pay, 1.0)
    # element 0: +0.5 + 0.25 - 2 ; 1: -0.5 + 0.25 + 2 ; 2: -2.75 ; 3: 0.5 - 0.25 - 2 ; 4: -0.5 + 0.25 + 2
    assert out[:5].tolist() == [-1.25, 1.75, -2.75, -1.75, 1.75]
    assert out[5:].tolist() == [3.0, -3.0]
    v = steps.vote(layers, 3, pay, 0.125)
    # positives minus negatives: 1, 1, -3, -1, 1
    assert v[:5].tolist() == [0.125, 0.125, -0.125, -0.125, 0.125]
    assert v[5:].tolist() == [0.375, -0.375]
    # a tie votes 0
    tie = {(0, 0): (scales[0], np.array([0b00001], np.uint32)),
           (1, 0): (scales[1], np.array([0b00000], np.uint32)),
           (0, 1): np.zeros(2, np.float32), (1, 1): np.zeros(2, np.float32)}
    vt = steps.vote(layers, 2, tie, 1.0)
    assert vt[0] == 0.0 and vt[1] == 1.0


def test_sign_step_updates_memory_per_worker():
    layers = [dict(rows=40, cols=3, kind="sign"), dict(rows=6, cols=1, kind="dense")]
    rng = np.random.default_rng(4)
    grad = rng.standard_normal((2, 126)).astype(np.float32)
    mem = np.zeros((2, 126), np.float32)
    out = steps.sparse_step(layers, grad, mem, 0.1, None, method="sign")
    for w in range(2):
        sc, words = out[(w, 0)]
        s2, w2, m2 = oracle.ef_sign_unit(grad[w, :120], np.zeros(120, np.float32), 0.1)
        assert sc == s2 and np.array_equal(words, w2) and np.array_equal(mem[w, :120], m2)
        assert not mem[w, 120:].any()


def test_sum_and_vote_at_forty_workers_against_numpy():
    """The oracle's aggregates over 40 workers (more than one 32-bit lane's
    worth) against their definitions written with numpy: the sum adds
    +-s_w worker by worker in fp32 from +0.0; the vote is the sign of
    (#positive - #negative) times the scale, 0 on a tie."""
    W, n = 40, 77
    layers = [dict(rows=n, cols=1, kind="sign")]
    rng = np.random.default_rng(12)
    neg = rng.integers(0, 2, (W, n)).astype(bool)
    scales = rng.uniform(0.01, 3.0, W).astype(np.float32)
    pay = {}
    for w in range(W):
        words = np.zeros((n + 31) // 32, np.uint32)
        for i in np.nonzero(neg[w])[0]:
            words[i // 32] |= np.uint32(1) << np.uint32(i % 32)
        pay[(w, 0)] = (scales[w], words)
    expect = np.zeros(n, np.float32)
    for w in range(W):
        expect = (expect + np.where(neg[w], -scales[w], scales[w])).astype(np.float32)
    expect = (expect * np.float32(0.5)).astype(np.float32)
    assert np.array_equal(steps.decompress(layers, W, pay, 0.5).view(np.uint32),
                          expect.view(np.uint32))
    margin = (~neg).sum(axis=0) - neg.sum(axis=0)
    vote = np.where(margin > 0, np.float32(0.25),
                    np.where(margin < 0, np.float32(-0.25), np.float32(0.0)))
    assert np.array_equal(steps.vote(layers, W, pay, 0.25), vote)
