"""The work-item order of the pipelined signSGD kernel (gce_sign_schedule),
checked on the host.

The kernel's waits end only if every memory-update tile comes after all norm
tiles of its (worker, layer): blocks take items in this order, an update waits
for its layer's scale, and a norm waits on nothing.  These tests check that
property, that each tile is normed once and updated once, that the norm runs
in ascending tile order and so do the updates, except that a layer of more
tiles than the look-ahead is updated from its last tile down (its last normed
tiles are the ones still in L2), and that the norm stays within the
look-ahead (beyond it only while a layer's norm tiles are still being
placed), on BERT-base-shaped and ragged tables.  The order is built by the
same C++ function the kernel's host code calls; no GPU is needed.
"""
import numpy as np
import pytest

from gradient_compression_error_b200 import workloads
from tests.helpers import gce

RUN = 64  # tiles per run of the schedule


def layer_tiles(layers):
    return [-(-(l["rows"] * l["cols"]) // 8192) for l in layers if l["kind"] == "sign"]


def expand(runs):
    """(kind, tile) of every item, in item order."""
    assert runs[-1][2] == -1
    kinds, tiles = [], []
    for (i0, t0, k, rev), (i1, _, _, _) in zip(runs, runs[1:]):
        assert i1 > i0 and k in (0, 1) and rev in (0, 1)
        assert not (k == 0 and rev)                     # norms always ascend
        kinds.append(np.full(i1 - i0, k, np.int8))
        t = np.arange(t0, t0 + i1 - i0, dtype=np.int64)
        tiles.append(t[::-1] if rev else t)
    return np.concatenate(kinds), np.concatenate(tiles)


def expected_update_order(tiles_per_layer, W, ahead):
    """Ascending tiles, each layer of more than `ahead` tiles reversed."""
    out, t = [], 0
    for _ in range(W):
        for n in tiles_per_layer:
            seg = np.arange(t, t + n, dtype=np.int64)
            out.append(seg[::-1] if ahead >= 1 and n > ahead else seg)
            t += n
    return np.concatenate(out)


def check(tiles_per_layer, W, ahead):
    g = gce()
    runs = g.sign_schedule(tiles_per_layer, W, ahead)
    tpw = sum(tiles_per_layer)
    T = W * tpw
    assert runs[-1] == (2 * T, T, -1, 0)
    kind, tile = expand(runs)
    assert len(kind) == 2 * T and tile.min() >= 0 and tile.max() < T
    norm_t, upd_t = tile[kind == 0], tile[kind == 1]
    assert np.array_equal(norm_t, np.arange(T))        # each tile normed once, in order
    # and updated once, long layers from the last tile down
    assert np.array_equal(upd_t, expected_update_order(tiles_per_layer, W, ahead))
    # segment (worker, layer) of every tile
    seg_of_local = np.repeat(np.arange(len(tiles_per_layer)), tiles_per_layer)
    seg = (np.arange(T) // tpw) * len(tiles_per_layer) + seg_of_local[np.arange(T) % tpw]
    pos = np.arange(2 * T)
    last_norm = np.zeros(seg.max() + 1, np.int64)
    np.maximum.at(last_norm, seg, pos[kind == 0])
    upd_pos = pos[kind == 1]
    if ahead >= 1:
        # every update after the last norm tile of its layer
        assert np.all(upd_pos > last_norm[seg]), (W, ahead)
        # the lead of the norm over the update: the look-ahead plus one run,
        # or more only while one layer's norm tiles are still being placed
        lead = np.cumsum(np.where(kind == 0, 1, -1))
        assert lead.max() <= max(ahead, max(tiles_per_layer)) + RUN
    return runs


BERT = layer_tiles(workloads.bert_base_topk(kind="sign"))
RAGGED = [23, 1, 2, 1, 37, 1]


@pytest.mark.parametrize("W", [1, 3, 8])
@pytest.mark.parametrize("ahead", [1, 64, 300, 768, 100000])
def test_bert_base_shaped_order(W, ahead):
    check(BERT, W, ahead)


@pytest.mark.parametrize("W", [1, 2, 5])
@pytest.mark.parametrize("ahead", [1, 2, 63, 64, 65, 768])
def test_ragged_order(W, ahead):
    check(RAGGED, W, ahead)


def test_one_tile_and_large_look_ahead():
    runs = check([1], 1, 768)
    assert runs == [(0, 0, 0, 0), (1, 0, 1, 0), (2, 1, -1, 0)]


def test_layer_longer_than_the_look_ahead_is_updated_backwards():
    """BERT-base's embedding (2862 tiles) at the default look-ahead of 768:
    its update starts at its last tile, the one normed most recently."""
    assert BERT[0] == 2862
    kind, tile = expand(check(BERT, 2, 768))
    upd = tile[kind == 1]
    assert upd[0] == BERT[0] - 1 and upd[BERT[0] - 1] == 0
    second = sum(BERT)                                  # worker 1's embedding
    k = np.flatnonzero(upd == second + BERT[0] - 1)[0]
    assert np.array_equal(upd[k:k + BERT[0]], np.arange(second + BERT[0] - 1, second - 1, -1))


def test_look_ahead_interleaves_norm_and_update_runs():
    """With many small layers and a short look-ahead the order alternates
    (the point of the schedule): updates start long before the last norm."""
    runs = check([4] * 200, 2, 64)
    kinds = [k for _, _, k, _ in runs[:-1]]
    first_update = kinds.index(1)
    assert first_update < 10 and 0 in kinds[first_update:]


def test_wait_test_order_puts_every_update_first():
    T = sum(RAGGED) * 2
    runs = gce().sign_schedule(RAGGED, 2, -1)
    assert all(r[3] == 0 for r in runs)
    kind, tile = expand(runs)
    assert np.all(kind[:T] == 1) and np.all(kind[T:] == 0)
    assert np.array_equal(tile[:T], np.arange(T)) and np.array_equal(tile[T:], np.arange(T))


def test_bad_arguments_are_refused():
    g = gce()
    for args in [([], 1, 64), ([3, 0], 1, 64), ([3], 0, 64), ([3], 1, -2), ([3], 1, (1 << 20) + 1)]:
        with pytest.raises(g.GceError):
            g.sign_schedule(*args)
