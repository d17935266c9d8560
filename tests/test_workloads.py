"""The seeded synthetic workloads (gradient_compression_error_b200.workloads).

The shapes stand in for the pages' models, so their sizes are pinned to what
the architectures give, computed here from each architecture's own definition
rather than from the module's shape lists.  BERT-base's count is also its
published parameter count.  The generator is checked for determinism, per-worker
seeds and exact per-layer scaling.  CPU only.
"""
import numpy as np
import torch

from gradient_compression_error_b200 import workloads as wl


def test_bert_base_is_the_published_parameter_count():
    layers = wl.bert_base_topk()
    hidden, inter, vocab, pos, types, n_layers = 768, 3072, 30522, 512, 2, 12
    emb = (vocab + pos + types) * hidden + 2 * hidden                 # + embedding LayerNorm
    per_layer = (4 * (hidden * hidden + hidden)                         # Q, K, V, attention out
                 + 2 * hidden                                           # attention LayerNorm
                 + hidden * inter + inter + inter * hidden + hidden     # feed-forward
                 + 2 * hidden)                                          # output LayerNorm
    pooler = hidden * hidden + hidden
    assert wl.total_elements(layers) == emb + n_layers * per_layer + pooler == 109_482_240
    assert len(layers) == 90
    # top-k at 1 % of every tensor: floor(n / 100), at least one slot
    for l in layers:
        assert l["cap"] == max(1, (l["rows"] * l["cols"] * 10000) // 1000000)


def test_vgg19_e_on_cifar100():
    cfg = [64, 64, "M", 128, 128, "M", 256, 256, 256, 256, "M",
           512, 512, 512, 512, "M", 512, 512, 512, 512, "M"]
    conv, bn, cin = 0, 0, 3
    for c in cfg:
        if c == "M":
            continue
        conv += c * cin * 9
        bn += 2 * c                                  # gamma and beta
        cin = c
    fc = 100 * 512 + 100
    layers = wl.vgg19("powersgd", 4)
    assert wl.total_elements(layers) == conv + bn + fc == 20_081_188
    assert sum(1 for l in layers if l["kind"] == "powersgd") == 17      # 16 convs + the FC weight


def test_resnet18_shaped_convolutions():
    layers = wl.resnet18_powersgd(2)
    convs = [l for l in layers if l["kind"] == "powersgd"]
    # four 3x3 convolutions per stage, weights out x (in * 3 * 3), in = out
    assert [(l["rows"], l["cols"]) for l in convs] == \
        [(c, c * 9) for c in (64, 128, 256, 512) for _ in range(4)]
    assert wl.total_elements(layers) == 12_541_440
    for l in convs:
        assert abs(l["sigma"] - 1.0 / np.sqrt(l["cols"])) < 1e-12


def test_sweep_shapes():
    assert wl.total_elements(wl.sweep(30)) == 1 << 30
    ps = wl.sweep(25, "powersgd")[0]
    assert (ps["rows"], ps["cols"]) == (1 << 12, 1 << 13)
    assert wl.sweep(20, ppm=1000)[0]["cap"] == (1 << 20) // 1000


def test_seeds_are_distinct_per_worker_step_and_workload():
    seeds = {wl.seed_for(c, w, s) for c in range(6) for w in range(64) for s in range(200)}
    assert len(seeds) == 6 * 64 * 200


def test_gradients_are_seeded_and_scaled_per_layer():
    layers = [dict(rows=100, cols=3, kind="topk", cap=3, sigma=0.25),
              dict(rows=50, cols=1, kind="dense", cap=0, sigma=1.0),
              dict(rows=7, cols=7, kind="topk", cap=2, sigma=3.0)]
    a = wl.gradients(layers, 3, 7, 2, device="cpu")
    b = wl.gradients(layers, 3, 7, 2, device="cpu")
    assert torch.equal(a, b)                                   # same seed, same bits
    assert not torch.equal(a[0], a[1])                         # workers draw apart
    assert not torch.equal(a, wl.gradients(layers, 3, 7, 3, device="cpu"))   # steps too
    unit = [dict(l, sigma=1.0) for l in layers]
    raw = wl.gradients(unit, 3, 7, 2, device="cpu")
    off = 0
    for l in layers:
        n = l["rows"] * l["cols"]
        expect = (raw[:, off:off + n] * np.float32(l["sigma"])).numpy()   # one fp32 multiply
        assert np.array_equal(a[:, off:off + n].numpy().view(np.uint32), expect.view(np.uint32))
        off += n


def test_vgg19_gradient_scale_schedule():
    assert [wl.vgg19_scale(t) for t in (0, 59, 60, 139, 140, 199)] == [1.0, 1.0, 0.1, 0.1,
                                                                         0.01, 0.01]


def test_table_layers_keep_only_the_table_keys():
    out = wl.table_layers([dict(rows=2, cols=3, kind="topk", cap=1, sigma=5.0)])
    assert out == [dict(rows=2, cols=3, kind="topk", cap=1)]
