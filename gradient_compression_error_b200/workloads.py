"""Seeded synthetic workloads: layer tables and gradient generators.

This module holds shapes, seeds and the gradient distributions of the
workloads only -- none of the compression arithmetic.  Both the CUDA path
and the CPU oracle take their inputs from here: gradients are drawn on the
device with torch and copied to the host for the oracle, so the two sides
share data, never code.

Workloads (the pages' models, with standard architecture shapes; the pages'
datasets are not used -- synthetic gradients stand in for them):
  memsgd_vector     one 1-D vector of 2^20 elements, top-k with k = 1024
  resnet18_powersgd ResNet-18 conv weights reshaped out x in*kh*kw
                    (64x576, 128x1152, 256x2304, 512x4608, 4 of each) plus
                    16 uncompressed BatchNorm vectors (gamma||beta)
  vgg19             VGG-19 (configuration E) on 32x32 inputs with a 100-way
                    classifier: 16 conv weights + the FC weight, 16 BatchNorm
                    vectors and the FC bias
  bert_base_topk    BERT-base: embeddings (30522x768, 512x768, 2x768), 12
                    encoder layers (4x 768x768, 3072x768, 768x3072, and the
                    layer's 9984 bias / LayerNorm values as one vector), the
                    768x768 pooler and its bias; every tensor is top-k at 1 %
  sweep             one flat buffer of 2^e elements (top-k / rand-k), or a
                    2^floor(e/2) x 2^ceil(e/2) matrix (PowerSGD)
"""
import math

ETA = 0.05


def _ppm_k(n, ppm):
    # number of payload slots for a fraction given in parts per million
    return max(1, (n * ppm) // 1000000)


def memsgd_vector(n=1 << 20, k=1024, kind="topk"):
    return [dict(rows=n, cols=1, kind=kind, cap=k, sigma=1.0)]


RESNET18_CONVS = [(64, 576)] * 4 + [(128, 1152)] * 4 + [(256, 2304)] * 4 + [(512, 4608)] * 4


def resnet18_powersgd(rank=2):
    layers = []
    for rows, cols in RESNET18_CONVS:
        layers.append(dict(rows=rows, cols=cols, kind="powersgd", cap=rank,
                           sigma=1.0 / math.sqrt(cols)))
        layers.append(dict(rows=2 * rows, cols=1, kind="dense", cap=0, sigma=1.0))
    return layers


VGG19_CONVS = [(64, 27), (64, 576), (128, 576), (128, 1152), (256, 1152), (256, 2304),
               (256, 2304), (256, 2304), (512, 2304), (512, 4608), (512, 4608), (512, 4608),
               (512, 4608), (512, 4608), (512, 4608), (512, 4608)]
VGG19_FC = (100, 512)


def vgg19(kind="powersgd", cap=4):
    """kind 'powersgd' (cap = r_max) or 'topk' (cap = k slots in ppm of each layer)."""
    layers = []

    def comp(rows, cols):
        n = rows * cols
        c = cap if kind == "powersgd" else _ppm_k(n, cap)
        return dict(rows=rows, cols=cols, kind=kind, cap=c, sigma=1.0 / math.sqrt(cols))

    for rows, cols in VGG19_CONVS:
        layers.append(comp(rows, cols))
        layers.append(dict(rows=2 * rows, cols=1, kind="dense", cap=0, sigma=1.0))
    layers.append(comp(*VGG19_FC))
    layers.append(dict(rows=VGG19_FC[0], cols=1, kind="dense", cap=0, sigma=1.0))
    return layers


def vgg19_scale(t):
    """Gradient scale of the VGG-19 run: 1.0, x0.1 at step 60, x0.1 again at 140."""
    return 1.0 if t < 60 else (0.1 if t < 140 else 0.01)


def bert_base_topk(ppm=10000, kind="topk"):
    shapes = [(30522, 768), (512, 768), (2, 768), (1536, 1)]
    for _ in range(12):
        shapes += [(768, 768)] * 4 + [(3072, 768), (768, 3072), (9984, 1)]
    shapes += [(768, 768), (768, 1)]
    return [dict(rows=r, cols=c, kind=kind, cap=_ppm_k(r * c, ppm), sigma=1.0) for r, c in shapes]


def sweep(e, method="topk", ppm=10000, rank=2):
    n = 1 << e
    if method == "powersgd":
        return [dict(rows=1 << (e // 2), cols=1 << ((e + 1) // 2), kind="powersgd", cap=rank,
                     sigma=1.0)]
    return [dict(rows=n, cols=1, kind=method, cap=0 if method == "sign" else _ppm_k(n, ppm),
                 sigma=1.0)]


def total_elements(layers):
    return sum(l["rows"] * l["cols"] for l in layers)


def seed_for(config, worker, step):
    """Seed of the gradient of (workload id, worker, step)."""
    return 0x5EED0000 + (config << 20) + (worker << 12) + step


def gradients(layers, W, config, step, device="cuda", scale=1.0, out=None):
    """[W, N] float32 gradients: N(0, 1) per worker from its own seed, each
    layer multiplied by its sigma (and by `scale`) in fp32."""
    import torch
    N = total_elements(layers)
    if out is None:
        out = torch.empty((W, N), dtype=torch.float32, device=device)
    for w in range(W):
        g = torch.Generator(device=device)
        g.manual_seed(seed_for(config, w, step))
        torch.randn(N, generator=g, device=device, dtype=torch.float32, out=out[w])
        off = 0
        for l in layers:
            n = l["rows"] * l["cols"]
            s = l.get("sigma", 1.0) * scale
            if s != 1.0:
                out[w, off:off + n].mul_(s)
            off += n
    return out


def table_layers(layers):
    """The layer dicts without the generator-only keys."""
    return [dict(rows=l["rows"], cols=l["cols"], kind=l["kind"], cap=l["cap"]) for l in layers]
