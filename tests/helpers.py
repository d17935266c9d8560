"""Shared test plumbing: GPU availability, library build, tensor<->numpy moves.

Holds no compression arithmetic: the CUDA path is reached through the
binding, the expected values through the oracle.
"""
import numpy as np
import pytest

try:
    import torch
    HAS_GPU = torch.cuda.is_available()
except Exception:  # pragma: no cover
    torch = None
    HAS_GPU = False


def need_gpu():
    if not HAS_GPU:
        pytest.skip("needs a CUDA device")


def gce():
    """The binding, with libgce.so built in-tree (fails loudly otherwise)."""
    from gradient_compression_error_b200 import build
    build.build()
    import gradient_compression_error_b200 as g
    return g


def host(t):
    return t.detach().cpu().numpy()


def bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


def units_of(layers, W):
    return [(w, l) for w in range(W) for l in range(len(layers))]


def payload_slice(table, w, l, k):
    o = w * table.vals_per_worker + table.info[l]["val_offset"]
    return slice(o, o + k)


def layer_slice(table, l):
    o = table.info[l]["offset"]
    return slice(o, o + table.info[l]["n"])
