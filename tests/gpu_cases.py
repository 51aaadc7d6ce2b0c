"""Shared helpers for the GPU parity tests: seeded layers moved to the
device, and the comparison rules.

Bar: indices, sets, lists and every fp32 value of the router and the
re-selection are bit-exact; the layer output y is within max-abs 2e-2 and
relative-L2 1e-2 of the fp64 oracle (bf16 weights, fp32 accumulation)."""
import functools

import numpy as np
import torch

import moe_synth as ms

MAX_ABS = 2e-2
REL_L2 = 1e-2

# extra shapes for edges: minimum sizes with E == k, maximum E and k,
# ragged d / d_ff (not multiples of the 256 / 128 stage widths)
EDGE_SHAPES = {
    "min": ms.LayerShape("min", d=64, E=8, k=8, F=64, bias="normal", bias_param=0.5),
    "maxek": ms.LayerShape("maxek", d=256, E=256, k=16, F=128, bias="zipf", bias_param=1.0),
    "ragged": ms.LayerShape("ragged", d=320, E=24, k=6, F=192, bias="normal", bias_param=0.8),
}


def shape(name):
    return ms.SHAPES[name] if name in ms.SHAPES else EDGE_SHAPES[name]


@functools.lru_cache(maxsize=4)
def host_layer(name, seed):
    return ms.make_weights(shape(name), seed)


@functools.lru_cache(maxsize=2)
def device_layer(name, seed):
    L = host_layer(name, seed)
    dev = {
        "Wg": torch.from_numpy(L["Wg"]).cuda(),
        "bias": torch.from_numpy(L["bias"]).cuda(),
        "Wgate": torch.from_numpy(L["Wgate"].view(np.int16)).cuda(),
        "Wup": torch.from_numpy(L["Wup"].view(np.int16)).cuda(),
        "Wdown": torch.from_numpy(L["Wdown"].view(np.int16)).cuda(),
    }
    torch.cuda.synchronize()
    return dev


def bits(t):
    a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return np.ascontiguousarray(a).view(np.uint32)


def assert_close_y(y_gpu, y_ref, what=""):
    y = np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == r.shape
    assert np.all(np.isfinite(y)), what
    err = np.abs(y - r)
    rel = np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-30)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return float(err.max()), float(rel)
