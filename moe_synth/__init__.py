"""Seeded synthetic MoE-layer inputs shared by the oracle tests, the GPU
parity tests and the benchmark.

This module holds no arithmetic of the method itself: it only draws random
inputs and encodes them.  Every array it returns is plain NumPy on the host.

Shapes follow the layers named by the source pages: a tiny layer for exact
checks, a 64-expert layer (the "all 64 experts" saturation example in
"Lynx: Enabling Efficient MoE Inference through Dynamic Batch-Aware Expert
Selection", section 1), and layers shaped like Qwen3-30B-A3B and
Qwen3-235B-A22B (the two models of "Opportunistic Expert Activation:
Batch-Aware Expert Routing for Faster Decode Without Retraining",
abstract).  The pages print no weights, so the values are synthetic:

* router weight ``Wg[E][d]`` fp32, N(0, 0.02);
* router bias ``bias[E]`` fp32, either N(0, sigma) or a Zipf skew
  ``-s * ln(rank)`` over a seeded permutation of the experts, centred to
  mean 0 (it stands in for the training-induced activation skew that the
  Lynx page describes in section 2);
* expert weights ``Wgate[E][F][d]``, ``Wup[E][F][d]``, ``Wdown[E][d][F]``
  N(0, 0.02), stored as bf16 bit patterns (round to nearest even);
* tokens ``x[B][d]`` fp32, N(0, 1), or, for a speculative-decode batch,
  ``x = mu_request + 0.3 * N(0, 1)`` with ``mu_request ~ N(0, 1)``.

Weights and tokens come from two independent child streams of
``numpy.random.SeedSequence(seed)``, so the same layer is reused across
batch sizes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

__all__ = [
    "LayerShape", "SHAPES", "bf16_bits", "make_weights", "make_tokens",
    "expert_bytes",
]


@dataclass(frozen=True)
class LayerShape:
    name: str
    d: int          # hidden size
    E: int          # number of experts
    k: int          # experts per token
    F: int          # expert intermediate size (d_ff)
    bias: str       # "normal" or "zipf"
    bias_param: float  # sigma for "normal", exponent s for "zipf"


SHAPES = {
    "tiny": LayerShape("tiny", d=256, E=16, k=4, F=128, bias="normal", bias_param=0.5),
    "e64": LayerShape("e64", d=2048, E=64, k=8, F=1024, bias="zipf", bias_param=1.1),
    "q30b": LayerShape("q30b", d=2048, E=128, k=8, F=768, bias="zipf", bias_param=1.0),
    "q235b": LayerShape("q235b", d=4096, E=128, k=8, F=1536, bias="zipf", bias_param=1.0),
}


def expert_bytes(shape: LayerShape) -> int:
    """Bytes of one expert's bf16 gate, up and down matrices."""
    return 3 * shape.d * shape.F * 2


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even.
    Inputs are finite normal samples, so NaN handling is not needed."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    w_ss, x_ss = ss.spawn(2)
    return w_ss, x_ss


def make_weights(shape: LayerShape, seed: int, experts: bool = True) -> dict:
    """Draw one layer.  Draw order: Wg, bias (or the Zipf permutation),
    then per expert e: Wgate[e], Wup[e], Wdown[e].

    With ``experts=False`` only the router arrays are returned (the expert
    matrices are not drawn), which is enough for routing-only tests."""
    w_ss, _ = _streams(seed)
    rng = np.random.default_rng(w_ss)
    d, E, F = shape.d, shape.E, shape.F
    Wg = (rng.standard_normal((E, d), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    if shape.bias == "normal":
        bias = (rng.standard_normal(E, dtype=np.float32) * np.float32(shape.bias_param)).astype(np.float32)
    elif shape.bias == "zipf":
        perm = rng.permutation(E)
        ranks = perm.astype(np.float64) + 1.0
        b = -shape.bias_param * np.log(ranks)
        bias = (b - b.mean()).astype(np.float32)
    else:
        raise ValueError(shape.bias)
    out = {"Wg": np.ascontiguousarray(Wg), "bias": np.ascontiguousarray(bias)}
    if not experts:
        return out
    Wgate = np.empty((E, F, d), dtype=np.uint16)
    Wup = np.empty((E, F, d), dtype=np.uint16)
    Wdown = np.empty((E, d, F), dtype=np.uint16)
    s = np.float32(0.02)
    for e in range(E):
        Wgate[e] = bf16_bits(rng.standard_normal((F, d), dtype=np.float32) * s)
        Wup[e] = bf16_bits(rng.standard_normal((F, d), dtype=np.float32) * s)
        Wdown[e] = bf16_bits(rng.standard_normal((d, F), dtype=np.float32) * s)
    out.update(Wgate=Wgate, Wup=Wup, Wdown=Wdown)
    return out


def make_tokens(shape: LayerShape, B: int, seed: int, kind: str = "normal",
                n_requests: int = 8) -> np.ndarray:
    """Draw a decode batch ``x[B][d]`` fp32.

    ``kind="normal"``: x ~ N(0, 1).
    ``kind="spec"``: B = n_requests * drafts tokens; token b belongs to
    request b // drafts; x = mu_request + 0.3 * N(0, 1), mu ~ N(0, 1)."""
    _, x_ss = _streams(seed)
    rng = np.random.default_rng([*x_ss.generate_state(2), B])
    d = shape.d
    if kind == "normal":
        x = rng.standard_normal((B, d), dtype=np.float32)
    elif kind == "spec":
        if B % n_requests:
            raise ValueError("B must be a multiple of n_requests")
        drafts = B // n_requests
        mu = rng.standard_normal((n_requests, d), dtype=np.float32)
        noise = rng.standard_normal((B, d), dtype=np.float32)
        x = np.repeat(mu, drafts, axis=0) + np.float32(0.3) * noise
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(x.astype(np.float32))
