"""Seeded synthetic inputs for the ternary linear layer.

This module only draws random inputs: ternary weight matrices, per-tensor
weight scales and fp32 activations, with the shapes and value distributions of
the workloads below.  It holds none of the layer's arithmetic (no quantising,
packing or multiplying), so the CUDA path and the CPU oracle can both be fed
from it without sharing any of the method's code.

Workloads (layer shapes of a 1.5B-class decoder: 28 layers of q, k, v, o,
gate, up, down, from "VibeVoice-ASR-BitNet Technical Report", §2.1/Figure 2
(28-layer decoder) and §2.2.2 (ternary weights, per-token INT8 activations)):

* single layer 1536 -> 1536, M = 1, weights P(-1,0,+1) = (0.25, 0.5, 0.25),
  activations N(0,1);
* one decoder layer's seven linears at M = 1, P = (0.3, 0.4, 0.3),
  activations N(0,1) with 1 % of entries multiplied by 20;
* the 28-layer stack of those seven linears at M in {1, 2, 4, 8};
* prefill, M = 2048 over the seven shapes, row m of the activations scaled by
  10**u_m with u_m ~ U(-2, 1);
* an edge sweep over M, K, N with special rows.

Every draw is made from ``numpy.random.default_rng(seed)`` with the seed
given by ``seed_for``; weight scales are U(0.01, 0.1) as fp32.
"""
from __future__ import annotations

import numpy as np

# (name, N out, K in) of one decoder layer's linears
LAYER_SHAPES = (
    ("q", 1536, 1536),
    ("k", 256, 1536),
    ("v", 256, 1536),
    ("o", 1536, 1536),
    ("gate", 8960, 1536),
    ("up", 8960, 1536),
    ("down", 1536, 8960),
)
# which of the layer's four distinct activation inputs feeds each linear:
# 0 = layer input (q, k, v), 1 = attention output (o), 2 = o output
# (gate, up), 3 = up output (down)
LAYER_INPUT_OF = (0, 0, 0, 1, 2, 2, 3)
LAYER_INPUT_K = (1536, 1536, 1536, 8960)
NUM_LAYERS = 28

P_SINGLE = (0.25, 0.5, 0.25)
P_LAYER = (0.3, 0.4, 0.3)

EDGE_M = (1, 2, 3, 4, 5, 7, 8, 13, 64)
EDGE_K = (128, 1536, 8960, 9024)
EDGE_N = (256, 1536, 8960)

_BASE_SEED = 0xB17E7


def seed_for(config: int, index: int = 0, layer: int = 0) -> int:
    """Seed of one draw: config number (1..5), shape index, layer index."""
    return _BASE_SEED + 1000 * config + 100000 * layer + index


def ternary(rng: np.random.Generator, n: int, k: int, p=P_LAYER) -> np.ndarray:
    """int8 [n, k], i.i.d. -1/0/+1 with probabilities p (thresholds on uint32)."""
    t1 = np.uint32(round(p[0] * 2**32))
    t2 = np.uint32(min(round((p[0] + p[1]) * 2**32), 2**32 - 1))
    r = rng.integers(0, 2**32, size=(n, k), dtype=np.uint32)
    w = (r >= t1).astype(np.int8)
    w += (r >= t2).astype(np.int8)
    w -= 1
    return w


def weight_scale(rng: np.random.Generator) -> float:
    return float(np.float32(rng.uniform(0.01, 0.1)))


def normal(rng: np.random.Generator, m: int, k: int) -> np.ndarray:
    return rng.standard_normal((m, k), dtype=np.float32)


def normal_outliers(rng: np.random.Generator, m: int, k: int,
                    frac: float = 0.01, mult: float = 20.0) -> np.ndarray:
    x = normal(rng, m, k)
    hit = rng.random((m, k)) < frac
    x[hit] *= np.float32(mult)
    return x


def normal_row_spread(rng: np.random.Generator, m: int, k: int,
                      lo: float = -2.0, hi: float = 1.0) -> np.ndarray:
    x = normal(rng, m, k)
    u = rng.uniform(lo, hi, size=(m, 1))
    return (x * (10.0 ** u)).astype(np.float32)


# ---------------------------------------------------------------- workloads

def single_layer(seed: int | None = None):
    """Single 1536 -> 1536 layer at M = 1: (w int8 [N,K], s_w, x fp32 [1,K])."""
    rng = np.random.default_rng(seed_for(1) if seed is None else seed)
    w = ternary(rng, 1536, 1536, P_SINGLE)
    s = weight_scale(rng)
    x = normal(rng, 1, 1536)
    return w, s, x


def layer_weights(layer: int, config: int = 3):
    """The seven (w, s_w) of decoder layer ``layer`` (independently seeded)."""
    out = []
    for i, (_, n, k) in enumerate(LAYER_SHAPES):
        rng = np.random.default_rng(seed_for(config, i, layer))
        out.append((ternary(rng, n, k, P_LAYER), weight_scale(rng)))
    return out


def layer_inputs(layer: int, m: int, config: int = 3):
    """The four distinct fp32 activation inputs of a layer at M = m."""
    out = []
    for j, k in enumerate(LAYER_INPUT_K):
        rng = np.random.default_rng(seed_for(config, 50 + j, layer) + 7 * m)
        out.append(normal_outliers(rng, m, k))
    return out


def prefill_inputs(m: int = 2048):
    """Prefill activations per distinct input width K (1536 and 8960)."""
    out = {}
    for j, k in enumerate((1536, 8960)):
        rng = np.random.default_rng(seed_for(4, 60 + j))
        out[k] = normal_row_spread(rng, m, k)
    return out


def edge_case(m: int, k: int, n: int, seed: int):
    """Random edge-sweep case plus special rows planted in weights/activations.

    Weight rows 0..3 are all-zero, all +1, all -1 and alternating +1/-1 (when
    n allows); activation rows: row 0 random, row 1 constant 0.75 (when m > 1),
    row 2 all zeros (m > 2), row 3 a single huge outlier (m > 3).
    """
    rng = np.random.default_rng(seed)
    w = ternary(rng, n, k, P_LAYER)
    specials = [0, 1, -1]
    for r, v in enumerate(specials[: n]):
        w[r, :] = v
    if n > 3:
        w[3, :] = np.where(np.arange(k) % 2 == 0, 1, -1).astype(np.int8)
    x = normal_outliers(rng, m, k)
    if m > 1:
        x[1, :] = np.float32(0.75)
    if m > 2:
        x[2, :] = 0.0
    if m > 3:
        x[3, :] = normal(rng, 1, k) * np.float32(1e-3)
        x[3, k // 2] = np.float32(1e4)
    return w, weight_scale(rng), x
