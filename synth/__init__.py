"""Seeded synthetic inputs for the scaled pairwise-rotated INT4 linear layer.

This module only draws random numbers and rounds them to the dtypes the layer
stores; it holds none of the method's arithmetic (no rotation, no packing, no
dequantisation).  Both the float64 oracle tests and the CUDA path take their
inputs from here, so the two sides see bit-identical data.

Tensor shapes follow the stored-tensor table of the GPTQModel wiki page
"ParoQuant" (section "Checkpoint and inference implementation / Stored
tensors"): with I = in_features = K, O = out_features = N and group size G,

    pairs           int16   [krot, K]      group-local channel indices
    theta           float32 [krot, K // 2] one angle per pair
    channel_scales  float32 [K]            runtime multiplier D^-1
    scales          float16 [K // G, N]    group dequantisation scales
    bias            float16 [N] or None

plus, as the packer's input (before AWQ packing):

    codes           uint8   [N, K]         4-bit weight codes 0..15 (out x in)
    zero_codes      uint8   [N, K // G]    4-bit zero points 0..15

Value distributions (the workload recipe):
  * x: N(0, 1) with a set of outlier channels multiplied by 20, then fp16.
  * channel_scales: exp(U(ln 0.5, ln 2)) -> fp32.
  * pairs: per stage and per group a random perfect matching, i.e. a random
    permutation of the G local channels whose consecutive entries (2p, 2p+1)
    form pair p (same page, sections "Pairwise Givens rotations" and "Stored
    tensors": pair indices are local to each group).
  * theta: U(-pi, pi) -> fp32 for active pairs, exactly 0 for dummy pairs
    (same page: "unused channels are filled with dummy pairs whose angles stay
    zero").
  * weight-side quantiser inputs (``make_float_weight``): W N(0, 0.02^2) with
    two rows x 8 -> fp16; quantiser scales U[0.006, 0.012] -> fp16.
  * codes: U{0..15}; zero codes all 8 (the unsigned export of the symmetric
    4-bit quantiser uses zero point 8, same page, "Straight-through
    estimation"); scales U[0.005, 0.02] -> fp16; bias 0 or N(0, 0.01) -> fp16.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

GROUP_SIZE = 128
KROT = 8


@dataclass
class Layer:
    """One packed rotated-W4 linear layer (pre-packing form)."""
    name: str
    K: int
    N: int
    group_size: int
    krot: int
    pairs: np.ndarray            # int16 [krot, K]
    theta: np.ndarray            # float32 [krot, K//2]
    channel_scales: np.ndarray   # float32 [K]
    codes: np.ndarray            # uint8 [N, K]
    zero_codes: np.ndarray       # uint8 [N, K//G]
    scales: np.ndarray           # float16 [K//G, N]
    bias: Optional[np.ndarray]   # float16 [N] or None
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    seed: int = 0


def make_layer(name: str, K: int, N: int, seed: int, *, group_size: int = GROUP_SIZE,
               krot: int = KROT, active_pairs: Optional[int] = None,
               bias_std: float = 0.0, n_outliers: int = 4,
               zero_point: Optional[int] = 8) -> Layer:
    """Draw one layer.  ``active_pairs`` is the number of pairs per stage and
    per group that get a random angle (default: all G/2); the rest keep 0.
    ``zero_point=None`` draws zero codes U{0..15} instead of the constant 8."""
    G = K if group_size == -1 else group_size
    assert G % 2 == 0 and K % G == 0
    half = G // 2
    if active_pairs is None:
        active_pairs = half
    rng = np.random.default_rng(seed)

    pairs = np.empty((krot, K), dtype=np.int16)
    theta = np.zeros((krot, K // 2), dtype=np.float32)
    for s in range(krot):
        for g in range(K // G):
            pairs[s, g * G:(g + 1) * G] = rng.permutation(G).astype(np.int16)
            act = rng.choice(half, size=active_pairs, replace=False)
            ang = rng.uniform(-np.pi, np.pi, size=active_pairs)
            theta[s, g * half + act] = ang.astype(np.float32)

    channel_scales = np.exp(rng.uniform(np.log(0.5), np.log(2.0), size=K)).astype(np.float32)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    if zero_point is None:
        zero_codes = rng.integers(0, 16, size=(N, K // G), dtype=np.uint8)
    else:
        zero_codes = np.full((N, K // G), zero_point, dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, size=(K // G, N)).astype(np.float16)
    bias = None
    if bias_std > 0:
        bias = (rng.standard_normal(N) * bias_std).astype(np.float16)
    outliers = np.sort(rng.choice(K, size=min(n_outliers, K), replace=False))
    return Layer(name, K, N, G, krot, pairs, theta, channel_scales, codes, zero_codes,
                 scales, bias, outliers, seed)


def make_activations(layer: Layer, M: int, seed: Optional[int] = None) -> np.ndarray:
    """x [M, K] fp16: N(0,1) with the layer's outlier channels scaled by 20."""
    rng = np.random.default_rng((layer.seed if seed is None else seed, 7, M))
    x = rng.standard_normal((M, layer.K))
    if layer.outlier_channels.size:
        x[:, layer.outlier_channels] *= 20.0
    return x.astype(np.float16)


def make_float_weight(layer: Layer, seed: Optional[int] = None, std: float = 0.02,
                      outlier_rows: int = 2):
    """Float inputs of the weight-side quantiser for ``layer``'s shape:

    * W [N, K] fp16 (out x in): N(0, std^2), with ``outlier_rows`` whole rows
      x 8 so that some groups clamp at the code range;
    * quantiser scales [K//G, N] fp16: U[0.3, 0.6] * std, about a third to a
      sixth of the largest |W_r| of a group of 128, so that a few per cent of
      the codes sit at -8 or 7.

    The rotation tables and channel scales are the layer's own."""
    rng = np.random.default_rng((layer.seed if seed is None else seed, 11))
    W = rng.standard_normal((layer.N, layer.K)) * std
    if outlier_rows:
        rows = rng.choice(layer.N, size=min(outlier_rows, layer.N), replace=False)
        W[rows] *= 8.0
    G = layer.group_size
    qscales = rng.uniform(0.3 * std, 0.6 * std, size=(layer.K // G, layer.N))
    return W.astype(np.float16), qscales.astype(np.float16)


def one_percent(K: int) -> int:
    return int(round(0.01 * K))


# --------------------------------------------------------------------------
# The five workloads.  Shapes are Llama-3-8B linears (hidden 4096,
# intermediate 14336, 8 KV heads of 128).
# --------------------------------------------------------------------------

LLAMA3_8B_LINEARS = [
    # (name, K=in_features, N=out_features)
    ("q_proj", 4096, 4096),
    ("k_proj", 4096, 1024),
    ("v_proj", 4096, 1024),
    ("o_proj", 4096, 4096),
    ("gate_proj", 4096, 14336),
    ("up_proj", 4096, 14336),
    ("down_proj", 14336, 4096),
]


def config_layers(cfg: int) -> list[Layer]:
    """Layers of workload ``cfg`` (0..4), seeds 1000*cfg + layer index (cfg 0: 0)."""
    if cfg == 0:
        return [make_layer("tiny", 256, 512, 0, n_outliers=4)]
    if cfg == 1:
        return [make_layer("q_proj", 4096, 4096, 1000, active_pairs=round(0.1 * 64),
                           n_outliers=4)]
    if cfg == 2:
        shapes = [("gate_proj", 4096, 14336), ("up_proj", 4096, 14336),
                  ("down_proj", 14336, 4096)]
        return [make_layer(n, K, N, 2000 + i, n_outliers=one_percent(K))
                for i, (n, K, N) in enumerate(shapes)]
    if cfg == 3:
        return [make_layer("gate_proj", 4096, 14336, 3000, bias_std=0.01,
                           n_outliers=one_percent(4096))]
    if cfg == 4:
        return [make_layer(n, K, N, 4000 + i, n_outliers=one_percent(K))
                for i, (n, K, N) in enumerate(LLAMA3_8B_LINEARS)]
    raise ValueError(cfg)


CONFIG_M = {0: [4], 1: [1, 4, 16], 2: [1, 8], 3: [2048, 8192], 4: [1, 4096]}


def config_layer_shapes(cfg: int) -> list[tuple[str, int, int]]:
    """(name, K, N) of each layer of ``cfg`` without drawing any data."""
    return {
        0: [("tiny", 256, 512)],
        1: [("q_proj", 4096, 4096)],
        2: [("gate_proj", 4096, 14336), ("up_proj", 4096, 14336), ("down_proj", 14336, 4096)],
        3: [("gate_proj", 4096, 14336)],
        4: list(LLAMA3_8B_LINEARS),
    }[cfg]
