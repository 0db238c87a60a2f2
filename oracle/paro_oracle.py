"""Float64 CPU oracle for the scaled pairwise-rotated INT4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, links or runs this module; only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm do.
It shares no code with the CUDA path.

Every function is a direct, slow, obviously-correct restatement of the
GPTQModel wiki page "ParoQuant":

* scaling + Givens stages: sections "Pairwise Givens rotations" (pair formula,
  stage order, inverse, group-local indices, group_size=-1) and "Activation and
  weight transforms" (X_r = X D^-1 R, saved channel_scales are D^-1);
* stored tensor shapes: section "Stored tensors";
* group-wise dequantisation and the transformed-domain linear
  Y = X_r Q(W_r)^T + b: sections "Triton plans and tuning" (unpack INT4,
  subtract zero points, multiply by group scales, accumulate) and "Activation
  and weight transforms"; the affine dequantiser x_hat = scale * (q - zero) is
  the one on the GPTQModel wiki page "GPTQ" (quantizer formulas).

Readings taken where the pages are silent (each one is listed in the design
notes and pinned by a test where something can pin it):

* pairs[s, g*G + 2p] and pairs[s, g*G + 2p + 1] are the local channels (i, j)
  of pair p of stage s in group g; theta[s, g*G/2 + p] is its angle; the
  channel at entry 2p plays the role of ``a`` in the pair formula.
* AWQ nibble order inside an int32 word: nibble t (bits 4t..4t+3) of word w
  holds output column 8w + AWQ_ORDER[t].  The pages say only "AWQ-layout";
  this order is the public AWQ convention.  Its agreement with real
  checkpoints is parity unpinned (no checkpoint is available).
* Dequantisation is (q - z) * s with q, z unpacked codes 0..15.
* theta and channel_scales are float32 at the boundary and are widened exactly.

Weight side (the step before packing): W_r = W D R with D = 1 / channel_scales
(section "Activation and weight transforms": the saved channel_scales are
D^-1), the rows of W (out x in) taking the activations' stages; then the
four-bit symmetric quantiser of section "Activation and weight transforms"
(signed codes -8..7 exported unsigned with zero point 8, quantiser scales
bounded to [1e-5, 1e5]).  The pages give the code range and the bounds but
not the rounding of the quotient: round to nearest with ties to even is the
reading taken (the rounding the pages name for the pseudo-quantisation
kernels in section "STE acceleration kernels").  The quantiser scales are an
input (learned during calibration).
"""
from __future__ import annotations

from typing import Optional

import numpy as np

# nibble t of a packed word holds column 8*w + AWQ_ORDER[t]
AWQ_ORDER = (0, 2, 4, 6, 1, 3, 5, 7)

# four-bit symmetric quantiser: signed levels, exported zero point, scale bounds
SYM_QMIN, SYM_QMAX = -8, 7
SYM_ZERO_CODE = 8
QSCALE_MIN, QSCALE_MAX = 1e-5, 1e5


def normalize_group_size(group_size: int, K: int) -> int:
    """group_size=-1 means the whole input width ("Pairwise Givens rotations")."""
    G = K if group_size == -1 else int(group_size)
    if G <= 0 or G % 2 != 0 or K % G != 0:
        raise ValueError(f"group size {group_size} invalid for K={K}")
    return G


def _stage_pair_indices(pairs_s: np.ndarray, G: int):
    """Global channel indices (i, j) of every pair of one stage, in pair order."""
    K = pairs_s.shape[0]
    local = pairs_s.astype(np.int64)
    group_base = (np.arange(K // 2) // (G // 2)) * G
    i = local[0::2] + group_base
    j = local[1::2] + group_base
    return i, j


def rotate(x: np.ndarray, channel_scales: Optional[np.ndarray], pairs: Optional[np.ndarray],
           theta: Optional[np.ndarray], group_size: int, krot: Optional[int] = None) -> np.ndarray:
    """X_r = (x * channel_scales) followed by krot Givens stages, in float64.

    x: [M, K] (any float dtype; widened exactly).  channel_scales: [K] or None
    (= all ones).  pairs: [krot, K] int16, theta: [krot, K//2].
    For each stage s in order and each pair (i, j) with angle t:
        a' = a cos t + b sin t,   b' = -a sin t + b cos t,   a = x_i, b = x_j.
    The pairs of one stage are disjoint, so all of them update at once.
    """
    X = np.array(x, dtype=np.float64, copy=True)
    if X.ndim != 2:
        raise ValueError("x must be 2-D [M, K]")
    K = X.shape[1]
    G = normalize_group_size(group_size, K)
    if channel_scales is not None:
        X *= np.asarray(channel_scales, dtype=np.float64).reshape(1, K)
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    for s in range(krot):
        i, j = _stage_pair_indices(pairs[s], G)
        t = np.asarray(theta[s], dtype=np.float64)
        c, sn = np.cos(t), np.sin(t)
        a = X[:, i].copy()
        b = X[:, j].copy()
        X[:, i] = a * c + b * sn
        X[:, j] = -a * sn + b * c
    return X


def inverse_rotate(xr: np.ndarray, channel_scales: Optional[np.ndarray], pairs: np.ndarray,
                   theta: np.ndarray, group_size: int) -> np.ndarray:
    """Undo ``rotate``: stages in reverse order with negated angles, then divide
    by the channel scales ("The inverse reverses stage order and negates the
    angles")."""
    X = np.array(xr, dtype=np.float64, copy=True)
    K = X.shape[1]
    G = normalize_group_size(group_size, K)
    for s in reversed(range(pairs.shape[0])):
        i, j = _stage_pair_indices(pairs[s], G)
        t = -np.asarray(theta[s], dtype=np.float64)
        c, sn = np.cos(t), np.sin(t)
        a = X[:, i].copy()
        b = X[:, j].copy()
        X[:, i] = a * c + b * sn
        X[:, j] = -a * sn + b * c
    if channel_scales is not None:
        X /= np.asarray(channel_scales, dtype=np.float64).reshape(1, K)
    return X


def awq_pack(codes: np.ndarray, zero_codes: np.ndarray, group_size: int):
    """Pack 4-bit codes into AWQ-layout int32 words.

    codes [N, K] uint8 (0..15, out x in), zero_codes [N, K//G] uint8.
    Returns qweight [K, N//8] int32 and qzeros [K//G, N//8] int32 where nibble
    t of word w in row k holds codes[8w + AWQ_ORDER[t], k].
    """
    N, K = codes.shape
    G = normalize_group_size(group_size, K)
    if N % 8 != 0:
        raise ValueError("N must be divisible by 8")
    if codes.max(initial=0) > 15 or zero_codes.max(initial=0) > 15:
        raise ValueError("codes must be 0..15")

    def pack_rows(c_nk: np.ndarray) -> np.ndarray:   # [N, R] -> [R, N//8]
        R = c_nk.shape[1]
        words = np.zeros((R, N // 8), dtype=np.uint64)
        ct = c_nk.T.astype(np.uint64)                # [R, N]
        for t in range(8):
            words |= ct[:, AWQ_ORDER[t]::8] << np.uint64(4 * t)
        return words.astype(np.uint32).view(np.int32)

    return pack_rows(codes), pack_rows(zero_codes)


def awq_unpack(qweight: np.ndarray, qzeros: np.ndarray, N: int, K: int, group_size: int):
    """Inverse of ``awq_pack``: returns codes [N, K] and zero_codes [N, K//G] (uint8)."""
    G = normalize_group_size(group_size, K)

    def unpack_rows(words: np.ndarray) -> np.ndarray:  # [R, N//8] -> [N, R]
        w = np.asarray(words).view(np.uint32).astype(np.uint64)
        R = w.shape[0]
        out = np.zeros((R, N), dtype=np.uint8)
        for t in range(8):
            out[:, AWQ_ORDER[t]::8] = ((w >> np.uint64(4 * t)) & np.uint64(0xF)).astype(np.uint8)
        return out.T.copy()

    codes = unpack_rows(qweight)
    zeros = unpack_rows(qzeros)
    assert codes.shape == (N, K) and zeros.shape == (N, K // G)
    return codes, zeros


def dequant(codes: np.ndarray, zero_codes: np.ndarray, scales: np.ndarray, group_size: int) -> np.ndarray:
    """Explicit group-wise dequantisation, float64, returned as W [K, N]:
    W[k, n] = (q[k, n] - z[k//G, n]) * s[k//G, n]."""
    N, K = codes.shape
    G = normalize_group_size(group_size, K)
    q = codes.T.astype(np.float64)                              # [K, N]
    z = np.repeat(zero_codes.T.astype(np.float64), G, axis=0)   # [K, N]
    s = np.repeat(np.asarray(scales, dtype=np.float64), G, axis=0)
    return (q - z) * s


def w4_linear(x: np.ndarray, qweight: np.ndarray, qzeros: np.ndarray, scales: np.ndarray,
              bias: Optional[np.ndarray], channel_scales: Optional[np.ndarray],
              pairs: Optional[np.ndarray], theta: Optional[np.ndarray],
              group_size: int, krot: int) -> np.ndarray:
    """Y = rotate(x * channel_scales) @ dequant(qweight, qzeros, scales) + bias, float64.

    x [M, K]; qweight [K, N//8] int32; qzeros [K//G, N//8] int32; scales [K//G, N];
    bias [N] or None.  krot == 0 skips the stages; channel_scales None skips scaling.
    """
    M, K = x.shape
    N = qweight.shape[1] * 8
    G = normalize_group_size(group_size, K)
    xr = rotate(x, channel_scales, pairs, theta, G, krot=krot)
    codes, zeros = awq_unpack(qweight, qzeros, N, K, G)
    W = dequant(codes, zeros, scales, G)
    Y = xr @ W
    if bias is not None:
        Y += np.asarray(bias, dtype=np.float64).reshape(1, N)
    return Y


def w4_linear_from_codes(x, codes, zero_codes, scales, bias, channel_scales, pairs, theta,
                         group_size, krot):
    """Same as ``w4_linear`` but starting from unpacked codes (skips the packer)."""
    K = x.shape[1]
    G = normalize_group_size(group_size, K)
    xr = rotate(x, channel_scales, pairs, theta, G, krot=krot)
    Y = xr @ dequant(codes, zero_codes, scales, G)
    if bias is not None:
        Y += np.asarray(bias, dtype=np.float64).reshape(1, -1)
    return Y


def w4_linear_columns(x, codes, zero_codes, scales, bias, channel_scales, pairs, theta,
                      group_size, krot, cols: np.ndarray) -> np.ndarray:
    """Y[:, cols] only: for checking sampled outputs of full-size layers."""
    K = x.shape[1]
    G = normalize_group_size(group_size, K)
    xr = rotate(x, channel_scales, pairs, theta, G, krot=krot)
    cols = np.asarray(cols)
    W = dequant(codes[cols], zero_codes[cols], scales[:, cols], G)   # [K, len(cols)]
    Y = xr @ W
    if bias is not None:
        Y += np.asarray(bias, dtype=np.float64)[cols].reshape(1, -1)
    return Y


def moe_linear_from_codes(x, expert_idx, codes, zero_codes, scales, bias, channel_scales, pairs, theta,
                          group_size, krot):
    """Stacked experts sharing one rotation (brain.gartu.xyz ParoQuant page,
    MLX section: the experts' weights are stacked in one tensor and their
    rotations are shared), float64.

    x [T, K]; expert_idx [T, topk] ints; codes [E, N, K] uint8 (out x in per
    expert); zero_codes [E, N, K//G]; scales [E, K//G, N]; bias [E, N] or None;
    one channel_scales / pairs / theta for every expert.  Returns y [T, topk, N]:
        X_r = rotate(x * channel_scales)                  (once, for all experts)
        y[t, j] = X_r[t] @ dequant(expert e = expert_idx[t, j]) + bias[e]
    A slot whose index lies outside 0..E-1 selects no expert: its row is 0
    (the reading taken for a routing value the pages do not define).
    """
    x = np.asarray(x)
    idx = np.asarray(expert_idx).astype(np.int64)
    T, K = x.shape
    E, N = codes.shape[0], codes.shape[1]
    topk = idx.shape[1]
    G = normalize_group_size(group_size, K)
    xr = rotate(x, channel_scales, pairs, theta, G, krot=krot)
    y = np.zeros((T, topk, N))
    for e in range(E):
        t_sel, j_sel = np.nonzero(idx == e)
        if t_sel.size == 0:
            continue
        W = dequant(codes[e], zero_codes[e], scales[e], G)            # [K, N]
        ye = xr[t_sel] @ W
        if bias is not None:
            ye += np.asarray(bias[e], dtype=np.float64).reshape(1, N)
        y[t_sel, j_sel] = ye
    return y


def transform_weight(W: np.ndarray, channel_scales: Optional[np.ndarray], pairs: Optional[np.ndarray],
                     theta: Optional[np.ndarray], group_size: int, krot: Optional[int] = None) -> np.ndarray:
    """W_r = W D R in float64: row n of W [N, K] (out x in) is multiplied by
    D = 1 / channel_scales per input channel and then takes the same krot
    stages as an activation row, so that X_r W_r^T = X W^T."""
    W = np.asarray(W)
    if W.ndim != 2:
        raise ValueError("W must be 2-D [N, K]")
    D = None
    if channel_scales is not None:
        D = 1.0 / np.asarray(channel_scales, dtype=np.float64)
    return rotate(W, D, pairs, theta, group_size, krot=krot)


def quantize_sym4(W_r: np.ndarray, scales: np.ndarray, group_size: int):
    """Four-bit symmetric quantisation of W_r [N, K] with group scales [K//G, N].

    s = scales[k // G, n] bounded to [QSCALE_MIN, QSCALE_MAX];
    q = clamp(round_half_even(W_r / s), -8, 7); code = q + 8 (uint8 0..15).
    Returns codes [N, K] and zero codes [N, K//G] (all 8), the ``awq_pack`` inputs.
    """
    W_r = np.asarray(W_r, dtype=np.float64)
    N, K = W_r.shape
    G = normalize_group_size(group_size, K)
    s = np.clip(np.asarray(scales, dtype=np.float64), QSCALE_MIN, QSCALE_MAX)
    if s.shape != (K // G, N):
        raise ValueError(f"scales must be [{K // G}, {N}]")
    s_nk = np.repeat(s.T, G, axis=1)                       # [N, K]
    q = np.clip(np.rint(W_r / s_nk), SYM_QMIN, SYM_QMAX)   # np.rint: ties to even
    codes = (q + SYM_ZERO_CODE).astype(np.uint8)
    zeros = np.full((N, K // G), SYM_ZERO_CODE, dtype=np.uint8)
    return codes, zeros


def quantize_weight(W, channel_scales, pairs, theta, scales, group_size, krot=None):
    """Packed runtime weights from float weights: AWQ-packed Q(W_r).
    Returns qweight [K, N//8] int32 and qzeros [K//G, N//8] int32."""
    K = np.asarray(W).shape[1]
    G = normalize_group_size(group_size, K)
    W_r = transform_weight(W, channel_scales, pairs, theta, G, krot=krot)
    codes, zeros = quantize_sym4(W_r, scales, G)
    return awq_pack(codes, zeros, G)
