"""Helpers shared by the GPU parity tests: device copies of synthetic layers and
the comparison rules.  Tolerances (from the layer's numerical contract):
  * rotated activations:  |d_i| <= 1e-3 * max(|ref_i|, rms(ref row))
  * linear outputs:       max|Y_gpu - Y_oracle| <= 2e-2 * rms(Y_oracle)
  * packing / indices:    bit-exact
  * weight codes:         bit-exact, except where the exact quotient W_r / s
                          lies within the fp32 error bound of the transform
                          of a rounding boundary (a half-integer between
                          -7.5 and 6.5): there either neighbouring code is
                          correct (``check_codes``)
"""
from __future__ import annotations

import numpy as np
import torch

ROT_TOL = 1e-3
LIN_TOL = 2e-2


def dev(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def layer_to_device(lay, pack_with_gpu=True):
    import rotation_w4_weight_b200 as pb
    d = dict(
        pairs=dev(lay.pairs), theta=dev(lay.theta), cs=dev(lay.channel_scales),
        scales=dev(lay.scales), bias=dev(lay.bias),
    )
    codes = dev(lay.codes)
    zeros = dev(lay.zero_codes)
    d["qweight"], d["qzeros"] = pb.pack_awq(codes, zeros, lay.group_size)
    del codes, zeros
    return d


def rot_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max_i |d_i| / max(|ref_i|, rms(ref row)) — must be <= ROT_TOL."""
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    denom = np.maximum(np.abs(ref), rms)
    denom = np.where(denom == 0, 1.0, denom)
    return float(np.max(np.abs(got - ref) / denom)) if got.size else 0.0


def lin_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max|Y_gpu - Y_ref| / rms(Y_ref) — must be <= LIN_TOL."""
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / (rms if rms > 0 else 1.0)


def code_margin(W, channel_scales, scales, G, krot):
    """Per-element bound on |t_gpu - t| for t = W_r / s, from the fp32 path:
    the 1/cs scaling and the final multiply (a few units in the last place),
    and per stage the hardware cos/sin (absolute error below 2^-20 each) and
    two roundings, each scaled by the group's norm (the stages are orthogonal,
    so that norm bounds every intermediate).  Doubled for safety."""
    Wd = np.asarray(W, np.float64)
    if channel_scales is not None:
        Wd = Wd / np.asarray(channel_scales, np.float64).reshape(1, -1)
    N, K = Wd.shape
    norm = np.sqrt((Wd.reshape(N, K // G, G) ** 2).sum(axis=2))          # [N, K/G]
    s = np.clip(np.asarray(scales, np.float64), 1e-5, 1e5).T              # [N, K/G]
    per_group = (krot * 2.2e-6 + 4e-7) * norm / s
    return 2.0 * np.repeat(per_group, G, axis=1)


def check_codes(codes_gpu, W, channel_scales, pairs, theta, scales, G, krot, rows=None):
    """Compare GPU codes [R, K] (rows ``rows`` of the layer, default all) with the
    oracle; returns (mismatches, ambiguous, total).  A mismatch is a code that
    differs where the oracle's code is unique, or by more than one level."""
    import oracle
    W = np.asarray(W)
    if rows is not None:
        W = W[rows]
        scales = np.asarray(scales)[:, rows]
    W_r = oracle.transform_weight(W, channel_scales, pairs, theta, G, krot=krot)
    ref_codes, _ = oracle.quantize_sym4(W_r, scales, G)
    s = np.repeat(np.clip(np.asarray(scales, np.float64), 1e-5, 1e5).T, G, axis=1)
    t = W_r / s
    # distance to the nearest boundary between two codes
    b = np.clip(np.floor(t) + 0.5, -7.5, 6.5)
    dist = np.minimum(np.abs(t - b), np.abs(t - np.clip(b - 1.0, -7.5, 6.5)))
    amb = dist <= code_margin(W, channel_scales, scales, G, krot)
    diff = codes_gpu.astype(np.int64) - ref_codes.astype(np.int64)
    bad = ((diff != 0) & ~amb) | (np.abs(diff) > 1)
    return int(bad.sum()), int(amb.sum()), int(diff.size)
