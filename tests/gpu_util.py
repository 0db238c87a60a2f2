"""Helpers shared by the GPU parity tests: device copies of synthetic layers and
the comparison rules.  Tolerances (from the layer's numerical contract):
  * rotated activations:  |d_i| <= 1e-3 * max(|ref_i|, rms(ref row))
  * linear outputs:       max|Y_gpu - Y_oracle| <= 2e-2 * rms(Y_oracle)
  * packing / indices:    bit-exact
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
