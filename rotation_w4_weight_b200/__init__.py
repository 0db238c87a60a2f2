"""B200 (sm_100a) library for ParoQuant's scaled pairwise-rotated INT4 linear layer.

The compute lives in the CUDA library ``libparo_b200.so`` behind the C ABI of
``include/paro.h``; this module only marshals torch tensors (device memory and
streams) into that ABI.  Functions mirror the C entry points:

    rotate            -> paro_rotate / paro_rotate_dt, or paro_rotate_rmat with a prepared R'
    pack_awq          -> paro_pack_awq
    unpack_awq        -> paro_unpack_awq
    w4_linear         -> paro_w4_linear / paro_w4_linear_dt (+ paro_w4_linear_workspace_size)
    w4_linear_group   -> paro_w4_linear_group / paro_w4_linear_group_dt (+ ..._workspace_size)
    quantize_w4       -> paro_quantize_w4_tc (+ its workspace size), or paro_quantize_w4 / paro_quantize_w4_dt
    validate_pairs    -> paro_validate_pairs (host helper)
    device_status     -> paro_device_status
    rotation_matrix   -> paro_rotation_matrix_prepare (+ paro_rotation_matrix_size)
    w4_moe_linear     -> paro_w4_moe_linear (+ paro_w4_moe_workspace_size, paro_w4_moe_launches)

Activations, scales, bias and outputs are fp16 or bf16 (one type per call,
taken from x): fp16 calls go to the plain entry points, bf16 calls to the
``*_dt`` twins with ``PARO_DTYPE_BF16``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from ._lib import (PARO_ERR_ALIGNMENT, PARO_ERR_CUDA, PARO_ERR_INVALID_ARG,  # noqa: F401
                   PARO_ERR_TIMEOUT, PARO_ERR_UNSUPPORTED, PARO_ERR_WORKSPACE, PARO_OK,
                   LIB_PATH, ParoError, check, lib, paro_device_status, paro_pack_awq,
                   paro_quantize_w4, paro_rotate, paro_status_string, paro_unpack_awq,
                   paro_validate_pairs, paro_version, paro_w4_linear, paro_w4_linear_workspace_size,
                   PARO_MAX_GROUP, ParoLinear, paro_w4_linear_group, paro_w4_linear_group_launches,
                   paro_w4_linear_group_workspace_size, PARO_DTYPE_BF16, paro_rotate_dt, paro_quantize_w4_dt,
                   paro_w4_linear_dt, paro_w4_linear_group_dt, paro_rotation_matrix_size,
                   paro_rotation_matrix_prepare, PARO_DTYPE_F16, paro_w4_moe_workspace_size,
                   paro_w4_moe_linear, paro_w4_moe_launches, paro_quantize_w4_workspace_size,
                   paro_quantize_w4_tc, paro_rotate_rmat)

__all__ = ["rotate", "pack_awq", "unpack_awq", "w4_linear", "w4_linear_workspace_size",
           "w4_linear_group", "w4_linear_group_launches", "quantize_w4", "validate_pairs", "device_status",
           "rotation_matrix", "w4_moe_linear", "w4_moe_launches", "ParoError", "LIB_PATH"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_ACT_TYPES = (torch.float16, torch.bfloat16)


def _act(t: torch.Tensor, name: str):
    """The activation type of a call (fp16 or bf16), taken from its input."""
    if t.dtype not in _ACT_TYPES:
        raise TypeError(f"{name} must be float16 or bfloat16, got {t.dtype}")
    return t.dtype


def _need(t: Optional[torch.Tensor], dtype, name: str, allow_none: bool = False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def rotate(x: torch.Tensor, channel_scales: Optional[torch.Tensor], pairs: Optional[torch.Tensor],
           theta: Optional[torch.Tensor], group_size: int = 128, krot: Optional[int] = None,
           out: Optional[torch.Tensor] = None, stream=None, rmat: Optional[torch.Tensor] = None) -> torch.Tensor:
    """X_r = rotate(x * channel_scales); ``out`` may be ``x`` (in place).

    With ``rmat`` (this layer's prepared R', ``rotation_matrix``) the product
    x R' runs on the tensor cores (channel_scales/pairs/theta are then not
    read; ``out`` must be another buffer)."""
    dt = _act(x, "x")
    _need(x, dt, "x")
    if rmat is not None:
        _need(rmat, torch.uint8, "rmat")
        if out is None:
            out = torch.empty_like(x)
        _need(out, dt, "out")
        M, K = x.shape
        check(paro_rotate_rmat(_ptr(x), _ptr(out), M, K, _ptr(rmat),
                               PARO_DTYPE_F16 if dt == torch.float16 else PARO_DTYPE_BF16, _stream(stream)),
              "paro_rotate_rmat")
        return out
    _need(channel_scales, torch.float32, "channel_scales", True)
    _need(pairs, torch.int16, "pairs", True)
    _need(theta, torch.float32, "theta", True)
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    if out is None:
        out = torch.empty_like(x)
    _need(out, dt, "out")
    M, K = x.shape
    args = (_ptr(x), _ptr(out), M, K, _ptr(channel_scales), _ptr(pairs), _ptr(theta), group_size, krot)
    if dt == torch.float16:
        check(paro_rotate(*args, _stream(stream)), "paro_rotate")
    else:
        check(paro_rotate_dt(*args, PARO_DTYPE_BF16, _stream(stream)), "paro_rotate_dt")
    return out


def pack_awq(codes: torch.Tensor, zero_codes: Optional[torch.Tensor], group_size: int = 128,
             stream=None):
    """codes uint8 [N, K], zero_codes uint8 [N, K/G] -> (qweight int32 [K, N/8], qzeros)."""
    _need(codes, torch.uint8, "codes")
    _need(zero_codes, torch.uint8, "zero_codes", True)
    N, K = codes.shape
    G = K if group_size == -1 else group_size
    qweight = torch.empty((K, N // 8), dtype=torch.int32, device=codes.device)
    qzeros = None
    if zero_codes is not None:
        qzeros = torch.empty((K // G, N // 8), dtype=torch.int32, device=codes.device)
    check(paro_pack_awq(_ptr(codes), _ptr(zero_codes), _ptr(qweight), _ptr(qzeros), N, K,
                        group_size, _stream(stream)), "paro_pack_awq")
    return qweight, qzeros


def quantize_w4(w: torch.Tensor, channel_scales: Optional[torch.Tensor], pairs: Optional[torch.Tensor],
                theta: Optional[torch.Tensor], scales: torch.Tensor, group_size: int = 128,
                krot: Optional[int] = None, out=None, stream=None, method: str = "auto",
                workspace: Optional[torch.Tensor] = None):
    """Float weights w fp16/bf16 [N, K] (out x in) -> (qweight int32 [K, N/8], qzeros int32 [K/G, N/8]):
    W_r = W D R, four-bit symmetric codes with the quantiser scales [K/G, N] (w's type), AWQ-packed.

    ``method``: "tensor" (paro_quantize_w4_tc: the stages as one matrix per
    group on the tensor cores; fp16 weights, N % 32 == 0), "pairs"
    (paro_quantize_w4[_dt]: stage by stage), or "auto" (tensor where it
    applies)."""
    dt = _act(w, "w")
    _need(w, dt, "w")
    _need(channel_scales, torch.float32, "channel_scales", True)
    _need(pairs, torch.int16, "pairs", True)
    _need(theta, torch.float32, "theta", True)
    _need(scales, dt, "scales")
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    N, K = w.shape
    G = K if group_size == -1 else group_size
    if out is None:
        out = (torch.empty((K, N // 8), dtype=torch.int32, device=w.device),
               torch.empty((K // G, N // 8), dtype=torch.int32, device=w.device))
    qweight, qzeros = out
    args = (_ptr(w), _ptr(channel_scales), _ptr(pairs), _ptr(theta), _ptr(scales), _ptr(qweight), _ptr(qzeros),
            N, K, group_size, krot)
    if method not in ("auto", "tensor", "pairs"):
        raise ValueError(f"method must be auto, tensor or pairs, got {method}")
    tensor = method == "tensor" or (method == "auto" and dt == torch.float16 and N % 32 == 0)
    if tensor:
        need = int(paro_quantize_w4_workspace_size(K))
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=w.device)
        check(paro_quantize_w4_tc(*args, _ptr(workspace), workspace.numel(), _stream(stream)),
              "paro_quantize_w4_tc")
    elif dt == torch.float16:
        check(paro_quantize_w4(*args, _stream(stream)), "paro_quantize_w4")
    else:
        check(paro_quantize_w4_dt(*args, PARO_DTYPE_BF16, _stream(stream)), "paro_quantize_w4_dt")
    return qweight, qzeros


def unpack_awq(qweight: torch.Tensor, qzeros: Optional[torch.Tensor], N: int, K: int,
               group_size: int = 128, stream=None):
    _need(qweight, torch.int32, "qweight")
    _need(qzeros, torch.int32, "qzeros", True)
    G = K if group_size == -1 else group_size
    codes = torch.empty((N, K), dtype=torch.uint8, device=qweight.device)
    zeros = None
    if qzeros is not None:
        zeros = torch.empty((N, K // G), dtype=torch.uint8, device=qweight.device)
    check(paro_unpack_awq(_ptr(qweight), _ptr(qzeros), _ptr(codes), _ptr(zeros), N, K,
                          group_size, _stream(stream)), "paro_unpack_awq")
    return codes, zeros


def w4_linear_workspace_size(M: int, K: int, N: int, group_size: int = 128) -> int:
    return int(paro_w4_linear_workspace_size(M, K, N, group_size))


def w4_linear(x: torch.Tensor, qweight: torch.Tensor, qzeros: torch.Tensor, scales: torch.Tensor,
              bias: Optional[torch.Tensor], channel_scales: Optional[torch.Tensor],
              pairs: Optional[torch.Tensor], theta: Optional[torch.Tensor],
              group_size: int = 128, krot: Optional[int] = None,
              workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              stream=None, rmat: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y = rotate(x * channel_scales) @ dequant(qweight, qzeros, scales) + bias (out in x's type).

    ``rmat``: this layer's prepared R' (``rotation_matrix``); the call then
    goes through the grouped entry point with one member, which is where the
    C ABI takes it."""
    if rmat is not None:
        m = dict(qweight=qweight, qzeros=qzeros, scales=scales, bias=bias, channel_scales=channel_scales,
                 pairs=pairs, theta=theta, krot=krot, rmat=rmat)
        return w4_linear_group(x, [m], group_size, workspace=workspace,
                               out=None if out is None else [out], stream=stream)[0]
    dt = _act(x, "x")
    _need(x, dt, "x")
    _need(qweight, torch.int32, "qweight")
    _need(qzeros, torch.int32, "qzeros")
    _need(scales, dt, "scales")
    _need(bias, dt, "bias", True)
    _need(channel_scales, torch.float32, "channel_scales", True)
    _need(pairs, torch.int16, "pairs", True)
    _need(theta, torch.float32, "theta", True)
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    M, K = x.shape
    N = qweight.shape[1] * 8
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=x.device)
    _need(out, dt, "out")
    need = w4_linear_workspace_size(M, K, N, group_size)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    args = (_ptr(x), _ptr(out), M, K, N, _ptr(qweight), _ptr(qzeros), _ptr(scales), _ptr(bias),
            _ptr(channel_scales), _ptr(pairs), _ptr(theta), group_size, krot)
    if dt == torch.float16:
        check(paro_w4_linear(*args, _ptr(workspace), ws_bytes, _stream(stream)), "paro_w4_linear")
    else:
        check(paro_w4_linear_dt(*args, PARO_DTYPE_BF16, _ptr(workspace), ws_bytes, _stream(stream)),
              "paro_w4_linear_dt")
    return out


def validate_pairs(pairs: np.ndarray, K: int, group_size: int = 128, krot: Optional[int] = None) -> bool:
    """Host check that each stage of each group is a permutation of 0..G-1."""
    p = np.ascontiguousarray(pairs, dtype=np.int16)
    if krot is None:
        krot = p.shape[0]
    st = paro_validate_pairs(p.ctypes.data_as(ctypes.c_void_p), K, group_size, krot)
    return st == PARO_OK


def device_status(clear: bool = True) -> int:
    """Synchronises and returns the device status word as a PARO_* code."""
    return int(paro_device_status(1 if clear else 0))


def _members(x: torch.Tensor, members, outs):
    arr = (ParoLinear * len(members))()
    for i, m in enumerate(members):
        _need(m["qweight"], torch.int32, "qweight")
        _need(m["qzeros"], torch.int32, "qzeros")
        _need(m["scales"], x.dtype, "scales")
        _need(m.get("bias"), x.dtype, "bias", True)
        _need(outs[i], x.dtype, "out")
        _need(m.get("channel_scales"), torch.float32, "channel_scales", True)
        _need(m.get("pairs"), torch.int16, "pairs", True)
        _need(m.get("theta"), torch.float32, "theta", True)
        krot = m.get("krot")
        if krot is None:
            krot = 0 if m.get("pairs") is None else m["pairs"].shape[0]
        N = m["qweight"].shape[1] * 8
        _need(m.get("rmat"), torch.uint8, "rmat", True)
        arr[i] = ParoLinear(N, m["qweight"].data_ptr(), m["qzeros"].data_ptr(), m["scales"].data_ptr(),
                            None if m.get("bias") is None else m["bias"].data_ptr(),
                            None if m.get("channel_scales") is None else m["channel_scales"].data_ptr(),
                            None if m.get("pairs") is None else m["pairs"].data_ptr(),
                            None if m.get("theta") is None else m["theta"].data_ptr(), krot,
                            outs[i].data_ptr(), None if m.get("rmat") is None else m["rmat"].data_ptr())
    return arr


def w4_linear_group(x: torch.Tensor, members, group_size: int = 128, workspace: Optional[torch.Tensor] = None,
                    out=None, stream=None):
    """Several linears over the same x (q/k/v, gate/up): ``members`` is a list of
    dicts with keys qweight, qzeros, scales and optionally bias, channel_scales,
    pairs, theta, krot and rmat (from ``rotation_matrix``).
    Returns the list of outputs [M, N_i] in x's type."""
    dt = _act(x, "x")
    _need(x, dt, "x")
    M, K = x.shape
    if out is None:
        out = [torch.empty((M, m["qweight"].shape[1] * 8), dtype=dt, device=x.device) for m in members]
    arr = _members(x, members, out)
    need = int(paro_w4_linear_group_workspace_size(M, K, len(members), arr, group_size))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    if dt == torch.float16:
        check(paro_w4_linear_group(_ptr(x), M, K, len(members), arr, group_size, _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "paro_w4_linear_group")
    else:
        check(paro_w4_linear_group_dt(_ptr(x), M, K, len(members), arr, group_size, PARO_DTYPE_BF16,
                                      _ptr(workspace), workspace.numel(), _stream(stream)),
              "paro_w4_linear_group_dt")
    return out


def w4_linear_group_launches(M: int, K: int, members, group_size: int = 128) -> int:
    """Kernel launches one ``w4_linear_group`` call of this shape issues.

    ``members``: dicts with N and optionally krot (default 8), channel_scales
    (bool, default True), same_rotation_as (index of an earlier member whose
    rotation tables this member shares) and rmat (bool: the member carries a
    prepared R'; default False).  Only shapes and table identity matter: the
    descriptors carry placeholder addresses, never dereferenced."""
    arr = (ParoLinear * len(members))()
    for i, m in enumerate(members):
        owner = m.get("same_rotation_as", i)
        tag = 256 * (owner + 1)                  # distinct per rotation, shared by its members
        krot = m.get("krot", 8)
        arr[i] = ParoLinear(m["N"], None, None, None, None, tag if m.get("channel_scales", True) else None,
                            tag if krot > 0 else None, tag if krot > 0 else None, krot, None,
                            tag if m.get("rmat", False) else None)
    return int(paro_w4_linear_group_launches(M, K, len(members), arr, group_size))


def rotation_matrix(channel_scales: Optional[torch.Tensor], pairs: Optional[torch.Tensor],
                    theta: Optional[torch.Tensor], K: int, group_size: int = 128, krot: Optional[int] = None,
                    dtype=torch.float16, stream=None) -> torch.Tensor:
    """This layer's R' parts, built once (uint8 device tensor of
    paro_rotation_matrix_size(K) bytes): pass it as ``rmat=`` on the layer's
    calls.  ``dtype`` is the activation type of those calls."""
    _need(channel_scales, torch.float32, "channel_scales", True)
    _need(pairs, torch.int16, "pairs", True)
    _need(theta, torch.float32, "theta", True)
    if dtype not in _ACT_TYPES:
        raise TypeError(f"dtype must be float16 or bfloat16, got {dtype}")
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    n = int(paro_rotation_matrix_size(K))
    if n == 0:
        raise ParoError(PARO_ERR_INVALID_ARG, "paro_rotation_matrix_size")
    src = [t for t in (channel_scales, pairs, theta) if t is not None]
    out = torch.empty(n, dtype=torch.uint8, device=src[0].device if src else torch.device("cuda"))
    code = PARO_DTYPE_F16 if dtype == torch.float16 else PARO_DTYPE_BF16
    check(paro_rotation_matrix_prepare(_ptr(channel_scales), _ptr(pairs), _ptr(theta), K, group_size, krot, code,
                                       _ptr(out), n, _stream(stream)), "paro_rotation_matrix_prepare")
    return out


def w4_moe_linear(x: torch.Tensor, expert_idx: torch.Tensor, qweight: torch.Tensor, qzeros: torch.Tensor,
                  scales: torch.Tensor, bias: Optional[torch.Tensor], channel_scales: Optional[torch.Tensor],
                  pairs: Optional[torch.Tensor], theta: Optional[torch.Tensor], group_size: int = 128,
                  krot: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Stacked experts sharing one rotation: y[t, j] = rotate(x[t]) @ W[expert_idx[t, j]] + b[...].

    x [T, K]; expert_idx int32 [T, topk]; qweight int32 [E, K, N/8]; qzeros
    int32 [E, K/G, N/8]; scales [E, K/G, N]; bias [E, N] or None.  Returns
    y [T, topk, N] in x's type."""
    dt = _act(x, "x")
    _need(x, dt, "x")
    _need(expert_idx, torch.int32, "expert_idx")
    _need(qweight, torch.int32, "qweight")
    _need(qzeros, torch.int32, "qzeros")
    _need(scales, dt, "scales")
    _need(bias, dt, "bias", True)
    _need(channel_scales, torch.float32, "channel_scales", True)
    _need(pairs, torch.int16, "pairs", True)
    _need(theta, torch.float32, "theta", True)
    if krot is None:
        krot = 0 if pairs is None else pairs.shape[0]
    T, K = x.shape
    topk = expert_idx.shape[1] if expert_idx.dim() == 2 else 1
    E, N = qweight.shape[0], qweight.shape[2] * 8
    if out is None:
        out = torch.empty((T, topk, N), dtype=dt, device=x.device)
    _need(out, dt, "out")
    need = int(paro_w4_moe_workspace_size(T, K, N, E, topk, group_size))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    check(paro_w4_moe_linear(_ptr(x), _ptr(out), T, K, N, E, topk, _ptr(expert_idx), _ptr(qweight), _ptr(qzeros),
                             _ptr(scales), _ptr(bias), _ptr(channel_scales), _ptr(pairs), _ptr(theta), group_size,
                             krot, PARO_DTYPE_F16 if dt == torch.float16 else PARO_DTYPE_BF16, _ptr(workspace),
                             workspace.numel(), _stream(stream)), "paro_w4_moe_linear")
    return out


def w4_moe_launches(T: int, K: int, N: int, E: int, topk: int, group_size: int = 128, krot: int = 8,
                    rotate: bool = True) -> int:
    """Kernel launches one ``w4_moe_linear`` call of this shape issues (host-only)."""
    return int(paro_w4_moe_launches(T, K, N, E, topk, group_size, krot, 1 if rotate else 0))
