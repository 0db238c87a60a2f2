"""ctypes binding of the C ABI in include/paro.h (argument marshalling only).

Every function of the header is exposed here under the same name.  The
library must exist (build it with ``python rotation_w4_weight_b200/build.py``);
importing this module without it raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libparo_b200.so")

PARO_OK = 0
PARO_ERR_INVALID_ARG = 1
PARO_ERR_UNSUPPORTED = 2
PARO_ERR_ALIGNMENT = 3
PARO_ERR_WORKSPACE = 4
PARO_ERR_CUDA = 5
PARO_ERR_TIMEOUT = 6

PARO_DTYPE_F16 = 0
PARO_DTYPE_BF16 = 1

EXPORTED = (
    "paro_status_string", "paro_version", "paro_rotate", "paro_pack_awq", "paro_unpack_awq",
    "paro_w4_linear_workspace_size", "paro_w4_linear", "paro_w4_linear_noalloc",
    "paro_validate_pairs", "paro_device_status", "paro_quantize_w4",
    "paro_w4_linear_group_workspace_size", "paro_w4_linear_group", "paro_w4_linear_group_launches",
    "paro_selftest_wait_timeout", "paro_rotate_dt", "paro_quantize_w4_dt", "paro_w4_linear_dt",
    "paro_w4_linear_group_dt", "paro_w4_linear_noalloc_dt", "paro_rotation_matrix_size",
    "paro_rotation_matrix_prepare", "paro_w4_moe_workspace_size", "paro_w4_moe_linear", "paro_w4_moe_launches",
    "paro_quantize_w4_workspace_size", "paro_quantize_w4_tc", "paro_rotate_rmat",
)

PARO_MAX_GROUP = 4


class ParoLinear(ctypes.Structure):
    """struct paro_linear of the header (one member of a grouped call)."""
    _fields_ = [("N", ctypes.c_int64), ("qweight", ctypes.c_void_p), ("qzeros", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("channel_scales", ctypes.c_void_p),
                ("pairs", ctypes.c_void_p), ("theta", ctypes.c_void_p), ("krot", ctypes.c_int),
                ("y", ctypes.c_void_p), ("rmat", ctypes.c_void_p)]

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int

_SIGNATURES = {
    "paro_status_string": (ctypes.c_char_p, [_int]),
    "paro_version": (ctypes.c_char_p, []),
    "paro_rotate": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _int, _int, _vp]),
    "paro_pack_awq": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _vp]),
    "paro_unpack_awq": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _int, _vp]),
    "paro_w4_linear_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _int]),
    "paro_w4_linear": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                              _int, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_linear_noalloc": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _int, _int, _vp]),
    "paro_validate_pairs": (_int, [_vp, _i64, _int, _int]),
    "paro_device_status": (_int, [_int]),
    "paro_quantize_w4": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _vp]),
    "paro_w4_linear_group_workspace_size": (ctypes.c_size_t, [_i64, _i64, _int, _vp, _int]),
    "paro_w4_linear_group": (_int, [_vp, _i64, _i64, _int, _vp, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_linear_group_launches": (_int, [_i64, _i64, _int, _vp, _int]),
    "paro_selftest_wait_timeout": (_int, [ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint64), _vp]),
    "paro_rotate_dt": (_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _int, _int, _int, _vp]),
    "paro_quantize_w4_dt": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _int, _vp]),
    "paro_w4_linear_dt": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _int, _int, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_linear_group_dt": (_int, [_vp, _i64, _i64, _int, _vp, _int, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_linear_noalloc_dt": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                         _vp, _int, _int, _int, _vp]),
    "paro_rotation_matrix_size": (ctypes.c_size_t, [_i64]),
    "paro_rotation_matrix_prepare": (_int, [_vp, _vp, _vp, _i64, _int, _int, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_moe_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _int, _int, _int]),
    "paro_w4_moe_linear": (_int, [_vp, _vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _int, _int, _int, _vp, ctypes.c_size_t, _vp]),
    "paro_w4_moe_launches": (_int, [_i64, _i64, _i64, _int, _int, _int, _int, _int]),
    "paro_quantize_w4_workspace_size": (ctypes.c_size_t, [_i64]),
    "paro_rotate_rmat": (_int, [_vp, _vp, _i64, _i64, _vp, _int, _vp]),
    "paro_quantize_w4_tc": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _int, _int, _vp, ctypes.c_size_t,
                                   _vp]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build the CUDA library first "
            "(python rotation_w4_weight_b200/build.py); there is no CPU fallback")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()

paro_status_string = lib.paro_status_string
paro_version = lib.paro_version
paro_rotate = lib.paro_rotate
paro_pack_awq = lib.paro_pack_awq
paro_unpack_awq = lib.paro_unpack_awq
paro_w4_linear_workspace_size = lib.paro_w4_linear_workspace_size
paro_w4_linear = lib.paro_w4_linear
paro_w4_linear_noalloc = lib.paro_w4_linear_noalloc
PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES = 8 << 20
paro_validate_pairs = lib.paro_validate_pairs
paro_device_status = lib.paro_device_status
paro_quantize_w4 = lib.paro_quantize_w4
paro_w4_linear_group_workspace_size = lib.paro_w4_linear_group_workspace_size
paro_w4_linear_group = lib.paro_w4_linear_group
paro_w4_linear_group_launches = lib.paro_w4_linear_group_launches
paro_selftest_wait_timeout = lib.paro_selftest_wait_timeout
paro_rotate_dt = lib.paro_rotate_dt
paro_quantize_w4_dt = lib.paro_quantize_w4_dt
paro_w4_linear_dt = lib.paro_w4_linear_dt
paro_w4_linear_group_dt = lib.paro_w4_linear_group_dt
paro_w4_linear_noalloc_dt = lib.paro_w4_linear_noalloc_dt
paro_rotation_matrix_size = lib.paro_rotation_matrix_size
paro_rotation_matrix_prepare = lib.paro_rotation_matrix_prepare
paro_w4_moe_workspace_size = lib.paro_w4_moe_workspace_size
paro_w4_moe_linear = lib.paro_w4_moe_linear
paro_w4_moe_launches = lib.paro_w4_moe_launches
paro_quantize_w4_workspace_size = lib.paro_quantize_w4_workspace_size
paro_quantize_w4_tc = lib.paro_quantize_w4_tc
paro_rotate_rmat = lib.paro_rotate_rmat


class ParoError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {paro_status_string(status).decode()} (status {status})")


def check(status: int, what: str) -> None:
    if status != PARO_OK:
        raise ParoError(status, what)
