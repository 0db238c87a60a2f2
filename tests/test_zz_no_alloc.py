"""paro_w4_linear_noalloc: the rotated W4 linear for callers that cannot allocate
device memory (graph capture in the global mode, allocation-free hot loops,
plugin hosts that own all device memory).  Its scratch is a static device array
inside the library.  Checked through the C ABI against paro_w4_linear on the
same inputs, twice in a row (the shared array keeps the previous call's
contents, so the second call must not depend on them).  This file is named to be
collected last."""
import ctypes

import numpy as np
import pytest

import synth
from tests.gpu_util import LIN_TOL, dev, layer_to_device, lin_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from rotation_w4_weight_b200 import _lib as L  # noqa: E402


def P(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def linear_ref(d, x, M, krot, use_cs):
    """paro_w4_linear with its own workspace: the reference result."""
    K, N = x.shape[1], d["qweight"].shape[1] * 8
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws_bytes = L.paro_w4_linear_workspace_size(M, K, N, 128)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    cs = d["cs"] if use_cs else None
    pairs = d["pairs"] if krot else None
    theta = d["theta"] if krot else None
    st = L.paro_w4_linear(P(x), P(y), M, K, N, P(d["qweight"]), P(d["qzeros"]), P(d["scales"]),
                          P(d["bias"]), P(cs), P(pairs), P(theta), 128, krot, P(ws), ws.numel(), None)
    assert st == L.PARO_OK
    return y.cpu().numpy().astype(np.float64)


def noalloc(d, x, M, krot, use_cs):
    K, N = x.shape[1], d["qweight"].shape[1] * 8
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    cs = d["cs"] if use_cs else None
    pairs = d["pairs"] if krot else None
    theta = d["theta"] if krot else None
    st = L.paro_w4_linear_noalloc(P(x), P(y), M, K, N, P(d["qweight"]), P(d["qzeros"]),
                                  P(d["scales"]), P(d["bias"]), P(cs), P(pairs), P(theta),
                                  128, krot, None)
    assert st == L.PARO_OK
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    return got


def run_both(lay, M, krot, use_cs):
    """Two checked calls in a row.  Between them a call on a different layer and
    different activations of the same shape overwrites the shared scratch, so a
    second call that read anything left over from an earlier one would differ
    from its own reference."""
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, M))
    other = synth.make_layer(lay.name + "_other", lay.K, lay.N, seed=lay.seed + 1000,
                             bias_std=0.01, zero_point=None)
    d2 = layer_to_device(other)
    x2 = dev(synth.make_activations(other, M))
    ref = linear_ref(d, x, M, krot, use_cs)
    ref2 = linear_ref(d2, x2, M, krot, use_cs)
    assert lin_err(noalloc(d, x, M, krot, use_cs), ref) <= LIN_TOL
    assert lin_err(noalloc(d2, x2, M, krot, use_cs), ref2) <= LIN_TOL
    assert lin_err(noalloc(d, x, M, krot, use_cs), ref) <= LIN_TOL
    assert L.paro_device_status(1) == L.PARO_OK


@pytest.mark.parametrize("M", [1, 16])
def test_noalloc_matches_workspace_version_decode(M):
    lay = synth.make_layer("na", 4096, 1024, seed=91, n_outliers=41)
    run_both(lay, M, 8, True)


@pytest.mark.parametrize("M", [40, 96, 300])   # above 64 rows the rotation runs on the tensor cores (R' in the scratch too)
def test_noalloc_matches_workspace_version_prefill_with_bias(M):
    lay = synth.make_layer("nb", 512, 512, seed=92, bias_std=0.01, zero_point=None)
    run_both(lay, M, 8, True)


def test_noalloc_plain_awq_needs_no_scratch():
    lay = synth.make_layer("nc", 256, 512, seed=93)
    run_both(lay, 4, 0, False)


def test_noalloc_plain_awq_has_no_size_limit():
    """A call that does not rotate stages nothing: shapes whose rotation would
    not fit the static scratch still run (here X_r would need 16 MiB)."""
    M, K, N = 2048, 4096, 256
    assert L.paro_w4_linear_workspace_size(M, K, N, 128) > L.PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES
    lay = synth.make_layer("nd", K, N, seed=94, zero_point=None)
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, M))
    assert lin_err(noalloc(d, x, M, 0, False), linear_ref(d, x, M, 0, False)) <= LIN_TOL
    assert L.paro_device_status(1) == L.PARO_OK


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    M, K, N = 2048, 4096, 512            # X_r needs 16 MiB > 8 MiB
    assert L.paro_w4_linear_workspace_size(M, K, N, 128) > L.PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(0x10000)         # never dereferenced: rejected on the host
    # channel scales make the call rotate (it needs the scratch)
    st = L.paro_w4_linear_noalloc(a, a, M, K, N, a, a, a, None, a, None, None, 128, 0, None)
    assert st == L.PARO_ERR_WORKSPACE
    # bad arguments get the status paro_w4_linear gives them, whatever the size
    st = L.paro_w4_linear_noalloc(a, None, M, K, N, a, a, a, None, a, None, None, 128, 0, None)
    assert st == L.PARO_ERR_INVALID_ARG
    st = L.paro_w4_linear_noalloc(a, a, M, K, N, a, a, a, None, a, None, None, 128, -1, None)
    assert st == L.PARO_ERR_INVALID_ARG
