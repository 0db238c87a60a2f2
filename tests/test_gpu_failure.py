"""Failure detection on the GPU without a fault: a bounded device wait that
runs out is reported through the device status word, the kernel returns
normally and the context stays usable.

The wait is the one every kernel of the library uses (an mbarrier wait
bounded by %globaltimer), here with a 2 ms limit on a barrier that nothing
arrives at and no copy in flight (paro_selftest_wait_timeout)."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import LIN_TOL, dev, layer_to_device, lin_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_w4_weight_b200 as pb  # noqa: E402
from rotation_w4_weight_b200 import _lib as L  # noqa: E402


def run_layer_and_check():
    lay = synth.make_layer("after", 512, 256, seed=95, bias_std=0.01, zero_point=None)
    d = layer_to_device(lay)
    for M in (3, 80):                                   # decode GEMV and prefill GEMM paths
        x = synth.make_activations(lay, M)
        y = pb.w4_linear(dev(x), d["qweight"], d["qzeros"], d["scales"], d["bias"], d["cs"], d["pairs"],
                         d["theta"], 128, 8)
        ref = oracle.w4_linear_from_codes(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                          lay.channel_scales, lay.pairs, lay.theta, 128, 8)
        assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL


def test_bounded_wait_runs_out_and_is_reported():
    assert L.paro_device_status(1) in (L.PARO_OK, L.PARO_ERR_TIMEOUT, L.PARO_ERR_INVALID_ARG)
    assert L.paro_device_status(0) == L.PARO_OK
    limit = 2_000_000                                   # 2 ms
    e = ctypes.c_uint64(0)
    assert L.paro_selftest_wait_timeout(limit, ctypes.byref(e), None) == L.PARO_OK
    # it waited at least the limit, and gave up soon after it
    assert limit <= e.value < limit + 50_000_000, e.value
    assert L.paro_device_status(0) == L.PARO_ERR_TIMEOUT      # reported, not cleared
    assert L.paro_device_status(1) == L.PARO_ERR_TIMEOUT      # reported and cleared
    assert L.paro_device_status(0) == L.PARO_OK
    # the context is intact: the layer still computes the right result
    run_layer_and_check()
    assert L.paro_device_status(1) == L.PARO_OK


def test_timeout_on_a_side_stream_then_normal_work():
    s = torch.cuda.Stream()
    e = ctypes.c_uint64(0)
    assert L.paro_selftest_wait_timeout(1_000_000, ctypes.byref(e), ctypes.c_void_p(s.cuda_stream)) == L.PARO_OK
    assert e.value >= 1_000_000
    assert L.paro_device_status(1) == L.PARO_ERR_TIMEOUT
    run_layer_and_check()
    assert L.paro_device_status(1) == L.PARO_OK
