"""GPU parity for group sizes G = 16, 32 and 64 (the rotation groups and the
quantisation groups share G; the kernels hold 128 / G groups per 128-channel
tile).  Every path against the float64 oracle on the same seeded inputs: the
rotation kernels (warp per row, shared-memory tile, tensor memory), the decode
GEMV and the prefill GEMM with the tensor-core rotation, grouped calls and the
weight quantiser."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import LIN_TOL, ROT_TOL, check_codes, dev, layer_to_device, lin_err, rot_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_w4_weight_b200 as pb  # noqa: E402

GROUPS = [16, 32, 64]


@pytest.fixture(autouse=True)
def _status_clean():
    assert pb.device_status(clear=True) == pb.PARO_OK
    yield
    assert pb.device_status(clear=True) == pb.PARO_OK


# (M, K, krot): warp-per-row decode kernel (M <= 16, krot <= 8), 4-row tile
# (krot > 8), 64-row shared-memory tile, tensor-memory kernel (M > 64)
ROT_CASES = [(1, 512, 8), (5, 256, 8), (7, 384, 12), (37, 256, 8), (300, 512, 8), (129, 256, 17)]


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("M,K,krot", ROT_CASES)
def test_rotate_group_sizes(G, M, K, krot):
    lay = synth.make_layer("rg", K, 32, seed=G * 31 + M + krot, group_size=G, krot=krot,
                           n_outliers=max(1, K // 100))
    x = synth.make_activations(lay, M)
    ref = oracle.rotate(x, lay.channel_scales, lay.pairs, lay.theta, G)
    got = pb.rotate(dev(x), dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), G,
                    krot).cpu().numpy().astype(np.float64)
    assert rot_err(got, ref) <= ROT_TOL


@pytest.mark.parametrize("G", GROUPS)
def test_rotate_group_sizes_pairs_stay_in_their_group(G):
    """One pair at a right angle in the last group of a tile moves exactly its
    two channels of that group: a wrong group offset would move others."""
    K, M = 256, 3
    pairs = np.tile(np.arange(G, dtype=np.int16), (1, K // G))
    theta = np.zeros((1, K // 2), np.float32)
    g = 128 // G - 1                                  # last group of the first tile
    theta[0, g * (G // 2) + 1] = np.float32(np.pi / 2)   # pair 1 of that group: channels 2, 3
    x = (np.arange(M * K, dtype=np.float32).reshape(M, K) % 17 - 8).astype(np.float16)
    got = pb.rotate(dev(x), None, dev(pairs), dev(theta), G, 1).cpu().numpy().astype(np.float64)
    ref = oracle.rotate(x, None, pairs, theta, G)
    assert rot_err(got, ref) <= ROT_TOL
    changed = np.nonzero(np.any(np.abs(got - x.astype(np.float64)) > 0, axis=0))[0]
    assert set(changed.tolist()) <= {g * G + 2, g * G + 3}


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("M", [1, 4, 16, 40, 300])   # GEMV, GEMV (2 token tiles), GEMM, GEMM + tensor-core rotation
def test_linear_group_sizes(G, M):
    K, N = 512, 384
    lay = synth.make_layer("lg", K, N, seed=G * 7 + M, group_size=G, bias_std=0.01, zero_point=None)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    y = pb.w4_linear(dev(x), d["qweight"], d["qzeros"], d["scales"], d["bias"], d["cs"], d["pairs"],
                     d["theta"], G, lay.krot)
    ref = oracle.w4_linear_from_codes(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                      lay.channel_scales, lay.pairs, lay.theta, G, lay.krot)
    assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL


@pytest.mark.parametrize("G", GROUPS)
def test_linear_group_sizes_plain_awq(G):
    """No rotation, no channel scales: the group-wise dequantisation alone."""
    K, N, M = 1024, 256, 3
    lay = synth.make_layer("pg", K, N, seed=G + 5, group_size=G, zero_point=None)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    for m in (M, 130):
        xm = synth.make_activations(lay, m)
        y = pb.w4_linear(dev(xm), d["qweight"], d["qzeros"], d["scales"], None, None, None, None, G, 0)
        ref = oracle.w4_linear_from_codes(xm, lay.codes, lay.zero_codes, lay.scales, None, None, None, None, G, 0)
        assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL
    del x


@pytest.mark.parametrize("G", [32, 64])
@pytest.mark.parametrize("M", [1, 96])
def test_group_call_group_sizes(G, M):
    K = 512
    lays = [synth.make_layer(f"m{i}", K, n, seed=G + 40 * i + M, group_size=G, zero_point=None)
            for i, n in enumerate((256, 128, 128))]
    ds = [layer_to_device(l) for l in lays]
    x = synth.make_activations(lays[0], M)
    members = [dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=None,
                    channel_scales=d["cs"], pairs=d["pairs"], theta=d["theta"], krot=l.krot)
               for l, d in zip(lays, ds)]
    ys = pb.w4_linear_group(dev(x), members, G)
    for l, y in zip(lays, ys):
        ref = oracle.w4_linear_from_codes(x, l.codes, l.zero_codes, l.scales, None, l.channel_scales,
                                          l.pairs, l.theta, G, l.krot)
        assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL


@pytest.mark.parametrize("G", GROUPS)
@pytest.mark.parametrize("N,K", [(136, 256), (328, 512)])
def test_quantize_group_sizes(G, N, K):
    lay = synth.make_layer("qg", K, N, seed=G + N + K, group_size=G)
    W, qs = synth.make_float_weight(lay)
    qw, qz = pb.quantize_w4(dev(W), dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), dev(qs), G, lay.krot)
    torch.cuda.synchronize()
    qw, qz = qw.cpu().numpy(), qz.cpu().numpy()
    assert qz.shape == (K // G, N // 8)
    assert np.all(qz.view(np.uint32) == 0x88888888)
    codes, zeros = oracle.awq_unpack(qw, qz, N, K, G)
    assert np.all(zeros == 8)
    bad, amb, tot = check_codes(codes, W, lay.channel_scales, lay.pairs, lay.theta, qs, G, lay.krot)
    assert bad == 0, (bad, amb, tot)
    assert amb <= 0.01 * tot, (amb, tot)
