"""GPU parity for bf16 activations (the *_dt entry points with PARO_DTYPE_BF16):
every kernel family against the float64 oracle, fed the exact bf16 values the
GPU sees.

Tolerances, from the arithmetic (bf16 keeps 8 significant bits, so one
round-to-nearest is off by at most 2^-8 of the value):
  * rotated activations: the only rounding is the final one to bf16, so
    |d_i| <= 2^-8 * |ref_i| plus the fp32 path (below 1e-5 of the row rms);
    checked as rot_err <= 5e-3.
  * linear outputs: X_r and, on the prefill path, each dequantised weight
    (q - z) * s are rounded once to bf16 (independent relative errors of at
    most 2^-8, i.e. a standard deviation of at most 2^-8 / sqrt(3) each), and Y
    is rounded once at the end.  The first two give an output error with a
    standard deviation of about 3.3e-3 of rms(Y); the last is at most 2^-8 of
    |Y_i|.  Checked as |d_i| <= 3e-2 * rms(Y) + 2^-8 * |Y_i| (about nine
    standard deviations: a wrong operand type or scale read is off by O(1)).
  * weight codes: as for fp16 (``check_codes``): the codes depend only on the
    values of w and the scales, which both types carry exactly.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import check_codes, dev, rot_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_w4_weight_b200 as pb  # noqa: E402
from rotation_w4_weight_b200 import _lib  # noqa: E402

ROT_TOL_BF16 = 5e-3
LIN_ABS_BF16 = 3e-2
LIN_REL_BF16 = 2.0 ** -8


@pytest.fixture(autouse=True)
def _status_clean():
    assert pb.device_status(clear=True) == pb.PARO_OK
    yield
    assert pb.device_status(clear=True) == pb.PARO_OK


def bf(a):
    """(bf16 CUDA tensor, float64 array of its exact values) for a float array."""
    if a is None:
        return None, None
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float32))).to(torch.bfloat16)
    return t.cuda(), t.float().numpy().astype(np.float64)


def lin_ok(got, ref):
    """Largest excess over the bound |d_i| <= LIN_ABS_BF16 * rms + LIN_REL_BF16 * |ref_i| (<= 0 passes)."""
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = LIN_ABS_BF16 * rms + LIN_REL_BF16 * np.abs(ref)
    return float(np.max(np.abs(got - ref) - bound))


def to64(t):
    return t.float().cpu().numpy().astype(np.float64)


def device_layer(lay):
    """Packed weights plus bf16 scales/bias, and the exact values of those for the oracle."""
    qweight, qzeros = pb.pack_awq(dev(lay.codes), dev(lay.zero_codes), lay.group_size)
    s_t, s_v = bf(lay.scales)
    b_t, b_v = bf(lay.bias)
    return dict(qweight=qweight, qzeros=qzeros, scales=s_t, bias=b_t, cs=dev(lay.channel_scales),
                pairs=dev(lay.pairs), theta=dev(lay.theta)), s_v, b_v


# (M, K, krot, G): warp-per-row decode kernel, 4-row tile (krot > 8), 64-row
# shared-memory tile, tensor-memory kernel (M > 64), and a smaller group
ROT_CASES = [(1, 512, 8, 128), (7, 384, 12, 128), (37, 256, 8, 128), (300, 512, 8, 128),
             (129, 256, 17, 128), (5, 256, 8, 32), (200, 256, 8, 64)]


@pytest.mark.parametrize("M,K,krot,G", ROT_CASES)
def test_rotate_bf16(M, K, krot, G):
    lay = synth.make_layer("rb", K, 32, seed=M + 3 * krot + G, group_size=G, krot=krot, n_outliers=max(1, K // 100))
    x_t, x_v = bf(synth.make_activations(lay, M).astype(np.float32))
    got = pb.rotate(x_t, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), G, krot)
    assert got.dtype == torch.bfloat16
    ref = oracle.rotate(x_v, lay.channel_scales, lay.pairs, lay.theta, G)
    assert rot_err(to64(got), ref) <= ROT_TOL_BF16


def test_rotate_bf16_beyond_fp16_range():
    """Values past the fp16 range (|x| up to 3e5) rotate in bf16."""
    K, M = 256, 3
    lay = synth.make_layer("rr", K, 32, seed=91, krot=8)
    x = synth.make_activations(lay, M).astype(np.float32) * 1.0e4
    x_t, x_v = bf(x)
    assert np.max(np.abs(x_v)) > 65504
    got = pb.rotate(x_t, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), 128, 8)
    ref = oracle.rotate(x_v, lay.channel_scales, lay.pairs, lay.theta, 128)
    assert rot_err(to64(got), ref) <= ROT_TOL_BF16


@pytest.mark.parametrize("G", [128, 32])
@pytest.mark.parametrize("M", [1, 4, 16, 40, 300])   # GEMV, GEMV (2 token tiles), GEMM, GEMM + tensor-core rotation
def test_linear_bf16(G, M):
    K, N = 512, 384
    lay = synth.make_layer("lb", K, N, seed=G + 11 * M, group_size=G, bias_std=0.01, zero_point=None)
    d, s_v, b_v = device_layer(lay)
    x_t, x_v = bf(synth.make_activations(lay, M).astype(np.float32))
    y = pb.w4_linear(x_t, d["qweight"], d["qzeros"], d["scales"], d["bias"], d["cs"], d["pairs"], d["theta"],
                     G, lay.krot)
    assert y.dtype == torch.bfloat16
    ref = oracle.w4_linear_from_codes(x_v, lay.codes, lay.zero_codes, s_v, b_v, lay.channel_scales,
                                      lay.pairs, lay.theta, G, lay.krot)
    assert lin_ok(to64(y), ref) <= 0


@pytest.mark.parametrize("M", [3, 130])
def test_linear_bf16_plain_awq(M):
    """No rotation and no channel scales: the bf16 group-wise dequantisation alone."""
    K, N = 1024, 256
    lay = synth.make_layer("pb", K, N, seed=M + 1, zero_point=None)
    d, s_v, _ = device_layer(lay)
    x_t, x_v = bf(synth.make_activations(lay, M).astype(np.float32))
    y = pb.w4_linear(x_t, d["qweight"], d["qzeros"], d["scales"], None, None, None, None, 128, 0)
    ref = oracle.w4_linear_from_codes(x_v, lay.codes, lay.zero_codes, s_v, None, None, None, None, 128, 0)
    assert lin_ok(to64(y), ref) <= 0


@pytest.mark.parametrize("M", [1, 96])
def test_group_call_bf16(M):
    K = 512
    lays = [synth.make_layer(f"gb{i}", K, n, seed=5 + 13 * i + M, zero_point=None, bias_std=0.01)
            for i, n in enumerate((256, 128, 128))]
    devs = [device_layer(l) for l in lays]
    x_t, x_v = bf(synth.make_activations(lays[0], M).astype(np.float32))
    members = [dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=d["bias"],
                    channel_scales=d["cs"], pairs=d["pairs"], theta=d["theta"], krot=l.krot)
               for l, (d, _, _) in zip(lays, devs)]
    ys = pb.w4_linear_group(x_t, members, 128)
    for l, (_, s_v, b_v), y in zip(lays, devs, ys):
        assert y.dtype == torch.bfloat16
        ref = oracle.w4_linear_from_codes(x_v, l.codes, l.zero_codes, s_v, b_v, l.channel_scales,
                                          l.pairs, l.theta, 128, l.krot)
        assert lin_ok(to64(y), ref) <= 0


def test_group_gate_up_decode_bf16():
    """Gate/up-shaped members at one token: the one-launch plan on the 2-stage
    ring with bf16 operands; sampled columns against the oracle."""
    K, N, M = 4096, 14336, 1
    lays = [synth.make_layer(n, K, N, seed=60 + i, zero_point=None, bias_std=0.01, n_outliers=41)
            for i, n in enumerate(["gate", "up"])]
    devs = [device_layer(l) for l in lays]
    x_t, x_v = bf(synth.make_activations(lays[0], M).astype(np.float32))
    members = [dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=d["bias"],
                    channel_scales=d["cs"], pairs=d["pairs"], theta=d["theta"], krot=l.krot)
               for l, (d, _, _) in zip(lays, devs)]
    assert pb.w4_linear_group_launches(M, K, [dict(N=N)] * 2) == 2
    ys = pb.w4_linear_group(x_t, members, 128)
    cols = np.sort(np.random.default_rng(7).choice(N, 128, replace=False))
    for l, (_, s_v, b_v), y in zip(lays, devs, ys):
        assert y.dtype == torch.bfloat16
        ref = oracle.w4_linear_columns(x_v, l.codes, l.zero_codes, s_v, b_v, l.channel_scales, l.pairs,
                                       l.theta, 128, l.krot, cols)
        assert lin_ok(to64(y)[:, cols], ref) <= 0


def test_noalloc_bf16_matches_workspace_call():
    K, N, M = 512, 256, 5
    lay = synth.make_layer("nb", K, N, seed=77, zero_point=None)
    d, _, _ = device_layer(lay)
    x_t, _ = bf(synth.make_activations(lay, M).astype(np.float32))
    y_ws = pb.w4_linear(x_t, d["qweight"], d["qzeros"], d["scales"], None, d["cs"], d["pairs"], d["theta"],
                        128, lay.krot)
    y_na = torch.empty_like(y_ws)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib.paro_w4_linear_noalloc_dt(p(x_t), p(y_na), M, K, N, p(d["qweight"]), p(d["qzeros"]), p(d["scales"]),
                                        None, p(d["cs"]), p(d["pairs"]), p(d["theta"]), 128, lay.krot,
                                        _lib.PARO_DTYPE_BF16,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pb.PARO_OK
    torch.cuda.synchronize()
    assert torch.equal(y_ws, y_na)


@pytest.mark.parametrize("G", [128, 64])
@pytest.mark.parametrize("N,K", [(136, 256), (328, 512)])
def test_quantize_bf16(G, N, K):
    lay = synth.make_layer("qb", K, N, seed=G + N + 3 * K, group_size=G)
    W, qs = synth.make_float_weight(lay)
    w_t, w_v = bf(W.astype(np.float32))
    s_t, s_v = bf(qs.astype(np.float32))
    qw, qz = pb.quantize_w4(w_t, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), s_t, G, lay.krot)
    torch.cuda.synchronize()
    qw, qz = qw.cpu().numpy(), qz.cpu().numpy()
    assert np.all(qz.view(np.uint32) == 0x88888888)
    codes, zeros = oracle.awq_unpack(qw, qz, N, K, G)
    assert np.all(zeros == 8)
    bad, amb, tot = check_codes(codes, w_v, lay.channel_scales, lay.pairs, lay.theta, s_v, G, lay.krot)
    assert bad == 0, (bad, amb, tot)
    assert amb <= 0.01 * tot, (amb, tot)


def test_bf16_and_fp16_agree_on_exactly_representable_inputs():
    """Inputs whose values are exact in both types (small integers times powers
    of two) and no rotation: the two types read the same numbers, so the fp32
    sums agree and the outputs differ only by the final rounding."""
    K, N, M = 256, 128, 2
    lay = synth.make_layer("eb", K, N, seed=3, zero_point=None, krot=0)
    rng = np.random.default_rng(4)
    x = rng.integers(-8, 8, size=(M, K)).astype(np.float32) * 0.25
    sc = (rng.integers(1, 8, size=lay.scales.shape).astype(np.float32) * 2.0 ** -6)
    qweight, qzeros = pb.pack_awq(dev(lay.codes), dev(lay.zero_codes), 128)
    y16 = pb.w4_linear(dev(x.astype(np.float16)), qweight, qzeros, dev(sc.astype(np.float16)), None, None, None,
                       None, 128, 0)
    y_b = pb.w4_linear(bf(x)[0], qweight, qzeros, bf(sc)[0], None, None, None, None, 128, 0)
    a, b = to64(y16), to64(y_b)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.abs(a) + 1e-6)
