"""GPU parity of the weight-side quantiser against the float64 oracle: W_r = W D R,
four-bit symmetric codes, AWQ packing, on both kernels: stage by stage
(paro_quantize_w4, "pairs") and as one matrix per group on the tensor cores
(paro_quantize_w4_tc, "tensor"; N % 32 == 0).  Codes are compared element by
element (unique where the exact quotient is clear of a rounding boundary, see
tests/gpu_util.check_codes); qzeros bit-exact.  Sizes span several 128-row
tiles with a ragged tail; the full-size case is checked on sampled rows."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import check_codes, dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_w4_weight_b200 as pb  # noqa: E402


@pytest.fixture(autouse=True)
def _status_clean():
    assert pb.device_status(clear=True) == pb.PARO_OK
    yield
    assert pb.device_status(clear=True) == pb.PARO_OK


def run_quant(lay, W, qs, krot=None, use_cs=True, method="pairs"):
    krot = lay.krot if krot is None else krot
    qw, qz = pb.quantize_w4(dev(W), dev(lay.channel_scales) if use_cs else None,
                            dev(lay.pairs) if krot else None, dev(lay.theta) if krot else None,
                            dev(qs), lay.group_size, krot, method=method)
    torch.cuda.synchronize()
    return qw.cpu().numpy(), qz.cpu().numpy()


def unpack(qw, qz, N, K, G):
    return oracle.awq_unpack(qw, qz, N, K, G)


def assert_parity(lay, W, qs, krot, use_cs, qw, qz, rows=None):
    N, K, G = lay.N, lay.K, lay.group_size
    codes, zeros = unpack(qw, qz, N, K, G)
    assert np.all(qz.view(np.uint32) == 0x88888888)
    assert np.all(zeros == 8)
    sel = codes if rows is None else codes[rows]
    bad, amb, tot = check_codes(sel, W, lay.channel_scales if use_cs else None,
                                lay.pairs if krot else None, lay.theta if krot else None,
                                qs, G, krot, rows=rows)
    assert bad == 0, (bad, amb, tot)
    assert amb <= 0.01 * tot, (amb, tot)      # the rule leaves almost every code unique
    return codes


@pytest.mark.parametrize("N,K,krot", [(328, 512, 8), (8, 256, 8), (136, 384, 3), (256, 256, 1),
                                      (384, 256, 17), (200, 1024, 8)])
def test_quantize_vs_oracle(N, K, krot):
    lay = synth.make_layer("q", K, N, seed=N + K + krot, krot=krot)
    W, qs = synth.make_float_weight(lay)
    qw, qz = run_quant(lay, W, qs)
    codes = assert_parity(lay, W, qs, krot, True, qw, qz)
    assert np.any(codes == 0) or np.any(codes == 15)   # the clamp is exercised


@pytest.mark.parametrize("N,K,krot,G", [(352, 512, 8, 128), (32, 256, 1, 128), (160, 384, 3, 128),
                                        (256, 256, 17, 128), (384, 1024, 8, 128), (352, 512, 8, 32),
                                        (160, 256, 4, 16), (256, 512, 8, 64)])
def test_quantize_tensor_cores_vs_oracle(N, K, krot, G):
    lay = synth.make_layer("qt", K, N, seed=N + K + krot + G, krot=krot, group_size=G)
    W, qs = synth.make_float_weight(lay)
    qw, qz = run_quant(lay, W, qs, method="tensor")
    codes = assert_parity(lay, W, qs, krot, True, qw, qz)
    assert np.any(codes == 0) or np.any(codes == 15)   # the clamp is exercised


def test_quantize_tensor_cores_and_pairs_agree_where_codes_are_unique():
    """Both kernels against each other: outside the ambiguity margin of the
    fp32 transform every code must be the same."""
    lay = synth.make_layer("qa", 1024, 512, seed=77)
    W, qs = synth.make_float_weight(lay)
    qt, zt = run_quant(lay, W, qs, method="tensor")
    qp, zp = run_quant(lay, W, qs, method="pairs")
    assert np.array_equal(zt, zp)
    ct, _ = unpack(qt, zt, lay.N, lay.K, 128)
    cp, _ = unpack(qp, zp, lay.N, lay.K, 128)
    diff = ct != cp
    assert diff.mean() <= 0.005, diff.mean()
    assert np.all(np.abs(ct.astype(int) - cp.astype(int)) <= 1)


@pytest.mark.parametrize("method,N", [("pairs", 264), ("tensor", 256)])
def test_quantize_scaling_only_and_plain(method, N):
    """krot = 0 with channel scales (W * D only), and with neither (plain symmetric
    quantisation of W): no ambiguity beyond the final multiply."""
    lay = synth.make_layer("p", 512, N, seed=5)
    W, qs = synth.make_float_weight(lay)
    for use_cs in (True, False):
        qw, qz = run_quant(lay, W, qs, krot=0, use_cs=use_cs, method=method)
        assert_parity(lay, W, qs, 0, use_cs, qw, qz)


@pytest.mark.parametrize("method", ["pairs", "tensor"])
def test_quantize_identity_state_exact_levels(method):
    """Zero angles, unit channel scales and weights on exact levels: the codes
    are known in closed form (every quotient is an integer or a tie)."""
    K, N, G = 256, 64, 128
    lay = synth.make_layer("e", K, N, seed=9)
    rng = np.random.default_rng(3)
    q = rng.integers(-10, 10, size=(N, K))                 # includes values past the clamp
    s = np.float16(0.125)
    W = (q * float(s)).astype(np.float16)
    W[0, :4] = np.array([0.5, 1.5, -0.5, -2.5]) * float(s)  # ties: to even
    qs = np.full((K // G, N), s, np.float16)
    qw, qz = pb.quantize_w4(dev(W), dev(np.ones(K, np.float32)), dev(lay.pairs),
                            dev(np.zeros_like(lay.theta)), dev(qs), G, lay.krot, method=method)
    torch.cuda.synchronize()
    codes, _ = unpack(qw.cpu().numpy(), qz.cpu().numpy(), N, K, G)
    want = np.clip(q, -8, 7) + 8
    want[0, :4] = np.array([0, 2, 0, -2]) + 8
    assert np.array_equal(codes, want.astype(np.uint8))


@pytest.mark.parametrize("method", ["pairs", "tensor"])
def test_quantize_then_linear_matches_oracle_replay(method):
    """The packed output serves paro_w4_linear directly: Y from the GPU-quantised
    layer equals the oracle's X_r Q(W_r)^T + b with the same codes."""
    lay = synth.make_layer("r", 1024, 512, seed=13, bias_std=0.01)
    W, qs = synth.make_float_weight(lay)
    qw, qz = pb.quantize_w4(dev(W), dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta),
                            dev(qs), 128, lay.krot, method=method)
    x = synth.make_activations(lay, 5)
    y = pb.w4_linear(dev(x), qw, qz, dev(qs), dev(lay.bias), dev(lay.channel_scales),
                     dev(lay.pairs), dev(lay.theta), 128, lay.krot)
    codes, zeros = unpack(qw.cpu().numpy(), qz.cpu().numpy(), lay.N, lay.K, 128)
    ref = oracle.w4_linear_from_codes(x, codes, zeros, qs, lay.bias, lay.channel_scales, lay.pairs,
                                      lay.theta, 128, lay.krot)
    got = y.cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(got - ref)) <= 2e-2 * rms


def test_quantize_empty_and_deterministic():
    lay = synth.make_layer("d", 256, 64, seed=4)
    W, qs = synth.make_float_weight(lay)
    a = run_quant(lay, W, qs)
    b = run_quant(lay, W, qs)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert pb.paro_quantize_w4(None, None, None, None, None, None, None, 0, 256, 128, 8, None) == pb.PARO_OK
    c = run_quant(lay, W, qs, method="tensor")
    d = run_quant(lay, W, qs, method="tensor")
    assert np.array_equal(c[0], d[0]) and np.array_equal(c[1], d[1])
    assert pb.paro_quantize_w4_tc(None, None, None, None, None, None, None, 0, 256, 128, 8, None, 0,
                                  None) == pb.PARO_OK


@pytest.mark.parametrize("method", ["pairs", "tensor"])
def test_quantize_full_size_gate_proj_sampled_rows(method):
    """Llama-3-8B gate_proj (14336 x 4096), all rows on the GPU in one call;
    96 sampled rows (every tile position class) checked against the oracle."""
    lay = synth.make_layer("gate_proj", 4096, 14336, seed=2000, n_outliers=41)
    W, qs = synth.make_float_weight(lay)
    qw, qz = run_quant(lay, W, qs, method=method)
    rng = np.random.default_rng(1)
    rows = np.sort(np.concatenate([rng.choice(lay.N, 90, replace=False), [0, 1, 127, 128, lay.N - 2, lay.N - 1]]))
    assert_parity(lay, W, qs, lay.krot, True, qw, qz, rows=rows)
