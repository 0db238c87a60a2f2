"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle on
the same seeded inputs.  Sizes span several tiles and ragged tails; full-size
workloads are checked on sampled output columns."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import LIN_TOL, ROT_TOL, dev, layer_to_device, lin_err, rot_err

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


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("N,K,G,randz", [(512, 256, 128, False), (64, 1024, 128, True),
                                         (4096, 4096, 128, False), (24, 96, 32, True),
                                         (1024, 14336, 128, True)])
def test_pack_bit_exact(N, K, G, randz):
    rng = np.random.default_rng(N + K)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (N, K // G), dtype=np.uint8) if randz else np.full((N, K // G), 8, np.uint8)
    qw_ref, qz_ref = oracle.awq_pack(codes, zeros, G)
    qw, qz = pb.pack_awq(dev(codes), dev(zeros), G)
    assert np.array_equal(qw.cpu().numpy(), qw_ref)
    assert np.array_equal(qz.cpu().numpy(), qz_ref)
    c2, z2 = pb.unpack_awq(qw, qz, N, K, G)
    assert np.array_equal(c2.cpu().numpy(), codes)
    assert np.array_equal(z2.cpu().numpy(), zeros)


def test_pack_high_nibble_ignored():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (64, 256), dtype=np.uint8)
    zeros = rng.integers(0, 256, (64, 2), dtype=np.uint8)
    qw, qz = pb.pack_awq(dev(codes), dev(zeros), 128)
    ref_w, ref_z = oracle.awq_pack(codes & 15, zeros & 15, 128)
    assert np.array_equal(qw.cpu().numpy(), ref_w) and np.array_equal(qz.cpu().numpy(), ref_z)


# ------------------------------------------------------------------ rotation

ROT_CASES = [
    # (M, K, krot, use_cs, active_pairs)
    (4, 256, 8, True, None),          # config 0 shape
    (1, 4096, 8, True, 6),            # decode, 10 % active pairs
    (16, 4096, 8, True, 6),
    (37, 512, 8, True, None),         # ragged rows
    (130, 1024, 8, False, None),      # several row tiles + tail, no scaling
    (2048, 4096, 8, True, None),
    (5, 384, 1, True, None),          # krot = 1
    (9, 256, 0, True, None),          # scaling only
    (33, 256, 64, True, None),        # krot at the supported maximum
    (129, 256, 64, True, None),       # krot maximum on the tensor-memory kernel
    (65, 384, 1, False, None),        # tensor-memory kernel, krot = 1, ragged tile
    (3, 14336, 8, True, None),        # down_proj width
    (300, 512, 16, True, None),       # tensor-memory kernel, per-warp address tables at their limit
    (300, 512, 17, True, None),       # tensor-memory kernel, one shared column table
    (20000, 1024, 8, True, None),     # CTAs walk several row tiles; ragged last tile
]


@pytest.mark.parametrize("M,K,krot,use_cs,active", ROT_CASES)
def test_rotate_vs_oracle(M, K, krot, use_cs, active):
    lay = synth.make_layer("r", K, 32, seed=M * 7 + K + krot, krot=max(krot, 1), active_pairs=active,
                           n_outliers=max(1, K // 100))
    pairs, theta = lay.pairs[:krot], lay.theta[:krot]
    cs = lay.channel_scales if use_cs else None
    x = synth.make_activations(lay, M)
    ref = oracle.rotate(x, cs, pairs, theta, 128, krot=krot)
    got = pb.rotate(dev(x), dev(cs), dev(pairs) if krot else None, dev(theta) if krot else None,
                    128, krot).cpu().numpy().astype(np.float64)
    assert rot_err(got, ref) <= ROT_TOL


@pytest.mark.parametrize("M", [40, 200])   # shared-memory and tensor-memory kernels
def test_rotate_in_place_and_identity_state(M):
    lay = synth.config_layers(0)[0]
    x = synth.make_activations(lay, M)
    xt = dev(x)
    pb.rotate(xt, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), 128, out=xt)
    ref = oracle.rotate(x, lay.channel_scales, lay.pairs, lay.theta, 128)
    assert rot_err(xt.cpu().numpy().astype(np.float64), ref) <= ROT_TOL
    # identity state: zero angles, unit scales -> bit-identical copy
    got = pb.rotate(dev(x), dev(np.ones(256, np.float32)), dev(lay.pairs),
                    dev(np.zeros_like(lay.theta)), 128)
    assert np.array_equal(got.cpu().numpy(), x)


def test_rotate_krot_zero_large_batch_is_scaling_only():
    lay = synth.config_layers(0)[0]
    x = synth.make_activations(lay, 300)
    got = pb.rotate(dev(x), dev(lay.channel_scales), None, None, 128, 0).cpu().numpy()
    # the kernel's documented arithmetic: fp32 product, one round-to-nearest to fp16
    ref32 = (x.astype(np.float32) * lay.channel_scales.astype(np.float32)).astype(np.float16)
    assert np.array_equal(got, ref32)
    exact = oracle.rotate(x, lay.channel_scales, None, None, 128, krot=0)
    assert rot_err(got.astype(np.float64), exact) <= ROT_TOL


def test_rotate_empty_batch():
    lay = synth.config_layers(0)[0]
    x = torch.empty((0, 256), dtype=torch.float16, device="cuda")
    out = pb.rotate(x, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), 128)
    assert out.shape == (0, 256)


def test_rotate_pair_index_out_of_group_is_flagged_not_faulting():
    lay = synth.config_layers(0)[0]
    bad = lay.pairs.copy()
    bad[3, 10] = 300                     # masked to 300 & 127 on the device; flagged
    x = synth.make_activations(lay, 4)
    pb.rotate(dev(x), None, dev(bad), dev(lay.theta), 128)
    assert pb.device_status(clear=True) == pb.PARO_ERR_INVALID_ARG
    assert pb.device_status(clear=True) == pb.PARO_OK


# ------------------------------------------------------------------ linear

def run_linear(lay, d, x, krot=None, use_cs=True):
    krot = lay.krot if krot is None else krot
    return pb.w4_linear(dev(x), d["qweight"], d["qzeros"], d["scales"], d["bias"],
                        d["cs"] if use_cs else None, d["pairs"] if krot else None,
                        d["theta"] if krot else None, lay.group_size, krot)


def oracle_linear(lay, x, krot=None, use_cs=True):
    krot = lay.krot if krot is None else krot
    return oracle.w4_linear_from_codes(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                       lay.channel_scales if use_cs else None,
                                       lay.pairs if krot else None, lay.theta if krot else None,
                                       lay.group_size, krot)


def test_config0_tiny_layer():
    lay = synth.config_layers(0)[0]
    d = layer_to_device(lay)
    x = synth.make_activations(lay, 4)
    got = run_linear(lay, d, x).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x)
    assert lin_err(got, ref) <= LIN_TOL


LIN_SHAPES = [(K, N) for K, N in [(256, 512), (1024, 544), (512, 1024)]]
LIN_M = [1, 2, 3, 4, 7, 8, 9, 15, 16, 17, 31, 64, 65, 200]


@pytest.mark.parametrize("K,N", LIN_SHAPES)
@pytest.mark.parametrize("M", LIN_M)
def test_linear_vs_oracle(M, K, N):
    lay = synth.make_layer("l", K, N, seed=K + N, bias_std=0.01, zero_point=None,
                           n_outliers=4)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x)
    assert lin_err(got, ref) <= LIN_TOL


# rotation kernel choice at decode sizes: one warp per (group, row) up to 8
# stages and 16 rows, the shared-memory kernel beyond
@pytest.mark.parametrize("krot", [1, 8, 9, 12])
@pytest.mark.parametrize("M", [1, 3, 4, 5, 9, 16])
def test_linear_decode_rotation_paths(M, krot):
    lay = synth.make_layer("k", 1024, 512, seed=90 + krot, krot=krot, bias_std=0.01, n_outliers=4)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x)
    assert lin_err(got, ref) <= LIN_TOL


@pytest.mark.parametrize("M", [2, 5])
def test_linear_decode_scales_only(M):
    """krot = 0 with channel scales: a scaling-only pass ahead of the GEMV."""
    lay = synth.make_layer("c", 512, 1024, seed=91)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x, krot=0).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x, krot=0)
    assert lin_err(got, ref) <= LIN_TOL


@pytest.mark.parametrize("M", [1, 16, 100])
def test_linear_plain_awq_baseline(M):
    """krot = 0 and no channel scales: a plain AWQ W4 linear."""
    lay = synth.make_layer("p", 512, 1024, seed=77, zero_point=None)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x, krot=0, use_cs=False).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x, krot=0, use_cs=False)
    assert lin_err(got, ref) <= LIN_TOL


def test_linear_identity_state_equals_plain():
    lay = synth.make_layer("i", 512, 512, seed=78)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, 8)
    d_id = dict(d)
    d_id["theta"] = dev(np.zeros_like(lay.theta))
    d_id["cs"] = dev(np.ones(512, np.float32))
    a = run_linear(lay, d_id, x).cpu().numpy()
    b = run_linear(lay, d, x, krot=0, use_cs=False).cpu().numpy()
    assert np.array_equal(a, b)


def test_linear_deterministic_and_workspace_reuse():
    lay = synth.make_layer("d", 4096, 1024, seed=79)
    d = layer_to_device(lay)
    ws = torch.empty(pb.w4_linear_workspace_size(16, 4096, 1024), dtype=torch.uint8, device="cuda")
    x = dev(synth.make_activations(lay, 16))
    outs = [pb.w4_linear(x, d["qweight"], d["qzeros"], d["scales"], None, d["cs"], d["pairs"],
                         d["theta"], 128, 8, workspace=ws).cpu().numpy() for _ in range(3)]
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])


def test_linear_empty_batch():
    lay = synth.config_layers(0)[0]
    d = layer_to_device(lay)
    out = run_linear(lay, d, np.zeros((0, 256), np.float16))
    assert out.shape == (0, 512)


# ------------------------------------------------------------------ full-size, sampled columns

def sampled_check(lay, M, ncols=96, seed=0):
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x).cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(seed)
    cols = np.unique(np.concatenate([[0, lay.N - 1], rng.choice(lay.N, ncols, replace=False)]))
    ref = oracle.w4_linear_columns(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                   lay.channel_scales, lay.pairs, lay.theta, lay.group_size,
                                   lay.krot, cols)
    err = lin_err(got[:, cols], ref)
    assert err <= LIN_TOL, (lay.name, M, err)
    return err


@pytest.mark.parametrize("M", synth.CONFIG_M[1])
def test_config1_q_proj_full_size(M):
    sampled_check(synth.config_layers(1)[0], M)


@pytest.mark.parametrize("idx", [0, 2])
@pytest.mark.parametrize("M", synth.CONFIG_M[2])
def test_config2_mlp_decode_full_size(idx, M):
    lay = synth.config_layers(2)[idx]
    sampled_check(lay, M)


@pytest.mark.parametrize("M", synth.CONFIG_M[3])
def test_config3_prefill_full_size(M):
    sampled_check(synth.config_layers(3)[0], M, ncols=48)


def test_config4_layer_set_decode_and_prefill():
    for lay in synth.config_layers(4):
        for M in synth.CONFIG_M[4]:
            sampled_check(lay, M, ncols=32)


# Prefill GEMM grids of more 256 x 256 tiles than SMs (several waves), full
# outputs against the oracle; K = 128 gives two k-blocks per tile (fewer than
# the dequantised-weight ring holds).
@pytest.mark.parametrize("M,K,N", [(600, 256, 14336), (1024, 128, 14336), (1300, 256, 14336)])
def test_linear_prefill_several_tiles_per_cta(M, K, N):
    lay = synth.make_layer("s", K, N, seed=M + K, bias_std=0.01, zero_point=None, n_outliers=2)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    got = run_linear(lay, d, x).cpu().numpy().astype(np.float64)
    ref = oracle_linear(lay, x)
    assert lin_err(got, ref) <= LIN_TOL
