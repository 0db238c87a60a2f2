"""GPU parity of grouped decoder-layer calls (paro_w4_linear_group): several
linears over the same x, each with its own weights and rotation tables, against
the float64 oracle member by member, and against separate paro_w4_linear calls."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import LIN_TOL, dev, layer_to_device, lin_err

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


def member(lay, d, krot=None, use_cs=True):
    krot = lay.krot if krot is None else krot
    return dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=d["bias"],
                channel_scales=d["cs"] if use_cs else None, pairs=d["pairs"] if krot else None,
                theta=d["theta"] if krot else None, krot=krot)


def oracle_cols(lay, x, cols, krot=None, use_cs=True):
    krot = lay.krot if krot is None else krot
    return oracle.w4_linear_columns(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                    lay.channel_scales if use_cs else None, lay.pairs if krot else None,
                                    lay.theta if krot else None, lay.group_size, krot, cols)


def check_group(lays, specs, M, ncols=256):
    """specs: per member (krot or None, use_cs); returns the grouped outputs."""
    ds = [layer_to_device(l) for l in lays]
    x = synth.make_activations(lays[0], M)
    mem = [member(l, d, k, c) for l, d, (k, c) in zip(lays, ds, specs)]
    outs = pb.w4_linear_group(dev(x), mem)
    torch.cuda.synchronize()
    rng = np.random.default_rng(M)
    for lay, (k, c), y, m in zip(lays, specs, outs, mem):
        cols = np.sort(rng.choice(lay.N, min(ncols, lay.N), replace=False))
        ref = oracle_cols(lay, x, cols, k, c)
        got = y.cpu().numpy().astype(np.float64)[:, cols]
        assert lin_err(got, ref) <= LIN_TOL, lay.name
        # the same member as a separate call: equal up to summation order
        single = pb.w4_linear(dev(x), m["qweight"], m["qzeros"], m["scales"], m["bias"], m["channel_scales"],
                              m["pairs"], m["theta"], 128, m["krot"])
        a, b = y.float(), single.float()
        rms = float(b.pow(2).mean().sqrt())
        assert float((a - b).abs().max()) <= 1e-2 * rms, lay.name
    return outs


def qkv(seed=0, krot=8):
    return [synth.make_layer(n, 4096, N, seed + i, krot=krot, bias_std=0.01, n_outliers=41)
            for i, (n, N) in enumerate([("q", 4096), ("k", 1024), ("v", 1024)])]


@pytest.mark.parametrize("M", [1, 4, 9, 16])
def test_group_qkv_decode(M):
    check_group(qkv(10), [(None, True)] * 3, M)


def test_group_mixed_members():
    """A plain AWQ member (no rotation), a member past the warp-per-row
    rotation's stage count, and a rotated one."""
    lays = [synth.make_layer("a", 1024, 512, 21, krot=8), synth.make_layer("b", 1024, 256, 22, krot=12),
            synth.make_layer("c", 1024, 768, 23, krot=8, bias_std=0.01)]
    check_group(lays, [(0, False), (None, True), (None, True)], 4)


@pytest.mark.parametrize("M", [3, 64])
def test_group_small_shapes_and_prefill_sizes(M):
    lays = [synth.make_layer("s%d" % i, 512, N, 30 + i, krot=8) for i, N in enumerate([256, 512, 768, 32])]
    check_group(lays, [(None, True)] * 4, M)


@pytest.mark.parametrize("M", [1, 4, 8])
def test_group_gate_up_decode(M):
    """The pair runs as one GEMV launch: a 2-stage ring puts two CTAs on an
    SM (at half the split up to 4 tokens, at the same split at 8)."""
    lays = [synth.make_layer(n, 4096, 14336, 40 + i, n_outliers=41) for i, n in enumerate(["gate", "up"])]
    check_group(lays, [(None, True)] * 2, M, ncols=128)
    assert pb.w4_linear_group_launches(M, 4096, [dict(N=14336)] * 2) == 2


def test_group_of_one_equals_single_call():
    lay = synth.make_layer("o", 4096, 4096, 50)
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, 1))
    m = member(lay, d)
    (y,) = pb.w4_linear_group(x, [m])
    y1 = pb.w4_linear(x, m["qweight"], m["qzeros"], m["scales"], m["bias"], m["channel_scales"], m["pairs"],
                      m["theta"], 128, m["krot"])
    assert torch.equal(y, y1)


def test_group_deterministic_and_empty():
    lays = qkv(60)
    ds = [layer_to_device(l) for l in lays]
    x = dev(synth.make_activations(lays[0], 2))
    mem = [member(l, d) for l, d in zip(lays, ds)]
    a = pb.w4_linear_group(x, mem)
    b = pb.w4_linear_group(x, mem)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    e = pb.w4_linear_group(dev(synth.make_activations(lays[0], 1))[:0], mem)
    assert all(t.shape[0] == 0 for t in e)


@pytest.mark.parametrize("M", [65, 300, 1000])
def test_group_prefill_batched_rotation(M):
    """Above 64 rows the rotating members share one R' build and one X R'
    launch (x read once per tile for all of them): a plain member, krot 8,
    krot 17 and scales only, each against the oracle and the separate call."""
    lays = [synth.make_layer("p%d" % i, 1024, N, 60 + i, krot=k, bias_std=0.01, n_outliers=10)
            for i, (N, k) in enumerate([(512, 8), (256, 8), (768, 17), (1024, 8)])]
    check_group(lays, [(0, False), (None, True), (None, True), (0, True)], M)


@pytest.mark.parametrize("M", [1, 40, 300])
def test_group_experts_sharing_one_rotation(M):
    """Experts with their own weights and one shared rotation (the same
    channel-scale, pair and angle tensors): x is rotated once and every expert
    reads that X_r; each output against the oracle and the separate call."""
    lays = [synth.make_layer("e%d" % i, 1024, 512, 70 + i, bias_std=0.01, n_outliers=10) for i in range(3)]
    for lay in lays[1:]:
        lay.pairs, lay.theta, lay.channel_scales = lays[0].pairs, lays[0].theta, lays[0].channel_scales
    ds = [layer_to_device(l) for l in lays]
    for d in ds[1:]:
        d["pairs"], d["theta"], d["cs"] = ds[0]["pairs"], ds[0]["theta"], ds[0]["cs"]
    x = synth.make_activations(lays[0], M)
    mem = [member(l, d) for l, d in zip(lays, ds)]
    outs = pb.w4_linear_group(dev(x), mem)
    torch.cuda.synchronize()
    specs = [dict(N=512), dict(N=512, same_rotation_as=0), dict(N=512, same_rotation_as=0)]
    # never more launches than three separate rotations (the batched prefill
    # rotation is two launches either way)
    assert pb.w4_linear_group_launches(M, 1024, specs) <= pb.w4_linear_group_launches(M, 1024, [dict(N=512)] * 3)
    rng = np.random.default_rng(M)
    for lay, y, m in zip(lays, outs, mem):
        cols = np.sort(rng.choice(lay.N, 128, replace=False))
        got = y.cpu().numpy().astype(np.float64)[:, cols]
        assert lin_err(got, oracle_cols(lay, x, cols)) <= LIN_TOL, lay.name
        single = pb.w4_linear(dev(x), m["qweight"], m["qzeros"], m["scales"], m["bias"], m["channel_scales"],
                              m["pairs"], m["theta"], 128, m["krot"])
        a, b = y.float(), single.float()
        assert float((a - b).abs().max()) <= 1e-2 * float(b.pow(2).mean().sqrt()), lay.name
