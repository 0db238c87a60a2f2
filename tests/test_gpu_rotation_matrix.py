"""GPU parity of the prepared R' (paro_rotation_matrix_prepare) and of the
calls that use it.

R' = diag(cs) G_0 ... G_{krot-1} per 128-channel tile.  The prepared parts
come from the same build kernel as the per-call build, so a call above 64
rows with them gives X_r and Y equal, bit for bit, to the call without them;
Y is also checked against the float64 oracle like every linear, and the
parts themselves against the oracle's rotation of the basis vectors."""
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


def rmat_of(lay, d, dtype=torch.float16):
    return pb.rotation_matrix(d["cs"], d["pairs"], d["theta"], lay.K, lay.group_size, lay.krot, dtype)


@pytest.mark.parametrize("G,krot,dtype", [(128, 8, torch.float16), (32, 3, torch.float16),
                                          (128, 8, torch.bfloat16), (64, 0, torch.float16)])
def test_prepared_rmat_is_the_rotation_of_the_basis(G, krot, dtype):
    """Row k of tile g's R' is basis vector e_k scaled and rotated; the parts
    store R' transposed (row g*128 + n holds output channel n of every basis
    row, the K-major B operand of X R').  hi + lo against the oracle's
    rotation of the identity (to the parts' precision)."""
    K = 256
    lay = synth.make_layer("rm", K, 32, seed=G + krot, group_size=G, krot=krot)
    d = layer_to_device(lay)
    r = rmat_of(lay, d, dtype).view(dtype).view(2, K, 128).float().cpu().numpy().astype(np.float64)
    R = r[0] + r[1]
    for g in range(K // 128):
        basis = np.zeros((128, K))
        basis[:, g * 128:(g + 1) * 128] = np.eye(128)
        ref = oracle.rotate(basis, lay.channel_scales, lay.pairs, lay.theta, G)[:, g * 128:(g + 1) * 128]
        # the parts keep about 22 (fp16) / 16 (bf16) bits; the fp32 build adds
        # the hardware sin/cos error (about 2^-21 per angle) over krot stages
        tol = 2e-5 if dtype == torch.float16 else 1e-4
        assert np.max(np.abs(R[g * 128:(g + 1) * 128].T - ref)) <= tol * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("M", [65, 300])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prefill_with_prepared_rmat(M, dtype):
    K, N = 1024, 512
    lay = synth.make_layer("pr", K, N, seed=M, zero_point=None, bias_std=0.01)
    d = layer_to_device(lay)
    R = rmat_of(lay, d, dtype)
    x = torch.from_numpy(synth.make_activations(lay, M).astype(np.float32)).to(dtype).cuda()
    scales = torch.from_numpy(lay.scales.astype(np.float32)).to(dtype).cuda()
    bias = torch.from_numpy(lay.bias.astype(np.float32)).to(dtype).cuda()
    args = (x, d["qweight"], d["qzeros"], scales, bias, d["cs"], d["pairs"], d["theta"], 128, lay.krot)
    ws = torch.empty(pb.w4_linear_workspace_size(M, K, N, 128), dtype=torch.uint8, device="cuda")
    y = pb.w4_linear(*args, workspace=ws, rmat=R)
    torch.cuda.synchronize()
    xr_ws = ws[: M * K * 2].clone()
    ws0 = torch.empty_like(ws)
    y0 = pb.w4_linear(*args, workspace=ws0)
    torch.cuda.synchronize()
    assert torch.equal(xr_ws, ws0[: M * K * 2])
    assert torch.equal(y, y0)
    if dtype == torch.float16:
        ref = oracle.w4_linear_from_codes(x.cpu().numpy(), lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                          lay.channel_scales, lay.pairs, lay.theta, 128, lay.krot)
        assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL


@pytest.mark.parametrize("M", [96, 4096])
def test_group_prefill_with_prepared_rmat(M):
    """Grouped prefill: members with a prepared R', one without (it is built
    in the call), one sharing the first member's rotation, one not rotating."""
    K = 1024
    lays = [synth.make_layer(f"gr{i}", K, n, seed=90 + i + M, zero_point=None, bias_std=0.01)
            for i, n in enumerate((512, 256, 256, 256))]
    ds = [layer_to_device(l) for l in lays]
    Rs = [rmat_of(l, d) for l, d in zip(lays, ds)]
    x = synth.make_activations(lays[0], M)
    members, plain, refs = [], [], []
    for i, (l, d) in enumerate(zip(lays, ds)):
        src = 0 if i == 2 else i
        sl, sd = lays[src], ds[src]
        rot = i != 3
        m = dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=d["bias"],
                 channel_scales=sd["cs"] if rot else None, pairs=sd["pairs"] if rot else None,
                 theta=sd["theta"] if rot else None, krot=sl.krot if rot else 0)
        plain.append(m)
        members.append(dict(m, rmat=Rs[src]) if rot and i != 1 else m)
        refs.append(None if M > 1024 else oracle.w4_linear_from_codes(
            x, l.codes, l.zero_codes, l.scales, l.bias, sl.channel_scales if rot else None,
            sl.pairs if rot else None, sl.theta if rot else None, 128, sl.krot if rot else 0))
    ys = pb.w4_linear_group(dev(x), members, 128)
    y0 = pb.w4_linear_group(dev(x), plain, 128)
    for y, yp, ref in zip(ys, y0, refs):
        assert torch.equal(y, yp)
        if ref is not None:
            assert lin_err(y.cpu().numpy().astype(np.float64), ref) <= LIN_TOL


def test_decode_ignores_rmat():
    """Up to 64 rows the stages run pair by pair; a prepared R' changes nothing."""
    K, N, M = 512, 256, 3
    lay = synth.make_layer("dr", K, N, seed=5)
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, M))
    args = (x, d["qweight"], d["qzeros"], d["scales"], None, d["cs"], d["pairs"], d["theta"], 128, lay.krot)
    assert torch.equal(pb.w4_linear(*args, rmat=rmat_of(lay, d)), pb.w4_linear(*args))


def test_prepare_flags_pair_index_outside_group():
    """An index past the group is masked into it (no access leaves the tile)
    and flagged in the status word, as in the per-call build."""
    K = 256
    lay = synth.make_layer("fx", K, 32, seed=9)
    d = layer_to_device(lay)
    bad = lay.pairs.copy()
    bad[0, 5] = 200
    r = pb.rotation_matrix(d["cs"], dev(bad), d["theta"], K, 128, lay.krot)
    assert r.numel() == K * 128 * 4
    assert pb.device_status(clear=True) == pb.PARO_ERR_INVALID_ARG


@pytest.mark.parametrize("M", [1, 65, 300])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_rotate_with_prepared_rmat(M, dtype):
    """paro_rotate_rmat: X_r = x R' on the tensor cores, the rotation of a
    linear call above 64 rows (bit for bit), within the rotation tolerance of
    the oracle."""
    K, N = 512, 256
    lay = synth.make_layer("rr", K, N, seed=M + 3)
    d = layer_to_device(lay)
    R = rmat_of(lay, d, dtype)
    x = torch.from_numpy(synth.make_activations(lay, M).astype(np.float32)).to(dtype).cuda()
    xr = pb.rotate(x, None, None, None, 128, 0, rmat=R)
    if M > 64:
        ws = torch.empty(pb.w4_linear_workspace_size(M, K, N, 128), dtype=torch.uint8, device="cuda")
        pb.w4_linear(x, d["qweight"], d["qzeros"], d["scales"].to(dtype), None, d["cs"], d["pairs"], d["theta"],
                     128, lay.krot, workspace=ws, rmat=R)
        torch.cuda.synchronize()
        assert torch.equal(xr, ws[: M * K * 2].view(dtype).view(M, K))
    ref = oracle.rotate(x.float().cpu().numpy().astype(np.float64), lay.channel_scales, lay.pairs, lay.theta, 128)
    got = xr.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
    tol = 1e-3 if dtype == torch.float16 else 5e-3
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), rms)) <= tol
