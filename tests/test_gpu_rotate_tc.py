"""GPU parity of the tensor-core rotation that paro_w4_linear uses above 64
token rows: R' = diag(cs) G_0 ... G_{krot-1} built per group, then
X_r = X R' on the tensor cores.  X_r is read back from the first M*K*2 bytes
of the workspace (the header guarantees it holds X_r after a rotating call)
and compared with the float64 oracle's rotation, element by element; Y is
compared with the oracle's linear where that is cheap."""
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


TC_CASES = [
    # (M, K, N, krot, use_cs, active pairs)
    (65, 256, 512, 8, True, None),         # smallest batch on this path: one 128-row tile, 63 rows clipped
    (128, 512, 256, 8, True, None),        # exactly one full tile per group
    (200, 1024, 256, 17, True, None),      # krot 17
    (256, 256, 512, 8, True, None),        # 4 tiles, fewer CTAs than SMs
    (300, 1024, 256, 8, True, None),       # ragged last row tile
    (512, 128, 256, 8, True, None),        # one group: every CTA shares it
    (1000, 384, 256, 1, False, None),      # krot = 1, no channel scales
    (257, 512, 256, 64, True, None),       # krot at the supported maximum
    (640, 512, 256, 0, True, None),        # scaling only: R' is diagonal
    (2048, 4096, 512, 8, True, 6),         # 10 % active pairs
    (1200, 14336, 256, 8, True, None),     # down_proj width: 112 groups, ranges cross groups
    (8192, 4096, 256, 8, True, None),      # full prefill rows: 2048 tiles over one wave of CTAs
]


def run_case(M, K, N, krot, use_cs, active, seed):
    lay = synth.make_layer("t", K, N, seed=seed, krot=max(krot, 1), active_pairs=active,
                           n_outliers=max(1, K // 100), bias_std=0.01)
    pairs, theta = lay.pairs[:krot], lay.theta[:krot]
    cs = lay.channel_scales if use_cs else None
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    need = pb.w4_linear_workspace_size(M, K, N)
    assert need >= M * K * 2 + 2 * K * 128 * 2
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)                          # NaN pattern: every X_r element must be written
    y = pb.w4_linear(dev(x), d["qweight"], d["qzeros"], d["scales"], d["bias"], dev(cs),
                     dev(pairs) if krot else None, dev(theta) if krot else None, 128, krot,
                     workspace=ws)
    torch.cuda.synchronize()
    xr = ws[: M * K * 2].view(torch.float16).view(M, K).cpu().numpy().astype(np.float64)
    ref = oracle.rotate(x, cs, pairs if krot else None, theta if krot else None, 128, krot=krot)
    assert np.isfinite(xr).all()
    err = rot_err(xr, ref)
    assert err <= ROT_TOL, err
    if M * K * N <= 2 ** 31:
        yref = oracle.w4_linear_from_codes(x, lay.codes, lay.zero_codes, lay.scales, lay.bias, cs,
                                           pairs if krot else None, theta if krot else None, 128, krot)
        assert lin_err(y.cpu().numpy().astype(np.float64), yref) <= LIN_TOL
    return xr


@pytest.mark.parametrize("M,K,N,krot,use_cs,active", TC_CASES)
def test_tensor_core_rotation_vs_oracle(M, K, N, krot, use_cs, active):
    run_case(M, K, N, krot, use_cs, active, seed=M + K + krot)


def test_tensor_core_rotation_identity_state_is_exact():
    """Zero angles and unit scales: R' = I exactly (Rlo = 0), so X_r == x bit for bit."""
    M, K, N = 384, 512, 256
    lay = synth.make_layer("e", K, N, seed=5)
    d = layer_to_device(lay)
    x = synth.make_activations(lay, M)
    ws = torch.empty(pb.w4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    pb.w4_linear(dev(x), d["qweight"], d["qzeros"], d["scales"], None, dev(np.ones(K, np.float32)),
                 d["pairs"], dev(np.zeros_like(lay.theta)), 128, lay.krot, workspace=ws)
    torch.cuda.synchronize()
    xr = ws[: M * K * 2].view(torch.float16).view(M, K).cpu().numpy()
    assert np.array_equal(xr, x)


def test_tensor_core_rotation_workspace_reuse_is_deterministic():
    """Two calls in a row through one workspace (the R' parts of the first call
    are overwritten by the second): identical outputs."""
    M, K, N = 600, 1024, 512
    lay = synth.make_layer("w", K, N, seed=6)
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, M))
    ws = torch.empty(pb.w4_linear_workspace_size(M, K, N), dtype=torch.uint8, device="cuda")
    outs = [pb.w4_linear(x, d["qweight"], d["qzeros"], d["scales"], None, d["cs"], d["pairs"],
                         d["theta"], 128, lay.krot, workspace=ws).cpu().numpy() for _ in range(2)]
    assert np.array_equal(outs[0], outs[1])
