"""Guard bands around every output: each output (and the workspace) lives in the
middle of a larger buffer whose margins hold a byte pattern; after the call the
margins must be untouched, and the output must equal the same call into a
plain buffer.  Shapes are ragged on purpose (partial row tiles, partial column
tiles and column boxes past N), so every clipped store and every bounds check
in the kernels is exercised.  This stands in for a memory checker, which is not
available on the GPU pool."""
import numpy as np
import pytest

import synth
from tests.gpu_util import dev, layer_to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_w4_weight_b200 as pb  # noqa: E402

GUARD = 4096          # bytes on each side (a multiple of 256 keeps the view aligned)
PATTERN = 0xA5


@pytest.fixture(autouse=True)
def _status_clean():
    assert pb.device_status(clear=True) == pb.PARO_OK
    yield
    assert pb.device_status(clear=True) == pb.PARO_OK


def guarded(shape, dtype):
    """(buffer, view): the view of `shape` sits between two GUARD-byte margins."""
    esize = torch.tensor([], dtype=dtype).element_size()
    n = int(np.prod(shape)) * esize
    buf = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(dtype).view(*shape)


def margins_intact(buf):
    b = buf.cpu().numpy()
    return bool((b[:GUARD] == PATTERN).all() and (b[-GUARD:] == PATTERN).all())


LINEAR_CASES = [
    # (M, K, N): decode (partial 128-column tile), prefill (partial row tile,
    # a GEMM column box straddling N and boxes wholly past it)
    (1, 512, 544), (5, 512, 544), (16, 512, 544),
    (65, 384, 544), (300, 384, 544), (300, 384, 1056), (40, 256, 288),
]


@pytest.mark.parametrize("M,K,N", LINEAR_CASES)
def test_linear_writes_stay_inside_output_and_workspace(M, K, N):
    lay = synth.make_layer("g", K, N, seed=M + N, bias_std=0.01, n_outliers=3)
    d = layer_to_device(lay)
    x = dev(synth.make_activations(lay, M))
    args = (x, d["qweight"], d["qzeros"], d["scales"], d["bias"], d["cs"], d["pairs"], d["theta"], 128, lay.krot)
    ref = pb.w4_linear(*args)
    ybuf, y = guarded((M, N), torch.float16)
    need = pb.w4_linear_workspace_size(M, K, N)
    wbuf, ws = guarded((need,), torch.uint8)
    pb.w4_linear(*args, workspace=ws, out=y)
    torch.cuda.synchronize()
    assert margins_intact(ybuf) and margins_intact(wbuf)
    assert torch.equal(y, ref)


@pytest.mark.parametrize("M", [3, 40, 200])
def test_rotate_writes_stay_inside_output(M):
    lay = synth.make_layer("r", 384, 32, seed=M, n_outliers=3)
    x = dev(synth.make_activations(lay, M))
    args = (x, dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), 128, lay.krot)
    ref = pb.rotate(*args)
    buf, out = guarded((M, 384), torch.float16)
    pb.rotate(*args, out=out)
    torch.cuda.synchronize()
    assert margins_intact(buf)
    assert torch.equal(out, ref)


def test_group_prefill_writes_stay_inside_outputs_and_workspace():
    M, K = 300, 384
    lays = [synth.make_layer("m%d" % i, K, N, seed=80 + i, bias_std=0.01) for i, N in enumerate([544, 256, 1056])]
    ds = [layer_to_device(l) for l in lays]
    x = dev(synth.make_activations(lays[0], M))
    members = [dict(qweight=d["qweight"], qzeros=d["qzeros"], scales=d["scales"], bias=d["bias"],
                    channel_scales=d["cs"], pairs=d["pairs"], theta=d["theta"], krot=l.krot)
               for l, d in zip(lays, ds)]
    refs = pb.w4_linear_group(x, members)
    bufs, outs = zip(*[guarded((M, l.N), torch.float16) for l in lays])
    arr = pb._members(x, members, list(outs))
    need = int(pb.paro_w4_linear_group_workspace_size(M, K, len(members), arr, 128))
    wbuf, ws = guarded((need,), torch.uint8)
    pb.w4_linear_group(x, members, workspace=ws, out=list(outs))
    torch.cuda.synchronize()
    assert all(margins_intact(b) for b in bufs) and margins_intact(wbuf)
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)


def test_quantizer_writes_stay_inside_packed_outputs():
    N, K = 264, 256                            # a partial 128-row tile of weight rows
    lay = synth.make_layer("q", K, N, seed=90)
    W, qs = synth.make_float_weight(lay)
    args = (dev(W), dev(lay.channel_scales), dev(lay.pairs), dev(lay.theta), dev(qs), 128, lay.krot)
    ref_w, ref_z = pb.quantize_w4(*args)
    wbuf, qw = guarded((K, N // 8), torch.int32)
    zbuf, qz = guarded((K // 128, N // 8), torch.int32)
    pb.quantize_w4(*args, out=(qw, qz))
    torch.cuda.synchronize()
    assert margins_intact(wbuf) and margins_intact(zbuf)
    assert torch.equal(qw, ref_w) and torch.equal(qz, ref_z)
