"""GPU parity of stacked experts sharing one rotation (paro_w4_moe_linear)
against the float64 oracle (moe_linear_from_codes) on the same seeded inputs:
decode segments (T <= 16) and prefill tiles, distinct and repeated experts
per token, experts no token selects, ragged per-expert row counts, tiles
that run past 256 rows, an index outside the experts (zero row, flagged),
no rotation, bf16 and smaller groups.  Tolerance as for every linear:
max |d| <= 2e-2 * rms(y)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import LIN_TOL, dev, lin_err

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


def make_experts(E, K, N, G=128, seed=0, bias=True, krot=8):
    """E experts with their own codes, zero points, scales and bias, and the
    first one's rotation shared by all."""
    lays = [synth.make_layer(f"ex{e}", K, N, seed=seed + 17 * e, group_size=G, krot=krot,
                             bias_std=0.01 if bias else 0.0, zero_point=None) for e in range(E)]
    codes = np.stack([l.codes for l in lays])
    zeros = np.stack([l.zero_codes for l in lays])
    scales = np.stack([l.scales for l in lays])
    b = np.stack([l.bias for l in lays]) if bias else None
    qw, qz = [], []
    for l in lays:
        w, z = pb.pack_awq(dev(l.codes), dev(l.zero_codes), G)
        qw.append(w)
        qz.append(z)
    return lays[0], dict(codes=codes, zeros=zeros, scales=scales, bias=b,
                         qweight=torch.stack(qw).contiguous(), qzeros=torch.stack(qz).contiguous())


def route(T, topk, E, seed, experts=None, distinct=True):
    """Seeded expert choices; `experts` limits them to a subset (the others stay empty)."""
    rng = np.random.default_rng(seed)
    pool = np.arange(E) if experts is None else np.asarray(experts)
    if distinct and topk <= pool.size:
        return np.stack([rng.choice(pool, topk, replace=False) for _ in range(T)]).astype(np.int32)
    return rng.choice(pool, (T, topk)).astype(np.int32)


def run(rot, ex, x, idx, G=128, rotate=True, dtype=torch.float16):
    def cast(a):
        return None if a is None else torch.from_numpy(np.asarray(a, np.float32)).to(dtype).cuda()
    y = pb.w4_moe_linear(cast(x), dev(idx), ex["qweight"], ex["qzeros"], cast(ex["scales"]), cast(ex["bias"]),
                         dev(rot.channel_scales) if rotate else None, dev(rot.pairs) if rotate else None,
                         dev(rot.theta) if rotate else None, G, rot.krot if rotate else 0)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64)


def ref_of(rot, ex, x, idx, G=128, rotate=True):
    return oracle.moe_linear_from_codes(x, idx, ex["codes"], ex["zeros"], ex["scales"], ex["bias"],
                                        rot.channel_scales if rotate else None, rot.pairs if rotate else None,
                                        rot.theta if rotate else None, G, rot.krot if rotate else 0)


# (T, topk, E, K, N, distinct): decode segments, then prefill tiles
CASES = [(1, 8, 64, 512, 256, True), (3, 2, 8, 512, 384, True), (5, 4, 4, 256, 256, False),
         (16, 4, 4, 512, 256, True), (16, 8, 16, 1024, 512, True), (17, 2, 8, 512, 256, True),
         (300, 2, 8, 512, 512, True), (700, 1, 2, 256, 256, True)]


@pytest.mark.parametrize("T,topk,E,K,N,distinct", CASES)
def test_moe_vs_oracle(T, topk, E, K, N, distinct):
    rot, ex = make_experts(E, K, N, seed=T + E)
    lay = synth.make_layer("xm", K, 32, seed=T)
    x = synth.make_activations(lay, T)
    idx = route(T, topk, E, seed=T * 7 + topk, distinct=distinct)
    y = run(rot, ex, x, idx)
    ref = ref_of(rot, ex, x, idx)
    assert y.shape == (T, topk, N)
    assert lin_err(y.reshape(T * topk, N), ref.reshape(T * topk, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [4, 200])
def test_moe_empty_experts_and_ragged_counts(T):
    """Only experts 1, 3 and 6 of 8 are ever selected, with very different counts."""
    E, K, N, topk = 8, 512, 256, 2
    rot, ex = make_experts(E, K, N, seed=11)
    x = synth.make_activations(synth.make_layer("xe", K, 32, seed=T), T)
    rng = np.random.default_rng(T)
    idx = rng.choice([1, 3, 6], size=(T, topk), p=[0.7, 0.25, 0.05]).astype(np.int32)
    y = run(rot, ex, x, idx)
    ref = ref_of(rot, ex, x, idx)
    assert lin_err(y.reshape(-1, N), ref.reshape(-1, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [2, 40])
def test_moe_index_outside_the_experts_gives_a_zero_row_and_a_flag(T):
    E, K, N, topk = 4, 256, 256, 2
    rot, ex = make_experts(E, K, N, seed=5)
    x = synth.make_activations(synth.make_layer("xi", K, 32, seed=T), T)
    idx = route(T, topk, E, seed=T)
    idx[0, 1] = E
    idx[T - 1, 0] = -1
    y = run(rot, ex, x, idx)
    assert pb.device_status(clear=True) == pb.PARO_ERR_INVALID_ARG
    ref = ref_of(rot, ex, x, idx)
    assert np.all(y[0, 1] == 0.0) and np.all(y[T - 1, 0] == 0.0)
    assert lin_err(y.reshape(-1, N), ref.reshape(-1, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [3, 64])
def test_moe_without_rotation_and_bias(T):
    E, K, N, topk = 4, 512, 256, 2
    rot, ex = make_experts(E, K, N, seed=23, bias=False)
    x = synth.make_activations(synth.make_layer("xn", K, 32, seed=T), T)
    idx = route(T, topk, E, seed=T + 1)
    y = run(rot, ex, x, idx, rotate=False)
    ref = ref_of(rot, ex, x, idx, rotate=False)
    assert lin_err(y.reshape(-1, N), ref.reshape(-1, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [2, 100])
def test_moe_group_size_32(T):
    E, K, N, topk = 4, 512, 256, 2
    rot, ex = make_experts(E, K, N, G=32, seed=31)
    x = synth.make_activations(synth.make_layer("xg", K, 32, seed=T), T)
    idx = route(T, topk, E, seed=T + 2)
    y = run(rot, ex, x, idx, G=32)
    ref = ref_of(rot, ex, x, idx, G=32)
    assert lin_err(y.reshape(-1, N), ref.reshape(-1, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [1, 80])
def test_moe_bf16(T):
    """bf16: the oracle gets the exact bf16 values of x, scales and bias; the
    bound adds one bf16 rounding of Y (2^-8 of each output)."""
    E, K, N, topk = 4, 512, 256, 2
    rot, ex = make_experts(E, K, N, seed=41)
    x = synth.make_activations(synth.make_layer("xb", K, 32, seed=T), T).astype(np.float32)
    idx = route(T, topk, E, seed=T + 3)
    y = run(rot, ex, x, idx, dtype=torch.bfloat16)

    def exact(a):
        return None if a is None else torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()
    ex_b = dict(ex, scales=exact(ex["scales"]), bias=exact(ex["bias"]))
    ref = ref_of(rot, ex_b, exact(x), idx).reshape(-1, N)
    rms = float(np.sqrt(np.mean(ref * ref)))
    assert np.max(np.abs(y.reshape(-1, N) - ref) - (3e-2 * rms + 2.0 ** -8 * np.abs(ref))) <= 0


def test_moe_large_prefill_sampled_columns():
    """4096 tokens, top-2 of 8 experts, K = 2048: tiles run past 256 rows per expert."""
    E, K, N, topk, T = 8, 2048, 1024, 2, 4096
    rot, ex = make_experts(E, K, N, seed=51)
    x = synth.make_activations(synth.make_layer("xl", K, 32, seed=3), T)
    idx = route(T, topk, E, seed=9)
    y = run(rot, ex, x, idx)
    rows = np.random.default_rng(1).choice(T, 48, replace=False)
    ref = ref_of(rot, ex, x[rows], idx[rows])
    assert lin_err(y[rows].reshape(-1, N), ref.reshape(-1, N)) <= LIN_TOL


@pytest.mark.parametrize("T", [1, 2])
def test_moe_decode_wide_experts(T):
    """Gate-shaped experts (4096 -> 14336, the wide GEMV plan) at one and two
    tokens, top-2 of 2.  Sampled columns of every slot against the oracle's
    columns of its expert."""
    E, K, N, topk = 2, 4096, 14336, 2
    rot, ex = make_experts(E, K, N, seed=61)
    x = synth.make_activations(synth.make_layer("xw", K, 32, seed=T), T)
    idx = route(T, topk, E, seed=T + 4)
    y = run(rot, ex, x, idx)
    cols = np.sort(np.random.default_rng(T).choice(N, 96, replace=False))
    for t in range(T):
        for j in range(topk):
            e = int(idx[t, j])
            ref = oracle.w4_linear_columns(x[t:t + 1], ex["codes"][e], ex["zeros"][e], ex["scales"][e],
                                           ex["bias"][e], rot.channel_scales, rot.pairs, rot.theta, 128,
                                           rot.krot, cols)
            assert lin_err(y[t, j][None, cols], ref) <= LIN_TOL, (t, j)
