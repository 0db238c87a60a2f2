"""Pins for the float64 oracle: checks against what the pages and the mathematics
fix, not against the oracle itself.

Each ``pin_*`` takes an implementation namespace ``impl`` exposing
``rotate``, ``inverse_rotate``, ``awq_pack``, ``awq_unpack``, ``dequant``,
``w4_linear_from_codes``, ``transform_weight``, ``quantize_sym4`` and
``quantize_weight`` with the oracle's signatures, and raises
AssertionError when the implementation disagrees.  ``test_oracle_pins.py``
runs them on the oracle; ``test_oracle_mutations.py`` runs them on copies of
the oracle with planted mistakes and checks that each mistake is caught.

Sources (GPTQModel wiki page "ParoQuant"):
  * "Pairwise Givens rotations": a' = a cos t + b sin t, b' = -a sin t + b cos t;
    stages in order; inverse = reversed order with negated angles; pair
    indices local to each group.
  * "Activation and weight transforms": R orthogonal; X_r = X D^-1 R,
    W_r = W D R, X_r W_r^T = X W^T without quantisation; the equivalent
    original-domain weight is Q(W_r) R^T D^-1.
  * "Stored tensors": identity state = zero angles and unit channel scales.
  * "Activation and weight transforms" (quantiser paragraph): four-bit
    symmetric codes -8..7, exported unsigned with zero point 8, quantiser
    scales bounded to [1e-5, 1e5]; nearest level with ties to even (the
    rounding named in "STE acceleration kernels").
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_tables(rng, K, G, krot, active=None):
    pairs = np.empty((krot, K), np.int16)
    theta = np.zeros((krot, K // 2), np.float64)
    half = G // 2
    for s in range(krot):
        for g in range(K // G):
            pairs[s, g * G:(g + 1) * G] = rng.permutation(G)
            n = half if active is None else active
            sel = rng.choice(half, n, replace=False)
            theta[s, g * half + sel] = rng.uniform(-np.pi, np.pi, n)
    return pairs, theta


def _givens_matrix_of_stage(pairs_s, theta_s, K, G):
    """Dense K x K matrix M of one stage in the row-vector convention
    (x' = x M), written entry by entry from the pair formula:
        x'_i = c x_i + s x_j   ->  M[i, i] = c,  M[j, i] = s
        x'_j = -s x_i + c x_j  ->  M[i, j] = -s, M[j, j] = c
    Built with explicit Python loops over groups and pairs."""
    M = np.zeros((K, K))
    for g in range(K // G):
        for p in range(G // 2):
            i = g * G + int(pairs_s[g * G + 2 * p])
            j = g * G + int(pairs_s[g * G + 2 * p + 1])
            t = float(theta_s[g * (G // 2) + p])
            c, s = math.cos(t), math.sin(t)
            M[i, i] = c
            M[j, i] = s
            M[i, j] = -s
            M[j, j] = c
    return M


def dense_R(pairs, theta, K, G):
    R = np.eye(K)
    for s in range(pairs.shape[0]):
        R = R @ _givens_matrix_of_stage(pairs[s], theta[s], K, G)
    return R


# ---------------------------------------------------------------- rotation pins

def pin_single_pair_closed_forms(impl):
    """t = pi/2: (a,b) -> (b,-a); t = pi: (a,b) -> (-a,-b); t = 0: identity."""
    K = G = 8
    pairs = np.array([[3, 5, 0, 1, 2, 4, 6, 7]], np.int16)   # pair 0 = (3, 5)
    x = np.array([[0.1, -0.2, 0.3, 1.25, 0.5, -0.75, 0.7, 0.9]])
    for t, (ea, eb) in [(math.pi / 2, (-0.75, -1.25)), (math.pi, (-1.25, 0.75)),
                        (0.0, (1.25, -0.75))]:
        theta = np.zeros((1, K // 2))
        theta[0, 0] = t
        y = impl.rotate(x, None, pairs, theta, G)
        assert abs(y[0, 3] - ea) <= 1e-15 and abs(y[0, 5] - eb) <= 1e-15, (t, y[0, 3], y[0, 5])
        others = [0, 1, 2, 4, 6, 7]
        assert np.array_equal(y[0, others], x[0, others])


def pin_stage_composition(impl):
    """Two stages with the same pairs and angles t1, t2 equal one stage t1 + t2."""
    rng = np.random.default_rng(11)
    K, G = 256, 128
    p1, t1 = _rand_tables(rng, K, G, 1)
    t2 = rng.uniform(-np.pi, np.pi, t1.shape)
    x = rng.standard_normal((5, K))
    two = impl.rotate(x, None, np.concatenate([p1, p1]), np.concatenate([t1, t2]), G)
    one = impl.rotate(x, None, p1, t1 + t2, G)
    assert np.max(np.abs(two - one)) <= 1e-13


def pin_inverse_restores(impl):
    """Reversed stage order with negated angles restores the input (<= 1e-12)."""
    rng = np.random.default_rng(12)
    K, G = 512, 128
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    x = rng.standard_normal((7, K)) * 3
    xr = impl.rotate(x, cs, pairs, theta, G)
    back = impl.inverse_rotate(xr, cs, pairs, theta, G)
    assert np.max(np.abs(back - x)) <= 1e-12 * max(1.0, np.max(np.abs(x)))


def pin_group_norms_preserved(impl):
    """R is orthogonal and group-local: each group's L2 norm of x*cs is kept."""
    rng = np.random.default_rng(13)
    K, G = 384, 128
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    x = rng.standard_normal((6, K))
    xr = impl.rotate(x, cs, pairs, theta, G)
    n0 = np.linalg.norm((x * cs).reshape(6, K // G, G), axis=2)
    n1 = np.linalg.norm(xr.reshape(6, K // G, G), axis=2)
    assert np.max(np.abs(n1 - n0) / n0) <= 1e-12


def pin_dense_R_brute_force(impl):
    """Small K: the stage-by-stage result equals (x * cs) @ R with R the product
    of dense per-stage Givens matrices built entry by entry."""
    rng = np.random.default_rng(14)
    for K, G, krot in [(128, 128, 1), (128, 128, 3), (256, 128, 2), (256, 128, 8), (64, 16, 4)]:
        pairs, theta = _rand_tables(rng, K, G, krot)
        cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
        x = rng.standard_normal((3, K))
        ref = (x * cs) @ dense_R(pairs, theta, K, G)
        got = impl.rotate(x, cs, pairs, theta, G)
        assert np.max(np.abs(got - ref)) <= 1e-12, (K, G, krot)


def pin_golden_g4(impl):
    g = json.load(open(os.path.join(GOLDEN, "rotation_g4_krot2.json")))
    theta = np.array([[math.pi / 2, 0.0], [math.pi / 3, math.pi]])
    got = impl.rotate(np.array(g["x"]), np.array(g["channel_scales"]),
                      np.array(g["pairs"], np.int16), theta, g["group_size"])
    assert np.max(np.abs(got - np.array(g["expected"]))) <= 1e-14, got


def pin_group_size_minus_one(impl):
    """group_size=-1 is the whole input width."""
    rng = np.random.default_rng(15)
    K = 64
    pairs, theta = _rand_tables(rng, K, K, 2)
    x = rng.standard_normal((2, K))
    a = impl.rotate(x, None, pairs, theta, -1)
    b = x @ dense_R(pairs, theta, K, K)
    assert np.max(np.abs(a - b)) <= 1e-12


def pin_unquantized_identity(impl):
    """X_r W_r^T = X W^T with W_r = W D R (rows of W rotated like activations
    but scaled by D = 1/channel_scales)."""
    rng = np.random.default_rng(16)
    K, G, N, M = 512, 128, 48, 9
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))      # D^-1
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    xr = impl.rotate(x, cs, pairs, theta, G)
    wr = impl.rotate(W, 1.0 / cs, pairs, theta, G)
    lhs = xr @ wr.T
    rhs = x @ W.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-10 * np.max(np.abs(rhs))


# ------------------------------------------------------------- packing pins

def pin_awq_golden_word(impl):
    g = json.load(open(os.path.join(GOLDEN, "awq_word.json")))
    codes = np.zeros((8, 128), np.uint8)
    codes[:, 0] = g["codes_of_columns_0_to_7"]
    qw, _ = impl.awq_pack(codes, np.zeros((8, 1), np.uint8), 128)
    assert int(np.uint32(qw.view(np.uint32)[0, 0])) == int(g["word_hex"], 16), hex(int(qw.view(np.uint32)[0, 0]))


def pin_awq_one_hot(impl):
    """A single code 15 at (n, k) lands in word (k, n//8) at nibble position
    pos[n % 8], pos = [0,4,1,5,2,6,3,7]; every other nibble is 0."""
    g = json.load(open(os.path.join(GOLDEN, "awq_word.json")))
    pos = g["nibble_position_of_column"]
    N, K, G = 24, 256, 128
    for n in range(N):
        for k in (0, 1, 127, 128, 255):
            codes = np.zeros((N, K), np.uint8)
            codes[n, k] = 15
            zeros = np.zeros((N, K // G), np.uint8)
            zeros[n, k // G] = 9
            qw, qz = impl.awq_pack(codes, zeros, G)
            u = qw.view(np.uint32)
            assert u[k, n // 8] == np.uint32(15 << (4 * pos[n % 8]))
            assert np.count_nonzero(u) == 1
            uz = qz.view(np.uint32)
            assert uz[k // G, n // 8] == np.uint32(9 << (4 * pos[n % 8]))
            assert np.count_nonzero(uz) == 1


def pin_awq_round_trip(impl):
    rng = np.random.default_rng(17)
    N, K, G = 64, 512, 128
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (N, K // G), dtype=np.uint8)
    qw, qz = impl.awq_pack(codes, zeros, G)
    assert qw.dtype == np.int32 and qw.shape == (K, N // 8) and qz.shape == (K // G, N // 8)
    c2, z2 = impl.awq_unpack(qw, qz, N, K, G)
    assert np.array_equal(c2, codes) and np.array_equal(z2, zeros)


# ---------------------------------------------------------- dequant + linear pins

def _brute_linear(x, codes, zeros, scales, bias, G):
    """Y[m, n] = sum_k x[m, k] * (codes[n, k] - zeros[n, k//G]) * scales[k//G, n] + bias[n],
    one output at a time."""
    M, K = x.shape
    N = codes.shape[0]
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(x[m, k]) * (int(codes[n, k]) - int(zeros[n, k // G])) * float(scales[k // G, n])
            Y[m, n] = acc + (0.0 if bias is None else float(bias[n]))
    return Y


def pin_identity_state_is_plain_w4(impl):
    """Zero angles and unit channel scales reduce the layer to a plain W4
    dequant-matmul, checked one output at a time."""
    rng = np.random.default_rng(18)
    M, K, N, G = 2, 256, 16, 128
    x = rng.standard_normal((M, K)).astype(np.float16)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (N, K // G), dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, (K // G, N)).astype(np.float16)
    bias = rng.standard_normal(N).astype(np.float16)
    pairs, _ = _rand_tables(rng, K, G, 8)
    theta = np.zeros((8, K // 2))
    ref = _brute_linear(x, codes, zeros, scales, bias, G)
    got = impl.w4_linear_from_codes(x, codes, zeros, scales, bias, np.ones(K), pairs, theta, G, 8)
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))
    got0 = impl.w4_linear_from_codes(x, codes, zeros, scales, bias, None, None, None, G, 0)
    assert np.max(np.abs(got0 - ref)) <= 1e-10 * np.max(np.abs(ref))


def pin_equivalent_weight_route(impl):
    """Y = X_r Q(W_r)^T + b equals X (Q(W_r) R^T D^-1)^T + b (equivalent
    original-domain weight)."""
    rng = np.random.default_rng(19)
    M, K, N, G = 3, 256, 24, 128
    x = rng.standard_normal((M, K))
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))       # D^-1
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (N, K // G), dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, (K // G, N))
    bias = rng.standard_normal(N)
    Wq = np.empty((N, K))                                       # Q(W_r), out x in
    for n in range(N):
        for k in range(K):
            Wq[n, k] = (int(codes[n, k]) - int(zeros[n, k // G])) * scales[k // G, n]
    R = dense_R(pairs, theta, K, G)
    W_eq = Wq @ R.T @ np.diag(cs)
    ref = x @ W_eq.T + bias
    got = impl.w4_linear_from_codes(x, codes, zeros, scales, bias, cs, pairs, theta, G, 8)
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


def pin_dequant_formula(impl):
    """(q - z) * s on single elements, one group boundary crossed."""
    N, K, G = 8, 256, 128
    codes = np.zeros((N, K), np.uint8)
    zeros = np.full((N, K // G), 8, np.uint8)
    scales = np.ones((K // G, N))
    codes[3, 5] = 15
    codes[6, 200] = 0
    zeros[6, 1] = 3
    scales[1, 6] = 0.5
    W = impl.dequant(codes, zeros, scales, G)
    assert W.shape == (K, N)
    assert W[5, 3] == 7.0
    assert W[200, 6] == -1.5
    assert W[0, 0] == -8.0
    assert W[130, 6] == -1.5


# ------------------------------------------------------- weight-side pins

def pin_weight_transform_identity(impl):
    """transform_weight gives W_r = W D R: with the activations' X_r = X D^-1 R,
    X_r W_r^T = X W^T (no quantisation), and zero angles with unit scales
    leave W unchanged."""
    rng = np.random.default_rng(21)
    K, G, N, M = 384, 128, 40, 5
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))      # D^-1
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K))
    lhs = impl.rotate(x, cs, pairs, theta, G) @ impl.transform_weight(W, cs, pairs, theta, G).T
    rhs = x @ W.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-10 * np.max(np.abs(rhs))
    same = impl.transform_weight(W, np.ones(K), pairs, np.zeros_like(theta), G)
    assert np.max(np.abs(same - W)) <= 1e-15 * np.max(np.abs(W))
    # one channel, one pair at a right angle: (a, b) -> (b, -a) after the 1/cs scaling
    p1 = np.tile(np.arange(G, dtype=np.int16), (1, K // G))
    t1 = np.zeros((1, K // 2))
    t1[0, 0] = np.pi / 2
    w1 = np.zeros((1, K))
    w1[0, 0], w1[0, 1] = 3.0, 5.0
    c1 = np.ones(K)
    c1[0], c1[1] = 2.0, 0.5
    got = impl.transform_weight(w1, c1, p1, t1, G)
    assert abs(got[0, 0] - 10.0) <= 1e-12 and abs(got[0, 1] + 1.5) <= 1e-12


def pin_sym4_closed_forms(impl):
    """Code of chosen quotients (exact in binary): nearest level, ties to even,
    clamping to -8..7, zero point 8, scale bounds."""
    K, G = 128, 128
    t = np.array([0.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.25, 6.5, 7.4, 7.5, 100.0,
                  -7.5, -8.4, -8.5, -100.0, 1.0, -1.0])
    want_q = np.array([0, 0, 2, 2, 0, -2, -2, 3, 6, 7, 7, 7, -8, -8, -8, -8, 1, -1])
    s = 0.25                                                  # power of two: W_r / s is exact
    W = np.zeros((8, K))
    W[0, :t.size] = t * s
    scales = np.full((K // G, 8), s)
    codes, zeros = impl.quantize_sym4(W, scales, G)
    assert codes.dtype == np.uint8 and codes.shape == (8, K) and zeros.shape == (8, K // G)
    assert np.array_equal(codes[0, :t.size].astype(int), want_q + 8), codes[0, :t.size]
    assert np.all(codes[1:] == 8) and np.all(zeros == 8)
    # bounds: a zero scale acts as 1e-5, a huge one as 1e5
    W2 = np.zeros((8, K))
    W2[0, 0] = 3e-5
    W2[1, 0] = 2.5e5
    W2[2, 0] = -7e5
    sc2 = np.ones((K // G, 8))
    sc2[0, 0] = 0.0
    sc2[0, 1] = 1e6
    sc2[0, 2] = 1e9
    c2, _ = impl.quantize_sym4(W2, sc2, G)
    assert int(c2[0, 0]) == 11 and int(c2[1, 0]) == 10 and int(c2[2, 0]) == 1, c2[:3, 0]


def pin_sym4_nearest_level_brute_force(impl):
    """Every code's level (code - 8) * s is a nearest one of the 16 levels
    -8 s .. 7 s to the value, found by trying them all; groups and columns
    each use their own scale."""
    rng = np.random.default_rng(22)
    N, K, G = 16, 256, 128
    scales = rng.uniform(0.05, 0.3, (K // G, N))
    W = rng.standard_normal((N, K)) * 0.8
    codes, zeros = impl.quantize_sym4(W, scales, G)
    levels = np.arange(-8, 8)
    for n in range(N):
        for k in range(K):
            sc = scales[k // G, n]
            d = np.abs(levels * sc - W[n, k])
            got = (int(codes[n, k]) - int(zeros[n, k // G])) * sc
            assert abs(got - W[n, k]) <= d.min() + 1e-12, (n, k)


def pin_quantized_replay(impl):
    """The packed layer replays Y = X_r Q(W_r)^T + b: the codes from
    quantize_sym4(transform_weight(W)) through w4_linear_from_codes equal a
    one-output-at-a-time sum over the nearest levels of W_r."""
    rng = np.random.default_rng(23)
    M, K, N, G = 2, 256, 16, 128
    pairs, theta = _rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    W = rng.standard_normal((N, K))
    x = rng.standard_normal((M, K))
    bias = rng.standard_normal(N)
    W_r = impl.transform_weight(W, cs, pairs, theta, G)
    scales = np.max(np.abs(W_r).reshape(N, K // G, G), axis=2).T / 6.0
    codes, zeros = impl.quantize_sym4(W_r, scales, G)
    got = impl.w4_linear_from_codes(x, codes, zeros, scales, bias, cs, pairs, theta, G, 8)
    xr = impl.rotate(x, cs, pairs, theta, G)
    levels = np.arange(-8, 8)
    ref = np.zeros((M, N))
    for n in range(N):
        for k in range(K):
            sc = scales[k // G, n]
            lv = levels[np.argmin(np.abs(levels * sc - W_r[n, k]))] * sc
            ref[:, n] += xr[:, k] * lv
    ref += bias
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))


def _nibble_codes(qw, N, K):
    """Codes [N, K] read out of AWQ words bit by bit, with the nibble position
    of each column taken from the golden word fixture (not from any packer)."""
    g = json.load(open(os.path.join(GOLDEN, "awq_word.json")))
    pos = g["nibble_position_of_column"]
    u = np.asarray(qw).view(np.uint32)
    codes = np.empty((N, K), np.int64)
    for n in range(N):
        for k in range(K):
            codes[n, k] = (int(u[k, n // 8]) >> (4 * pos[n % 8])) & 0xF
    return codes


def pin_quantize_weight_packed(impl):
    """quantize_weight (transform, quantise, pack in one call) against a route
    that shares none of its steps: W_r = (W / cs) @ R with R the dense product
    of per-stage Givens matrices built entry by entry, every word read back
    nibble by nibble from the golden positions, and each code's level a
    nearest of the 16 levels -8 s .. 7 s of W_r (found by trying them all).
    Zero words are all 0x88888888 (zero point 8 in every nibble)."""
    rng = np.random.default_rng(24)
    N, K, G, krot = 16, 256, 128, 5
    pairs, theta = _rand_tables(rng, K, G, krot)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    W = rng.standard_normal((N, K)) * 0.7
    W_r = (W / cs) @ dense_R(pairs, theta, K, G)
    scales = rng.uniform(0.6, 1.2, (K // G, N)) * np.max(np.abs(W_r)) / 7.0
    qw, qz = impl.quantize_weight(W, cs, pairs, theta, scales, G, krot)
    qw, qz = np.asarray(qw), np.asarray(qz)
    assert qw.dtype == np.int32 and qw.shape == (K, N // 8), (qw.dtype, qw.shape)
    assert qz.dtype == np.int32 and qz.shape == (K // G, N // 8), (qz.dtype, qz.shape)
    assert np.all(qz.view(np.uint32) == np.uint32(0x88888888))
    codes = _nibble_codes(qw, N, K)
    levels = np.arange(-8, 8)
    for n in range(N):
        for k in range(K):
            sc = scales[k // G, n]
            best = np.min(np.abs(levels * sc - W_r[n, k]))
            got = abs((codes[n, k] - 8) * sc - W_r[n, k])
            assert got <= best + 1e-12, (n, k, codes[n, k])
    # krot=None takes every stage of the table
    qw2, _ = impl.quantize_weight(W, cs, pairs, theta, scales, G)
    assert np.array_equal(np.asarray(qw2), qw)


def pin_moe_stacked_experts_brute_force(impl):
    """moe_linear_from_codes against a route that shares none of its steps:
    X_r = (x * cs) @ R with R the dense product of per-stage Givens matrices
    built entry by entry (one rotation for every expert), then every output of
    every slot summed one term at a time with the slot's expert's codes, zero
    points, scales and bias.  The routing has an expert no token selects, an
    expert selected twice by one token, ragged per-expert counts and one
    index outside 0..E-1 (its row must be 0)."""
    rng = np.random.default_rng(25)
    T, K, N, G, E, topk, krot = 4, 128, 8, 64, 4, 2, 3
    pairs, theta = _rand_tables(rng, K, G, krot)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    x = rng.standard_normal((T, K))
    codes = rng.integers(0, 16, (E, N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (E, N, K // G), dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, (E, K // G, N))
    bias = rng.standard_normal((E, N))
    idx = np.array([[2, 0], [2, 2], [0, 3], [E, 2]])          # expert 1 empty; (3, 0) invalid
    xr = (x * cs) @ dense_R(pairs, theta, K, G)
    ref = np.zeros((T, topk, N))
    for t in range(T):
        for j in range(topk):
            e = int(idx[t, j])
            if not 0 <= e < E:
                continue
            ref[t, j] = _brute_linear(xr[t:t + 1], codes[e], zeros[e], scales[e], bias[e], G)[0]
    got = np.asarray(impl.moe_linear_from_codes(x, idx, codes, zeros, scales, bias, cs, pairs, theta, G, krot))
    assert got.shape == (T, topk, N), got.shape
    assert np.max(np.abs(got - ref)) <= 1e-10 * np.max(np.abs(ref))
    # no bias: the rows of the invalid slot stay exactly zero as well
    got0 = np.asarray(impl.moe_linear_from_codes(x, idx, codes, zeros, scales, None, cs, pairs, theta, G, krot))
    assert np.all(got0[3, 0] == 0.0)


def pin_moe_single_expert_is_the_dense_layer(impl):
    """With one expert and top-1 routing the layer is the dense rotated W4
    linear (itself pinned above), token for token."""
    rng = np.random.default_rng(26)
    T, K, N, G, krot = 5, 256, 16, 128, 4
    pairs, theta = _rand_tables(rng, K, G, krot)
    cs = np.exp(rng.uniform(np.log(0.5), np.log(2), K))
    x = rng.standard_normal((T, K))
    codes = rng.integers(0, 16, (1, N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (1, N, K // G), dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, (1, K // G, N))
    got = np.asarray(impl.moe_linear_from_codes(x, np.zeros((T, 1), np.int64), codes, zeros, scales, None, cs,
                                                pairs, theta, G, krot))
    ref = impl.w4_linear_from_codes(x, codes[0], zeros[0], scales[0], None, cs, pairs, theta, G, krot)
    assert np.max(np.abs(got[:, 0] - ref)) <= 1e-12 * np.max(np.abs(ref))


ALL_PINS = [
    pin_single_pair_closed_forms, pin_stage_composition, pin_inverse_restores,
    pin_group_norms_preserved, pin_dense_R_brute_force, pin_golden_g4,
    pin_group_size_minus_one, pin_unquantized_identity, pin_awq_golden_word,
    pin_awq_one_hot, pin_awq_round_trip, pin_identity_state_is_plain_w4,
    pin_equivalent_weight_route, pin_dequant_formula,
    pin_weight_transform_identity, pin_sym4_closed_forms, pin_sym4_nearest_level_brute_force,
    pin_quantized_replay, pin_quantize_weight_packed, pin_moe_stacked_experts_brute_force,
    pin_moe_single_expert_is_the_dense_layer,
]
