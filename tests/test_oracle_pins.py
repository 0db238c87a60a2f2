"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def test_w4_linear_packed_equals_from_codes():
    """The packed route (pack -> unpack -> dequant) and the codes route agree exactly."""
    rng = np.random.default_rng(3)
    M, K, N, G = 3, 256, 32, 128
    x = rng.standard_normal((M, K)).astype(np.float16)
    codes = rng.integers(0, 16, (N, K), dtype=np.uint8)
    zeros = rng.integers(0, 16, (N, K // G), dtype=np.uint8)
    scales = rng.uniform(0.005, 0.02, (K // G, N)).astype(np.float16)
    pairs, theta = oracle_pins._rand_tables(rng, K, G, 8)
    cs = np.exp(rng.uniform(-0.5, 0.5, K)).astype(np.float32)
    qw, qz = oracle.awq_pack(codes, zeros, G)
    a = oracle.w4_linear(x, qw, qz, scales, None, cs, pairs, theta, G, 8)
    b = oracle.w4_linear_from_codes(x, codes, zeros, scales, None, cs, pairs, theta, G, 8)
    assert np.array_equal(a, b)
    cols = np.array([0, 5, 31])
    c = oracle.w4_linear_columns(x, codes, zeros, scales, None, cs, pairs, theta, G, 8, cols)
    # a BLAS matmul over a column subset may sum in another order
    assert np.max(np.abs(c - b[:, cols])) <= 1e-12 * np.max(np.abs(b))


def test_invalid_group_size_rejected():
    with pytest.raises(ValueError):
        oracle.normalize_group_size(3, 12)
    with pytest.raises(ValueError):
        oracle.normalize_group_size(128, 200)
    assert oracle.normalize_group_size(-1, 96) == 96
