"""The algorithmic cost model behind bench.py's throughput and roofline
numbers: bytes the method itself must move per call (int4 weights, group
scales and zeros, activations in and out, bias, rotation tables) and 2*M*N*K
flops, at the Llama-3-8B shapes of the workloads (no GPU needed)."""
import math

import bench


def test_decode_bytes_per_call():
    # q_proj 4096 -> 4096 at M = 1, 4, 16; gate/up 4096 -> 14336 and down 14336 -> 4096 at M = 1, 8
    # (q_proj, M = 1: 8388608 weights + 262144 scales + 65536 zeros + 8192 x + 8192 y + 147456 tables)
    expect = {(4096, 4096, 1): 8880128, (4096, 4096, 4): 8929280, (4096, 4096, 16): 9125888,
              (4096, 14336, 1): 30691328, (4096, 14336, 8): 30949376,
              (14336, 4096, 1): 31059968, (14336, 4096, 8): 31318016}
    for (K, N, M), b in expect.items():
        assert bench.call_bytes(K, N, M, False) == b, (K, N, M)


def test_weight_stream_dominates_and_tables_are_counted_once():
    K, N = 4096, 4096
    weights = K * N // 2 + (K // 128) * N * 2 + (K // 128) * N // 2
    tables = 8 * K * 2 + 8 * (K // 2) * 4 + K * 4
    assert bench.call_bytes(K, N, 1, False) == weights + 1 * K * 2 + 1 * N * 2 + tables
    # the GEMV alone reads X_r instead of x and no tables
    assert bench.gemv_bytes(K, N, 1, False) == weights + K * 2 + N * 2
    # bias adds N fp16 values
    assert bench.call_bytes(K, N, 1, True) - bench.call_bytes(K, N, 1, False) == N * 2


def test_prefill_flops():
    assert math.isclose(bench.call_flops(4096, 14336, 2048) / 1e9, 240.5, rel_tol=1e-3)
    assert math.isclose(bench.call_flops(4096, 14336, 8192) / 1e9, 962.1, rel_tol=1e-3)


def test_quantiser_bytes():
    K, N = 4096, 14336
    expect = N * K * 2 + (K // 128) * N * 2 + K * N // 2 + (K // 128) * N // 2 + 8 * K * 2 + 8 * (K // 2) * 4 + K * 4
    assert bench.quantize_bytes(K, N) == expect
