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


def test_spec_fields_and_cpu_baseline_fields():
    """Data-sheet context beside the measured denominators, and the CPU
    baseline's thread counts (the oracle's BLAS threads; the host's cores)."""
    s = bench.spec_fields("hbm", 3850.0)
    assert s == {"peak_spec": 7700.0, "frac_of_spec": 0.5}
    t = bench.spec_fields("tensor", 1125.0)
    assert t == {"peak_spec": 2250.0, "frac_of_spec": 0.5}
    c = bench.cpu_baseline_fields(0.0312345678, "GB/s", "sample text")
    assert c["value"] == 0.03123 and c["unit"] == "GB/s" and c["kind"] == "oracle" and c["sample"] == "sample text"
    assert 1 <= c["cores"] and 1 <= c["host_cores"]
    assert c["cores"] == bench.oracle_threads()

