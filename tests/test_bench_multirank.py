"""The N > 1 path of bench.py on CPU: two gloo ranks (no GPU).

bench.py runs one independent replica of the workload per GPU ("replicas
only": the path has no exchange step).  What is multi-rank is the bookkeeping:
every timed number is the slowest rank's (all_reduce MAX), whole-job
throughput counts every rank's work, and the reference arm runs on rank 0
alone while the other ranks exit without work.  These tests run that logic on
two gloo processes.
"""
import os
import socket
import sys
import types

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # slowest rank decides: rank r took 1 + r ms
        ms = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        value = bench.job_throughput(world, 10, 1e6, ms)
        # reference arm: the oracle is replaced by a stub (its cost is not the point here)
        bench.oracle_sample = lambda workload, budget, max_steps=None: (1.5, "stub sample", 0.01)
        args = types.SimpleNamespace(workload="q_proj_decode", steps=4, warmup=3)
        ref = bench.run_reference(args, rank, world)
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr((ms, value, None if ref is None else (ref["impl"], ref["n_gpus"], ref["value"],
                                                                  ref["config"]["parallelism"]))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = {}
    for r in range(world):
        with open(tmp_path / f"rank{r}.txt") as f:
            got[r] = eval(f.read())
    for r in range(world):
        ms, value, _ = got[r]
        assert ms == 2.0                              # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 10 * 1e6 / 2e-3)
    assert got[0][2] == ("reference", 2, 1.5, "replicas x2")
    assert got[1][2] is None                          # only rank 0 runs the reference arm


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, None) == 3.25
    assert bench.job_throughput(1, 5, 2.0, 1.0) == pytest.approx(10000.0)
