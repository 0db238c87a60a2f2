#!/usr/bin/env python
"""Benchmark of the rotated W4 linear (decode HBM GB/s / prefill TFLOP/s).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload layer|q_proj_decode|mlp_decode|
                 prefill|layer_decode|layer_prefill|quantize_gate_proj] [--impl ours|reference]

One "step" is one pass of the whole hot path (scale + Givens stages + W4
dequant-GEMM) over every call of the workload:
  layer (default): the full Llama-3-8B decoder-layer linear set (q, k, v, o,
                 gate, up, down) at M = 1 (decode, the line's value in HBM GB/s)
                 and at M = 4096 (prefill, TFLOP/s, in the line's "prefill"
                 object); each half is timed, roofline-checked and baselined
                 on its own
  q_proj_decode: Llama-3-8B q_proj 4096->4096, M = 1, 4, 16 (three calls)
  mlp_decode:    gate/up 4096->14336 and down 14336->4096, M = 1 and 8 (six calls)
  prefill:       gate_proj-shaped 4096->14336, M = 2048 and 8192, bias (two calls)
  layer_decode / layer_prefill: the seven linears of a decoder layer at M = 1 / 4096
  quantize_gate_proj: the weight-side step before packing (W_r = W D R,
                 four-bit symmetric codes, AWQ words) on a float gate_proj
                 14336 x 4096, in HBM GB/s (one call per step)
Inputs are seeded synthetic layers (the workload recipe), resident in HBM; the
weights are cycled over enough replicas that every timed call reads its weights
from HBM, not L2.  Prints ONE JSON line on rank 0.

--impl reference times the float64 CPU oracle (the reference arm) on bounded
samples of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
GROUP = 128
KROT = 8

# "groups": linears that read the same x go through one grouped call
# (paro_w4_linear_group: q/k/v and gate/up of a decoder layer)
WORKLOADS = {
    "q_proj_decode": dict(cfg=1, layers=[0], Ms=[1, 4, 16], kind="decode", groups=[[0]]),
    "mlp_decode": dict(cfg=2, layers=[0, 1, 2], Ms=[1, 8], kind="decode", groups=[[0, 1], [2]]),
    "prefill": dict(cfg=3, layers=[0], Ms=[2048, 8192], kind="prefill", groups=[[0]]),
    "layer_decode": dict(cfg=4, layers=list(range(7)), Ms=[1], kind="decode",
                         groups=[[0, 1, 2], [3], [4, 5], [6]]),
    "layer_prefill": dict(cfg=4, layers=list(range(7)), Ms=[4096], kind="prefill",
                          groups=[[0, 1, 2], [3], [4, 5], [6]]),
    "quantize_gate_proj": dict(cfg=2, layers=[0], Ms=[], kind="quantize"),
    # both halves of the decoder-layer set in one line
    "layer": dict(cfg=4, kind="pair", halves=["layer_decode", "layer_prefill"]),
    # stacked experts sharing one rotation: a Mixtral-8x7B-shaped expert gate
    # projection (8 experts of 4096 -> 14336, top-2 routing), decode and prefill
    "moe_decode": dict(kind="moe", E=8, topk=2, K=4096, N=14336, T=1),
    "moe_prefill": dict(kind="moe", E=8, topk=2, K=4096, N=14336, T=4096),
}
REPLAYS = 7          # timed replays of the K-step graph; the median is reported


_LAYERS = {}


def cfg_layers(cfg):
    """The seeded layers of a workload config, drawn once per process (the
    arrays are read, never written)."""
    if cfg not in _LAYERS:
        _LAYERS[cfg] = synth.config_layers(cfg)
    return _LAYERS[cfg]


# ----------------------------------------------------------------- algorithmic cost model
def call_bytes(K, N, M, bias, krot=KROT, rotated=True):
    """Bytes the method itself must move for one call (weights, scales, zeros,
    activations in and out, bias, rotation tables)."""
    b = K * N // 2 + (K // GROUP) * N * 2 + (K // GROUP) * N // 2 + M * K * 2 + M * N * 2
    if bias:
        b += N * 2
    if rotated:
        b += krot * K * 2 + krot * (K // 2) * 4 + K * 4
    return b


def quantize_bytes(K, N, krot=KROT):
    """Bytes of one weight-quantiser call: float W in, quantiser scales in,
    packed weights and zeros out, rotation tables."""
    return (N * K * 2 + (K // GROUP) * N * 2 + K * N // 2 + (K // GROUP) * N // 2
            + krot * K * 2 + krot * (K // 2) * 4 + K * 4)


def gemv_bytes(K, N, M, bias):
    """Bytes of the GEMV kernel alone (reads X_r instead of x; no tables)."""
    return call_bytes(K, N, M, bias, rotated=False)


def call_flops(K, N, M):
    return 2 * M * N * K


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# B200 data-sheet figures, for context beside the measured denominators:
# HBM3e 7.7 TB/s (HGX), dense fp16/bf16 tensor 2.25 PFLOP/s
SPEC_HBM_GBS = 7700.0
SPEC_F16_TFLOPS = 2250.0


def spec_fields(bound, achieved):
    spec = SPEC_HBM_GBS if bound == "hbm" else SPEC_F16_TFLOPS
    return {"peak_spec": spec, "frac_of_spec": round(achieved / spec, 4)}


def fp16_matmul_tflops(device, n=8192, iters=10):
    """torch.matmul (cuBLAS) on fp16 n x n x n, timed with CUDA events on the
    current stream after warm-up: the dense fp16 rate of this GPU in this run,
    a reference beside the bf16 denominator (not part of any timed step)."""
    import torch
    a = torch.randn(n, n, dtype=torch.float16, device=device)
    b = torch.randn(n, n, dtype=torch.float16, device=device)
    c = torch.empty(n, n, dtype=torch.float16, device=device)
    for _ in range(3):
        torch.matmul(a, b, out=c)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        torch.matmul(a, b, out=c)
    e1.record()
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1)
    del a, b, c
    return round(2.0 * n ** 3 * iters / (ms * 1e-3) / 1e12, 1)


def source_digest():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "rotation_w4_weight_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
        e = t.get(kernel_key)
        if e and e.get("src") == source_digest():
            return e.get("bytes_per_launch")
    except Exception:
        pass
    return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a window."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- multi-rank helpers
def max_over_ranks(value, world, device):
    """The largest `value` over all ranks (identity for one rank): every timed
    number of a multi-GPU run is the slowest rank's."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps, per_step, ms):
    """Whole-job throughput: every rank runs `steps` steps of `per_step` units
    (bytes or flops) in `ms` milliseconds (the slowest rank's time)."""
    return world * steps * per_step / (ms * 1e-3)


def timed_replays(replay, stream, world, device, replays=REPLAYS):
    """Times `replays` runs of `replay()` (one CUDA graph of exactly K steps)
    with CUDA events on `stream`, each bracketed by a barrier and device syncs.
    Returns the per-replay milliseconds, each the max over ranks."""
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    out = []
    for _ in range(replays):
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)
        e0.record(stream)
        replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        out.append(max_over_ranks(e0.elapsed_time(e1), world, device))
    return out


def spread(ms_list, steps):
    """Median, fastest and slowest replay, per step (ms)."""
    return {"replays": len(ms_list), "median_ms_per_step": round(statistics.median(ms_list) / steps, 5),
            "min_ms_per_step": round(min(ms_list) / steps, 5),
            "max_ms_per_step": round(max(ms_list) / steps, 5)}


def workload_config(workload, world):
    """The workload description shared by both arms' JSON lines."""
    wl = WORKLOADS[workload]
    if wl["kind"] == "moe":
        return {"workload": workload, "experts": wl["E"], "topk": wl["topk"], "K": wl["K"], "N": wl["N"],
                "tokens": wl["T"], "routing": "seeded uniform top-k without repeats, a new draw every call",
                "group_size": GROUP, "krot": KROT, "accumulate": "f32", "parallelism": f"replicas x{world}"}
    if wl["kind"] == "pair":
        dec, pre = (workload_config(h, world) for h in wl["halves"])
        return {"workload": workload, "layers": dec["layers"], "calls": dec["calls"],
                "M": {"decode": dec["M"], "prefill": pre["M"]}, "group_size": GROUP, "krot": KROT,
                "accumulate": "f32", "parallelism": f"replicas x{world}",
                "rotation": {"decode": dec["rotation"], "prefill": pre["rotation"]}}
    layers = [synth.config_layer_shapes(wl["cfg"])[i] for i in wl["layers"]]
    if wl["kind"] == "quantize":
        return {"workload": workload, "weights": [(n, N, K) for n, K, N in layers],
                "input": "float W fp16 [N, K] and quantiser scales fp16 [K/128, N]",
                "group_size": GROUP, "krot": KROT, "parallelism": f"replicas x{world}"}
    return {"workload": workload, "layers": [(n, K, N) for n, K, N in layers], "M": wl["Ms"],
            "calls": [[layers[i][0] for i in g] for g in wl["groups"]],
            "group_size": GROUP, "krot": KROT, "accumulate": "f32", "parallelism": f"replicas x{world}",
            "rotation": ("stages pair by pair per call" if wl["kind"] == "decode" else
                         "X R' on the tensor cores, R' prepared once per layer outside the timed region")}


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank, workload=None):
    import torch
    import rotation_w4_weight_b200 as pb

    workload = workload or args.workload
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[workload]
    layers = [cfg_layers(wl["cfg"])[i] for i in wl["layers"]]
    Ms = wl["Ms"]
    decode = wl["kind"] == "decode"

    def T(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # one packed copy of each layer, then device replicas so the timed calls stream from HBM
    base = []
    for lay in layers:
        qw, qz = pb.pack_awq(T(lay.codes), T(lay.zero_codes), GROUP)
        base.append(dict(lay=lay, qweight=qw, qzeros=qz, scales=T(lay.scales), bias=T(lay.bias),
                         cs=T(lay.channel_scales), pairs=T(lay.pairs), theta=T(lay.theta)))
        # prefill: the layer's R' is a layer constant, built once at load time
        # (as the packed weights are) and passed with every call
        base[-1]["rmat"] = (None if decode else
                            pb.rotation_matrix(base[-1]["cs"], base[-1]["pairs"], base[-1]["theta"], lay.K,
                                               GROUP, KROT))
    weight_bytes = sum(l.K * l.N // 2 + (l.K // GROUP) * l.N * 5 // 2 for l in layers)
    reps = max(1, min(64, -(-3 * L2_BYTES // weight_bytes)))
    replicas = []
    for r in range(reps):
        replicas.append([{k: (v.clone() if torch.is_tensor(v) and k in ("qweight", "qzeros", "scales") else v)
                          for k, v in b.items()} for b in base])
    calls = [(li, M) for li in range(len(layers)) for M in Ms]
    groups = wl["groups"]
    gcalls = [(gi, M) for gi in range(len(groups)) for M in Ms]
    # members of a group share their first layer's activations
    xs = {}
    for gi, M in gcalls:
        xg = T(synth.make_activations(layers[groups[gi][0]], M))
        for li in groups[gi]:
            xs[(li, M)] = xg
    ys = {(li, M): torch.empty((M, layers[li].N), dtype=torch.float16, device=dev) for li, M in calls}
    ws = {(gi, M): torch.empty(max(256, sum(pb.w4_linear_workspace_size(M, layers[li].K, layers[li].N)
                                            for li in groups[gi])), dtype=torch.uint8, device=dev)
          for gi, M in gcalls}
    xrs = {(li, M): torch.empty((M, layers[li].K), dtype=torch.float16, device=dev) for li, M in calls}

    def launches(gi, M, rotate=True):
        grp = groups[gi]
        return pb.w4_linear_group_launches(
            M, layers[grp[0]].K, [dict(N=layers[li].N, krot=KROT if rotate else 0, channel_scales=rotate,
                                       rmat=rotate and not decode) for li in grp], GROUP)

    stream = torch.cuda.Stream(device=dev)
    step_bytes = sum(call_bytes(layers[li].K, layers[li].N, M, layers[li].bias is not None)
                     for li, M in calls)
    step_flops = sum(call_flops(layers[li].K, layers[li].N, M) for li, M in calls)

    def member(b, rotate=True):
        return dict(qweight=b["qweight"], qzeros=b["qzeros"], scales=b["scales"], bias=b["bias"],
                    channel_scales=b["cs"] if rotate else None, pairs=b["pairs"] if rotate else None,
                    theta=b["theta"] if rotate else None, krot=KROT if rotate else 0,
                    rmat=b["rmat"] if rotate else None)

    def one_call(rep, gi, M):
        grp = groups[gi]
        if len(grp) == 1:
            li = grp[0]
            b = replicas[rep][li]
            pb.w4_linear(xs[(li, M)], b["qweight"], b["qzeros"], b["scales"], b["bias"], b["cs"],
                         b["pairs"], b["theta"], GROUP, KROT, workspace=ws[(gi, M)], out=ys[(li, M)],
                         stream=stream, rmat=b["rmat"])
        else:
            pb.w4_linear_group(xs[(grp[0], M)], [member(replicas[rep][li]) for li in grp], GROUP,
                               workspace=ws[(gi, M)], out=[ys[(li, M)] for li in grp], stream=stream)

    def one_step(i):
        for c, (gi, M) in enumerate(gcalls):
            one_call((i * len(gcalls) + c) % reps, gi, M)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
    torch.cuda.synchronize(dev)
    assert pb.device_status() == pb.PARO_OK

    # capture the K timed steps as one CUDA graph (launch-bound decode calls)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(args.steps):
            one_step(args.warmup + i)
    def replay(graph):
        with torch.cuda.stream(stream):          # a graph replays on the current stream
            graph.replay()

    replay(g)                                    # untimed graph warm-up
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    t_end = time.time() + 0.6
    while time.time() < t_end:                   # load before the window so clocks settle
        replay(g)
        torch.cuda.synchronize(dev)
    step_ms = timed_replays(lambda: replay(g), stream, world, dev)
    ms = statistics.median(step_ms)
    t_end = time.time() + 0.4
    while time.time() < t_end:
        replay(g)
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    assert pb.device_status() == pb.PARO_OK
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    # ---- dominant kernel, timed live: X_r is produced once per call shape by
    #      paro_rotate (outside the timed graph); the graph holds the GEMV/GEMM
    #      launches alone, exactly as paro_w4_linear issues them after rotating.
    for li, M in calls:
        b = replicas[0][li]
        pb.rotate(xs[(li, M)], b["cs"], b["pairs"], b["theta"], GROUP, KROT, out=xrs[(li, M)],
                  stream=stream)
    kern_bytes = 0
    kern_flops = 0
    n_launch = 0
    # (a group's GEMV reads the first member's X_r for every member: the same
    # bytes and work as the members' own X_r)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=stream):
        for i in range(args.steps):
            for c, (gi, M) in enumerate(gcalls):
                rep = (i * len(gcalls) + c) % reps
                grp = groups[gi]
                if len(grp) == 1:
                    b = replicas[rep][grp[0]]
                    pb.w4_linear(xrs[(grp[0], M)], b["qweight"], b["qzeros"], b["scales"], b["bias"],
                                 None, None, None, GROUP, 0, out=ys[(grp[0], M)], stream=stream)
                else:
                    pb.w4_linear_group(xrs[(grp[0], M)], [member(replicas[rep][li], False) for li in grp],
                                       GROUP, out=[ys[(li, M)] for li in grp], stream=stream)
                for li in grp:
                    lay = layers[li]
                    kern_bytes += gemv_bytes(lay.K, lay.N, M, lay.bias is not None)
                    kern_flops += call_flops(lay.K, lay.N, M)
                n_launch += launches(gi, M, rotate=False)
    replay(g2)
    torch.cuda.synchronize(dev)
    # rotated and unrotated graphs timed in alternation, so both see the same
    # clock and power state (timed one after the other, the second ran in a
    # different state under the power cap)
    rot_list, kern_list = [], []
    for _ in range(REPLAYS):
        rot_list += timed_replays(lambda: replay(g), stream, world, dev, replays=1)
        kern_list += timed_replays(lambda: replay(g2), stream, world, dev, replays=1)
    kern_ms = statistics.median(kern_list)
    rot_ms = statistics.median(rot_list)
    peaks = load_peaks()
    if decode:
        achieved = kern_bytes / (kern_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm"], 4),
                "traffic": traffic_for(workload),
                "kernel": "w4_gemv_kernel (decode GEMV, split-K cluster)",
                "avg_launch_us": round(kern_ms * 1e3 / n_launch, 3),
                "bytes_per_launch": kern_bytes // n_launch, "peak_source": peaks["src"],
                **spec_fields("hbm", achieved)}
    else:
        # the GEMM graph runs for many milliseconds under the power cap: the
        # sustained dense peak is its denominator (the burst one is for a kernel timed alone)
        achieved = kern_flops / (kern_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_sus"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_sus"], 4),
                "traffic": traffic_for(workload),
                "kernel": "w4_tc_gemm_kernel (prefill tcgen05 GEMM)", "avg_launch_us": round(kern_ms * 1e3 / n_launch, 3),
                "flops_per_launch": kern_flops // n_launch,
                "peak_source": peaks["src"] + " bf16 sustained (fp16 runs at the bf16 rate)",
                "peak_burst": peaks["bf16"], "frac_of_burst": round(achieved / peaks["bf16"], 4),
                "fp16_matmul_tflops": fp16_matmul_tflops(dev), **spec_fields("tensor", achieved)}
    del g2

    # ---- end to end through the public call with host buffers (pinned), per step:
    #      H2D of the step's activations, the calls, D2H of the outputs
    hx = {(groups[gi][0], M): xs[(groups[gi][0], M)].cpu().pin_memory() for gi, M in gcalls}
    hy = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in ys.items()}
    h2d = sum(v.numel() * 2 for v in hx.values())
    d2h = sum(v.numel() * 2 for v in hy.values())
    e_steps = max(1, min(args.steps, 200 if decode else 20))

    def e2e_step(i):
        for c, (gi, M) in enumerate(gcalls):
            grp = groups[gi]
            xs[(grp[0], M)].copy_(hx[(grp[0], M)], non_blocking=True)
            one_call((i * len(gcalls) + c) % reps, gi, M)
            for li in grp:
                hy[(li, M)].copy_(ys[(li, M)], non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(e_steps):
            e2e_step(i)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e_steps

    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    if decode:
        value = job_throughput(world, args.steps, step_bytes, ms) / 1e9
        unit = "GB/s"
        e2e_val = job_throughput(world, 1, step_bytes, e2e_ms) / 1e9
    else:
        value = job_throughput(world, args.steps, step_flops, ms) / 1e12
        unit = "TFLOP/s"
        e2e_val = job_throughput(world, 1, step_flops, e2e_ms) / 1e12
    metric = metric_name(workload)

    out = {
        "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": dict(workload_config(workload, world),
                       l2=f"weights cycled over {reps} device replicas "
                          f"({reps * weight_bytes / 2**20:.0f} MiB > 3x L2)",
                       timing=f"median of {len(step_ms)} replays of a CUDA graph of the K steps, "
                              "CUDA events, max over ranks"),
        "timing": spread(step_ms, args.steps),
        "roofline": roof,
        "e2e": {"value": round(e2e_val, 2), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "how": "pinned host x -> device, paro_w4_linear calls, device y -> pinned host; no graph"},
        # the same calls with krot = 0 and no channel scales are the GEMV/GEMM
        # graph timed for the roofline: the fused path's cost over it
        "rotation_overhead": {"frac": round(rot_ms / kern_ms - 1.0, 4),
                              "ms_per_step_rotated": round(rot_ms / args.steps, 5),
                              "ms_per_step_unrotated": round(kern_ms / args.steps, 5),
                              "rotated_timing": spread(rot_list, args.steps),
                              "unrotated_timing": spread(kern_list, args.steps),
                              "how": "same K steps as CUDA graphs; unrotated = krot 0, no channel "
                                     "scales, same kernels on X_r; the two graphs' replays "
                                     "alternate, medians of each"},
        "gpu_launches": sum(launches(gi, M) for gi, M in gcalls) * args.steps,
        "clocks": clocks,
        "bytes_per_step": step_bytes, "flops_per_step": step_flops,
    }
    return out


def run_pair(args, rank, world, local_rank):
    """Both halves of a paired workload (decode at the line's top level, prefill
    in its "prefill" object), one after the other on the same GPU."""
    import torch
    wl = WORKLOADS[args.workload]
    dec_name, pre_name = wl["halves"]
    dec = run_ours(args, rank, world, local_rank, dec_name)
    torch.cuda.empty_cache()
    pre = run_ours(args, rank, world, local_rank, pre_name)
    torch.cuda.empty_cache()
    out = dict(dec)
    out["metric"] = metric_name(args.workload)
    out["config"] = dict(workload_config(args.workload, world), l2=dec["config"]["l2"],
                         timing=dec["config"]["timing"])
    out["decode_workload"] = dec_name
    out["prefill"] = {k: pre[k] for k in ("metric", "value", "unit", "ms_per_step", "timing", "roofline",
                                          "e2e", "rotation_overhead", "gpu_launches", "clocks",
                                          "bytes_per_step", "flops_per_step")}
    out["prefill"]["workload"] = pre_name
    out["prefill"]["steps"] = args.steps
    return out


# ----------------------------------------------------------------- weight quantiser
def run_quantize(args, rank, world, local_rank):
    """paro_quantize_w4 on a float gate_proj: one call per step, inputs resident
    in HBM and cycled over replicas larger than L2 together."""
    import torch
    import rotation_w4_weight_b200 as pb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    lay = cfg_layers(wl["cfg"])[wl["layers"][0]]
    W, qs = synth.make_float_weight(lay)

    def T(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    Wd, qsd = T(W), T(qs)
    cs, pairs, theta = T(lay.channel_scales), T(lay.pairs), T(lay.theta)
    reps = max(2, -(-3 * L2_BYTES // (W.nbytes + qs.nbytes)))
    Ws = [Wd] + [Wd.clone() for _ in range(reps - 1)]
    outs = [(torch.empty((lay.K, lay.N // 8), dtype=torch.int32, device=dev),
             torch.empty((lay.K // GROUP, lay.N // 8), dtype=torch.int32, device=dev)) for _ in range(2)]
    per_call = quantize_bytes(lay.K, lay.N)
    stream = torch.cuda.Stream(device=dev)
    qws = torch.empty(pb.paro_quantize_w4_workspace_size(lay.K), dtype=torch.uint8, device=dev)

    def one_step(i):
        pb.quantize_w4(Ws[i % reps], cs, pairs, theta, qsd, GROUP, KROT, out=outs[i % 2], stream=stream,
                       method="tensor", workspace=qws)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
    torch.cuda.synchronize(dev)
    assert pb.device_status() == pb.PARO_OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(args.steps):
            one_step(args.warmup + i)

    def replay():
        with torch.cuda.stream(stream):
            g.replay()

    replay()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    t_end = time.time() + 0.6
    while time.time() < t_end:
        replay()
        torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)
    t_end = time.time() + 0.4
    while time.time() < t_end:
        replay()
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = max_over_ranks(ms, world, dev)
    assert pb.device_status() == pb.PARO_OK
    del g

    # two kernels per call (the R'' build, ~9 us, and the quantising product):
    # the roofline takes the whole call, so it understates the product kernel
    peaks = load_peaks()
    achieved = per_call * args.steps / (ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm"], 4), "traffic": traffic_for("quantize_gate_proj"),
            "kernel": "rotate_tc_kernel<__half, true> (weight quantiser on the tensor cores) + R'' build, per call",
            "avg_launch_us": round(ms * 1e3 / args.steps, 3), "bytes_per_launch": per_call,
            "peak_source": peaks["src"], **spec_fields("hbm", achieved)}

    # end to end through the public call with host buffers: pinned W in, packed words out
    hW = Ws[0].cpu().pin_memory()
    hq = (torch.empty(outs[0][0].shape, dtype=torch.int32).pin_memory(),
          torch.empty(outs[0][1].shape, dtype=torch.int32).pin_memory())
    e_steps = max(1, min(args.steps, 20))

    def e2e_step():
        Ws[0].copy_(hW, non_blocking=True)
        pb.quantize_w4(Ws[0], cs, pairs, theta, qsd, GROUP, KROT, out=outs[0], stream=stream, method="tensor",
                       workspace=qws)
        hq[0].copy_(outs[0][0], non_blocking=True)
        hq[1].copy_(outs[0][1], non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)

    return {
        "metric": metric_name(args.workload),
        "value": round(job_throughput(world, args.steps, per_call, ms) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(args.workload, world),
                       l2=f"float weights cycled over {reps} device replicas "
                          f"({reps * (W.nbytes + qs.nbytes) / 2**20:.0f} MiB > 3x L2)",
                       timing="CUDA graph of the K steps, CUDA events, max over ranks"),
        "roofline": roof,
        "e2e": {"value": round(job_throughput(world, 1, per_call, e2e_ms) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(hW.numel() * 2),
                "d2h_bytes_per_step": int((hq[0].numel() + hq[1].numel()) * 4),
                "ms_per_step": round(e2e_ms, 4),
                "how": "pinned host W -> device, paro_quantize_w4_tc, packed words -> pinned host; no graph"},
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "bytes_per_step": per_call,
    }


def moe_setup(wl, seed=0):
    """The workload's experts (codes, zero points, scales per expert; no bias)
    and the shared rotation, drawn once per process."""
    key = ("moe", wl["E"], wl["K"], wl["N"], seed)
    if key not in _LAYERS:
        lays = [synth.make_layer(f"expert{e}", wl["K"], wl["N"], seed=1000 + 17 * e, krot=KROT,
                                 zero_point=None) for e in range(wl["E"])]
        _LAYERS[key] = lays
    return _LAYERS[key]


def moe_routing(wl, calls, seed=0):
    rng = np.random.default_rng(seed)
    return [np.stack([rng.choice(wl["E"], wl["topk"], replace=False) for _ in range(wl["T"])]).astype(np.int32)
            for _ in range(calls)]


def moe_call_bytes(wl, idx):
    """Bytes one call must move: x, the distinct selected experts' weights,
    scales and zero words, and y."""
    K, N = wl["K"], wl["N"]
    experts = len(np.unique(idx))
    return (wl["T"] * K * 2 + experts * (K * N // 2 + (K // GROUP) * N * 2 + (K // GROUP) * N // 2)
            + idx.size * N * 2)


def run_moe(args, rank, world, local_rank):
    """paro_w4_moe_linear on the workload's experts: one call per step with a
    fresh routing, experts resident in HBM (8 experts > L2 together)."""
    import torch
    import rotation_w4_weight_b200 as pb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    lays = moe_setup(wl)
    rot = lays[0]

    def T(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    qw, qz = zip(*[pb.pack_awq(T(l.codes), T(l.zero_codes), GROUP) for l in lays])
    qweight, qzeros = torch.stack(qw).contiguous(), torch.stack(qz).contiguous()
    del qw, qz
    scales = T(np.stack([l.scales for l in lays]))
    cs, pairs, theta = T(rot.channel_scales), T(rot.pairs), T(rot.theta)
    routes = moe_routing(wl, 64)
    idx_d = [T(r) for r in routes]
    xs = [T(synth.make_activations(rot, wl["T"], seed=i)) for i in range(4)]
    out = torch.empty((wl["T"], wl["topk"], wl["N"]), dtype=torch.float16, device=dev)
    ws = torch.empty(pb.paro_w4_moe_workspace_size(wl["T"], wl["K"], wl["N"], wl["E"], wl["topk"], GROUP),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    decode = wl["T"] <= 16

    def one_step(i):
        pb.w4_moe_linear(xs[i % len(xs)], idx_d[i % len(idx_d)], qweight, qzeros, scales, None, cs, pairs, theta,
                         GROUP, KROT, workspace=ws, out=out, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
    torch.cuda.synchronize(dev)
    assert pb.device_status() == pb.PARO_OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(args.steps):
            one_step(args.warmup + i)

    def replay():
        with torch.cuda.stream(stream):
            g.replay()

    replay()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    t_end = time.time() + 0.6
    while time.time() < t_end:
        replay()
        torch.cuda.synchronize(dev)
    step_ms = timed_replays(replay, stream, world, dev)
    ms = statistics.median(step_ms)
    clocks = sampler.stop()
    assert pb.device_status() == pb.PARO_OK
    del g
    bytes_steps = sum(moe_call_bytes(wl, routes[(args.warmup + i) % len(routes)]) for i in range(args.steps))
    flops_per = 2 * wl["T"] * wl["topk"] * wl["K"] * wl["N"]
    peaks = load_peaks()
    step_s = ms * 1e-3 / args.steps
    if decode:
        achieved = bytes_steps / args.steps / step_s / 1e9
        value, unit = job_throughput(world, args.steps, bytes_steps / args.steps, ms) / 1e9, "GB/s"
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "traffic": None,
                "kernel": "whole call (rotation, routing with the gather of the routed rows, expert GEMV segments)",
                "avg_launch_us": round(step_s * 1e6, 3), "bytes_per_launch": int(bytes_steps / args.steps),
                "peak_source": peaks["src"], **spec_fields("hbm", achieved)}
    else:
        achieved = flops_per / step_s / 1e12
        value, unit = job_throughput(world, args.steps, flops_per, ms) / 1e12, "TFLOP/s"
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_sus"], 4), "traffic": None,
                "kernel": "whole call (rotation, routing, gather, expert GEMM tiles)",
                "avg_launch_us": round(step_s * 1e6, 3), "flops_per_launch": flops_per,
                "peak_source": "measured bf16 sustained (fp16 runs at the bf16 rate)",
                **spec_fields("tensor", achieved)}
    return {
        "metric": metric_name(args.workload), "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": dict(workload_config(args.workload, world),
                       l2=f"{wl['E']} experts resident ({wl['E'] * wl['K'] * wl['N'] // 2 / 2**20:.0f} MiB > L2)",
                       timing=f"median of {REPLAYS} replays of a CUDA graph of the K steps, CUDA events"),
        "timing": spread(step_ms, args.steps), "roofline": roof,
        "gpu_launches": pb.w4_moe_launches(wl["T"], wl["K"], wl["N"], wl["E"], wl["topk"], GROUP, KROT) * args.steps,
        "clocks": clocks,
    }


def moe_oracle_sample(workload, budget_s, max_steps=None):
    """The float64 oracle's stacked-expert layer on column samples (64 columns
    of every expert, full rotation per call), until `budget_s` seconds."""
    import oracle
    wl = WORKLOADS[workload]
    lays = moe_setup(wl)
    rot = lays[0]
    routes = moe_routing(wl, 4)
    rng = np.random.default_rng(0)
    done = t_total = 0.0
    n = 0
    ncols = 64
    while True:
        cols = np.sort(rng.choice(wl["N"], ncols, replace=False))
        idx = routes[n % len(routes)]
        x = synth.make_activations(rot, wl["T"], seed=n)
        codes = np.stack([l.codes[cols] for l in lays])
        zeros = np.stack([l.zero_codes[cols] for l in lays])
        scales = np.stack([l.scales[:, cols] for l in lays])
        t0 = time.perf_counter()
        oracle.moe_linear_from_codes(x, idx, codes, zeros, scales, None, rot.channel_scales, rot.pairs,
                                     rot.theta, GROUP, KROT)
        t_total += time.perf_counter() - t0
        frac = ncols / wl["N"]
        done += (moe_call_bytes(wl, idx) * frac if wl["T"] <= 16 else
                 2 * wl["T"] * wl["topk"] * wl["K"] * wl["N"] * frac)
        n += 1
        if t_total >= budget_s or (max_steps and n >= max_steps):
            unit = 1e9 if wl["T"] <= 16 else 1e12
            desc = (f"float64 oracle on {n} calls of {workload} restricted to {ncols} sampled output columns "
                    f"of every expert (full rotation per call)")
            return done / t_total / unit, desc, t_total


def quantize_oracle_sample(workload, budget_s, max_steps=None):
    """The float64 oracle's weight quantiser on row samples of the workload's
    weight (256 rows per sample), until `budget_s` seconds or max_steps samples."""
    import oracle
    wl = WORKLOADS[workload]
    lay = cfg_layers(wl["cfg"])[wl["layers"][0]]
    W, qs = synth.make_float_weight(lay)
    rng = np.random.default_rng(0)
    done = 0.0
    t_total = 0.0
    n = 0
    rows_per = 256
    while True:
        rows = np.sort(rng.choice(lay.N, rows_per, replace=False))
        t0 = time.perf_counter()
        oracle.quantize_weight(W[rows], lay.channel_scales, lay.pairs, lay.theta, qs[:, rows], GROUP, KROT)
        t_total += time.perf_counter() - t0
        done += quantize_bytes(lay.K, lay.N) * rows_per / lay.N
        n += 1
        if t_total >= budget_s or (max_steps and n >= max_steps):
            desc = (f"float64 oracle weight quantiser on {n} samples of {rows_per} rows of "
                    f"{lay.name} {lay.N}x{lay.K} (transform, quantise, pack)")
            return done / t_total / 1e9, desc, t_total


# ----------------------------------------------------------------- CPU oracle (baseline / reference)
def oracle_threads():
    """Threads the oracle actually uses: its matmuls run on NumPy's BLAS thread
    pool, everything else on one thread."""
    try:
        from threadpoolctl import threadpool_info
        n = [int(i["num_threads"]) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline_fields(val, unit, desc):
    return {"value": round(val, 5), "unit": unit, "cores": oracle_threads(),
            "host_cores": len(os.sched_getaffinity(0)), "kind": "oracle", "sample": desc}


def oracle_sample(workload, budget_s, max_steps=None):
    """Times the float64 oracle on column samples of the workload's calls until
    `budget_s` seconds of CPU work (or max_steps samples) are done.  Returns
    (value in the workload's unit, description, seconds)."""
    import oracle
    wl = WORKLOADS[workload]
    if wl["kind"] == "quantize":
        return quantize_oracle_sample(workload, budget_s, max_steps)
    if wl["kind"] == "moe":
        return moe_oracle_sample(workload, budget_s, max_steps)
    layers = [cfg_layers(wl["cfg"])[i] for i in wl["layers"]]
    decode = wl["kind"] == "decode"
    rng = np.random.default_rng(0)
    done_bytes = done_flops = 0.0
    t_total = 0.0
    n = 0
    ncols = 512 if decode else 64
    while True:
        for lay in layers:
            for M in wl["Ms"]:
                x = synth.make_activations(lay, M)
                cols = np.sort(rng.choice(lay.N, min(ncols, lay.N), replace=False))
                t0 = time.perf_counter()
                oracle.w4_linear_columns(x, lay.codes, lay.zero_codes, lay.scales, lay.bias,
                                         lay.channel_scales, lay.pairs, lay.theta, GROUP, KROT, cols)
                t_total += time.perf_counter() - t0
                frac = len(cols) / lay.N
                done_bytes += call_bytes(lay.K, lay.N, M, lay.bias is not None) * frac
                done_flops += call_flops(lay.K, lay.N, M) * frac
                n += 1
                if t_total >= budget_s or (max_steps and n >= max_steps):
                    val = (done_bytes / t_total / 1e9) if decode else (done_flops / t_total / 1e12)
                    desc = (f"float64 oracle on {n} calls of {workload} restricted to {ncols} "
                            f"sampled output columns each (full rotation per call)")
                    return val, desc, t_total


def metric_name(workload):
    if WORKLOADS[workload]["kind"] == "pair":
        return ("rotated W4 linear, Llama-3-8B decoder-layer linear set: decode HBM GB/s at M=1 "
                "(value) and prefill TFLOP/s at M=4096 (prefill.value), % of roofline")
    if WORKLOADS[workload]["kind"] == "quantize":
        return f"weight quantiser HBM throughput ({workload})"
    if WORKLOADS[workload]["kind"] == "moe":
        return ("stacked-expert rotated W4 linear " +
                ("decode HBM throughput" if WORKLOADS[workload]["T"] <= 16 else "prefill tensor throughput") +
                f" ({workload})")
    decode = WORKLOADS[workload]["kind"] == "decode"
    return ("rotated W4 linear decode HBM throughput" if decode else
            "rotated W4 linear prefill tensor throughput") + f" ({workload})"


def reference_half(workload, steps, warmup, world):
    """One workload of the reference arm: the oracle on bounded samples."""
    wl = WORKLOADS[workload]
    decode = wl["kind"] in ("decode", "quantize") or (wl["kind"] == "moe" and wl["T"] <= 16)
    per_step_budget = max(0.2, min(2.0, 150.0 / max(1, steps + warmup)))
    oracle_sample(workload, per_step_budget * warmup, max_steps=warmup)
    val, desc, secs = oracle_sample(workload, per_step_budget * steps, max_steps=max(1, steps))
    unit = "GB/s" if decode else "TFLOP/s"
    return {
        "impl": "reference", "metric": metric_name(workload),
        "value": round(val, 5), "unit": unit, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(secs * 1e3 / max(1, steps), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": dict(workload_config(workload, world), timing="host wall clock of the oracle"),
        "cpu_baseline": cpu_baseline_fields(val, unit, desc),
        "e2e": {"value": round(val, 5), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle, on rank 0 only (other ranks return
    None and exit without work)."""
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    if wl["kind"] != "pair":
        return reference_half(args.workload, args.steps, args.warmup, world)
    dec_name, pre_name = wl["halves"]
    # both halves share the few minutes the arm may take
    dec = reference_half(dec_name, max(1, args.steps // 2), args.warmup, world)
    pre = reference_half(pre_name, max(1, args.steps // 2), args.warmup, world)
    dec["metric"] = metric_name(args.workload)
    dec["steps"] = args.steps
    dec["config"] = dict(workload_config(args.workload, world), timing="host wall clock of the oracle")
    dec["prefill"] = {k: pre[k] for k in ("metric", "value", "unit", "ms_per_step", "cpu_baseline", "e2e")}
    return dec


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="layer")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle CPU work for the cpu_baseline field")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    wl = WORKLOADS[args.workload]
    if wl["kind"] == "quantize":
        out = run_quantize(args, rank, world, local_rank)
    elif wl["kind"] == "moe":
        out = run_moe(args, rank, world, local_rank)
    elif wl["kind"] == "pair":
        out = run_pair(args, rank, world, local_rank)
    else:
        out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if wl["kind"] == "pair":
            for half, obj in zip(wl["halves"], (out, out["prefill"])):
                val, desc, _ = oracle_sample(half, args.cpu_budget / 2)
                obj["cpu_baseline"] = cpu_baseline_fields(val, obj["unit"], desc)
        else:
            val, desc, _ = oracle_sample(args.workload, args.cpu_budget)
            out["cpu_baseline"] = cpu_baseline_fields(val, out["unit"], desc)
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
