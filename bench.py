#!/usr/bin/env python
"""Benchmark of the KDA forward/prefill pass on B200: one JSON line on rank 0.

Workload: B=4, T=32768, H=32, K=V=128 (the long-context prefill the headline
metric is quoted on), bf16 q/k/v/g/beta, g ~ N(0, 2), no initial state, fp32
final state out.  Inputs are synthetic and seeded, generated on the device with
the same distributions as ``kda_inputs`` (the recipe); they total ~5.4 GB, far
above the 126 MB L2, so no explicit flush is needed between steps.

A step is one kda_fwd call over the whole batch (every step of the hot path).
``value`` is tokens/s over the timed steps (device time, CUDA events, max over
ranks); ``e2e`` is the same metric through ``kda_fwd_host`` with pinned host
buffers and the host<->device copies inside the timed region.

Multi-GPU: one process per GPU (torchrun), each rank runs its own batch of the
same shape (independent sequences; KDA has no cross-sequence term), so scaling
is weak and there is no collective on the data path.

``--impl reference`` times the fp64 CPU oracle (token-by-token recurrence) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(name="long_B4_T32768_H32_g2", B=4, T=32768, H=32, K=128, V=128, g_std=2.0)
METRIC = "KDA fwd prefill tokens/s (H=32,K=V=128, T=32K) and % of roofline"
UNIT = "tokens/s"
BYTES_PER_TOKEN_HEAD = 4 * 256 + 2 + 256  # q,k,v,g + beta in, out written (bf16)
STATE_BYTES = 128 * 128 * 4  # fp32 final state per (sequence, head)
FLOPS_PER_TOKEN_HEAD = 140629  # chunked algorithm at C=64, D=128 (triangles halved)
FALLBACK_HBM_GBS = 6650.0
KERNEL = "chunk_kernel"  # the one kernel of a kda_fwd call
KERNEL_SRC = ["linear_attention_09_b200/csrc/kda_chunk.cu", "linear_attention_09_b200/csrc/sm100.cuh"]
PROFILE = "chunk_kernel_long_B4_T32768_H32.md"  # ncu summary: traffic per launch + source hash
# arithmetic of the path: bf16 in/out; tf32, fp16 and bf16 tensor-core products with fp32
# accumulation; fp32 activations, solve and state
DTYPE = "bf16-io/tf32+fp16+bf16-mma/fp32-acc"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=3)
    # profiling aids: a smaller batch / sequence of the same workload (default: the full one)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--seqlen", type=int, default=None)
    ap.add_argument("--heads", type=int, default=None)
    # the decode step (one token per sequence, state in HBM) instead of the prefill
    ap.add_argument("--op", default="prefill", choices=["prefill", "decode", "backward"])
    ap.add_argument("--bwd-schedule", default="chunked", choices=["chunked", "token"],
                    help="schedule of kda_bwd for --op backward")
    ap.add_argument("--decode-seqs", type=int, default=256)
    # time one of the five parity workloads (kda_inputs recipe) instead of the headline
    ap.add_argument("--config-id", type=int, default=None, choices=[0, 1, 2, 3, 4])
    ap.add_argument("--schedule", default="auto", choices=["auto", "fused", "split"],
                    help="forward kernel schedule (kda_set_schedule); auto picks per launch")
    a = ap.parse_args()
    if a.batch:
        WORKLOAD["B"] = a.batch
    if a.seqlen:
        WORKLOAD["T"] = a.seqlen
    if a.heads:
        WORKLOAD["H"] = a.heads
    if a.batch or a.seqlen or a.heads:
        WORKLOAD["name"] = f"long_B{WORKLOAD['B']}_T{WORKLOAD['T']}_H{WORKLOAD['H']}_g2"
    return a


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(B, T, H, N, init_bytes=0):
    return B * T * H * BYTES_PER_TOKEN_HEAD + N * H * (STATE_BYTES + init_bytes) + H * (4 + 512)


def device_inputs(seed, device):
    """Seeded synthetic inputs drawn on the device (same distributions as the recipe)."""
    w = WORKLOAD
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, T, H, K, V = w["B"], w["T"], w["H"], w["K"], w["V"]

    def normal(shape, std=1.0):
        x = torch.empty(shape, dtype=torch.float32, device=device)
        x.normal_(0.0, std, generator=gen)
        return x.to(torch.bfloat16)

    q = normal((B, T, H, K))
    k = normal((B, T, H, K))
    v = normal((B, T, H, V))
    g = normal((B, T, H, K), w["g_std"])
    beta = normal((B, T, H))
    A_log = torch.empty(H, device=device).uniform_(1.0, 16.0, generator=gen).log_()
    dt_bias = torch.empty((H, K), device=device).normal_(0.0, 0.1, generator=gen)
    return dict(q=q, k=k, v=v, g=g, beta=beta, A_log=A_log, dt_bias=dt_bias,
                scale=1.0 / math.sqrt(K), lower_bound=-5.0)


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms",
                 "100", "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 8:
                continue
            try:
                rows.append(dict(sm=float(p[1]), max=float(p[2]), power=float(p[3]),
                                 reasons=[n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown",
                                                              "sw_thermal_slowdown", "sw_power_cap"),
                                                             p[4:8]) if v.lower() == "active"]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [r for r in rows if r["power"] > 200.0] or rows
        reasons = sorted({x for r in busy for x in r["reasons"]})
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": reasons,
                "samples": len(busy)}


def profile_traffic(kernel_source, profile=PROFILE, key="traffic_bytes_per_launch"):
    """DRAM bytes (``key``: per launch, or per unit) from a committed ncu summary, if the
    kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", profile)
    try:
        txt = open(path).read()
    except OSError:
        return None, None
    m = re.search(key + r":\s*([0-9.eE+]+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]+)", txt)
    if not m or not h or h.group(1) != source_hash(kernel_source):
        return None, None
    return float(m.group(1)), path


def source_hash(paths):
    hs = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            hs.update(f.read())
    return hs.hexdigest()[:16]


def cpu_baseline(min_seconds=10.0, max_passes=8):
    """The fp64 oracle on a bounded sample of the workload: one sequence of the full
    T tokens for every head (one (sequence, head) pair per host core at a time),
    repeated until at least ``min_seconds`` of CPU work have been timed."""
    import kda_inputs as ki
    import oracle
    cores = oracle.threads()
    H = WORKLOAD["H"]
    w = ki.Workload("sample", B=1, T=WORKLOAD["T"], H=H, g_std=WORKLOAD["g_std"])
    inp = ki.make_inputs(w, 3)
    passes, dt = 0, 0.0
    while passes < max_passes and (passes == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        oracle.forward_inputs(inp, want_final=True)
        dt += time.perf_counter() - t0
        passes += 1
    tokens = WORKLOAD["T"] * passes
    return {"value": tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{passes} pass(es) over 1 sequence x {WORKLOAD['T']} tokens x {H} heads "
                      f"(out and final state), {dt:.1f} s"}


def cpu_config_baseline(config_id, min_seconds=10.0):
    """The fp64 oracle on a bounded sample of parity workload ``config_id``: all heads of
    the first m sequences, m doubling until one pass takes at least a second, then
    repeated until ``min_seconds`` of CPU work.  tokens/s counts a token once for its H
    heads (the sampled token-heads divided by H)."""
    import kda_inputs as ki
    import numpy as np
    import oracle
    inp = ki.make_inputs(config_id)
    seqs, H = inp.seq_bounds(), inp.H
    m = 1
    while True:
        mask = np.zeros(len(seqs) * H, np.uint8)
        mask[: m * H] = 1
        t0 = time.perf_counter()
        oracle.forward_inputs(inp, want_final=True, mask=mask)
        dt = time.perf_counter() - t0
        if dt >= 1.0 or m >= len(seqs):
            break
        m = min(len(seqs), 2 * m)
    passes = 1
    while dt < min_seconds and passes < 64:
        t0 = time.perf_counter()
        oracle.forward_inputs(inp, want_final=True, mask=mask)
        dt += time.perf_counter() - t0
        passes += 1
    tokens = sum(n for _, _, n in seqs[:m]) * passes
    return {"value": tokens / dt, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{passes} pass(es) over {m} of {len(seqs)} sequence(s) x {H} heads of "
                      f"workload {ki.WORKLOADS[config_id].name} (out and final state), {dt:.1f} s"}


def dist_setup(n):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    if args.config_id is not None:
        import kda_inputs as ki
        base = cpu_config_baseline(args.config_id)
        name = ki.WORKLOADS[args.config_id].name
        print(json.dumps({
            "impl": "reference", "metric": f"KDA fwd prefill tokens/s, workload {name}",
            "value": base["value"], "unit": UNIT, "n_gpus": args.gpus, "steps": 1, "warmup": 0,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": name, "parallelism": "cpu"},
            "cpu_baseline": base,
            "e2e": {"value": base["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0
    times = []
    base = None
    for _ in range(max(1, min(args.steps, 3))):
        base = cpu_baseline()
        times.append(base["value"])
    value = statistics.median(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": len(times), "warmup": 0,
            "ms_per_step": WORKLOAD["B"] * WORKLOAD["T"] / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD["name"], "global_batch": WORKLOAD["B"],
                       "seq_len": WORKLOAD["T"], "heads": WORKLOAD["H"], "parallelism": "cpu"},
            "cpu_baseline": {**base, "value": value},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


DECODE_BYTES_PER_TOKEN_HEAD = 2 * 128 * 128 * 4 + 4 * 128 * 2 + 2 + 128 * 2  # state r+w, q k v g, beta, out
DECODE_SRC = ["linear_attention_09_b200/csrc/kda_decode.cu"]
DECODE_PROFILE = "decode_kernel_N128_H32.md"  # ncu DRAM bytes per token-head + source hash


def run_decode_bench(args, world, rank, local):
    """Decode step: N sequences x H heads, one token each, fp32 state updated in place."""
    import linear_attention_09_b200 as kda
    from linear_attention_09_b200 import build as kbuild
    kbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    N, H = args.decode_seqs, WORKLOAD["H"]
    gen = torch.Generator(device=device)
    gen.manual_seed(args.seed + 1000 * rank)
    rnd = lambda *shape, std=1.0: (torch.randn(*shape, device=device, generator=gen) * std)
    q, k, v = (rnd(N, H, 128).to(torch.bfloat16) for _ in range(3))
    g = rnd(N, H, 128, std=WORKLOAD["g_std"]).to(torch.bfloat16)
    beta = rnd(N, H).to(torch.bfloat16)
    A_log = torch.empty(H, device=device).uniform_(1.0, 16.0, generator=gen).log_()
    dt_bias = rnd(H, 128, std=0.1)
    state = rnd(N, H, 128, 128, std=0.05)
    out = torch.empty((N, H, 128), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        kda.kda_decode(q, k, v, g, beta, 1.0 / math.sqrt(128), A_log, dt_bias, -5.0, state,
                       out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    peak, peak_src = peaks()
    bytes_launch = N * H * DECODE_BYTES_PER_TOKEN_HEAD
    achieved = bytes_launch / (ms_local / args.steps / 1e3) / 1e9
    per_unit, _ = profile_traffic(DECODE_SRC, DECODE_PROFILE, "traffic_bytes_per_token_head")
    traffic = None if per_unit is None else per_unit * N * H
    if rank == 0:
        print(json.dumps({
            "metric": "KDA decode step token-heads/s (H=32, K=V=128, fp32 state in HBM)",
            "value": N * H * world * args.steps / (ms / 1e3), "unit": "token-heads/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16-io/fp32", "data": "synthetic",
            "config": {"workload": f"decode_N{N}_H{H}", "sequences": N * world, "heads": H,
                       "l2": f"state {N * H * 64 // 1024} MB per rank > 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                         "alg_bytes_per_launch": bytes_launch, "kernel": "decode_kernel"},
            "clocks": clk.summary(), "gpu_launches": args.steps}), flush=True)
    return 0


# Backward pass: compulsory bytes per token-head (q, k, v, g, dO, beta read as bf16;
# dq, dk, dv, dg, dbeta written as fp32) and the minimal arithmetic of reverse mode
# through the token recurrence: one forward step (alpha S, S^T k, rank-1 update: 5 K V
# FLOP) and the reverse step (12 K V FLOP), FMA = 2 FLOP.
BWD_BYTES_PER_TOKEN_HEAD = 5 * 256 + 2 + 4 * 512 + 4
BWD_FLOPS_PER_TOKEN_HEAD = 17 * 128 * 128
# fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward_bench(args, world, rank, local):
    """Backward pass on the headline prefill shape: kda_bwd with dL/dout given and
    dL/dS_0 returned (no dL/dS_final), device-resident inputs, CUDA-event timing."""
    import linear_attention_09_b200 as kda
    from linear_attention_09_b200 import build as kbuild
    kbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = WORKLOAD
    B, T, H = w["B"], w["T"], w["H"]  # --batch / --seqlen already applied by parse()
    inp = device_inputs(args.seed + 1000 * rank, device)
    gen = torch.Generator(device=device)
    gen.manual_seed(args.seed + 7 + 1000 * rank)
    dO = torch.empty((B, T, H, w["V"]), device=device).normal_(0.0, 1.0, generator=gen)
    dO = dO.to(torch.bfloat16)
    ws = torch.empty(kda.kda_bwd_workspace_size(B, T, H), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    kda.kda_set_bwd_schedule(args.bwd_schedule)

    def step():
        kda.kda_bwd(**inp, d_out=dO, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    launches = kda.kda_last_launch_count()
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    th = B * T * H
    flops = th * BWD_FLOPS_PER_TOKEN_HEAD
    achieved = flops / (ms_local / args.steps / 1e3) / 1e12
    bytes_launch = th * BWD_BYTES_PER_TOKEN_HEAD + B * H * STATE_BYTES
    if rank == 0:
        print(json.dumps({
            "metric": "KDA bwd tokens/s (H=32, K=V=128, T=32K)", "value":
            B * T * world * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16-in/fp32", "data": "synthetic",
            "config": {"workload": f"bwd_B{B}_T{T}_H{H}_g2", "global_batch": B * world,
                       "seq_len": T, "heads": H, "schedule": args.bwd_schedule,
                       "l2": f"inputs + gradients {bytes_launch / 1e9:.1f} GB per rank > 126 MB L2"},
            "roofline": {"bound": "alu", "achieved": achieved, "peak": FP32_PEAK_TFLOPS,
                         "unit": "TFLOP/s", "frac": achieved / FP32_PEAK_TFLOPS, "traffic": None,
                         "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz",
                         "alg_flops_per_launch": flops, "alg_bytes_per_launch": bytes_launch,
                         "hbm_gbs_algorithmic": bytes_launch / (ms_local / args.steps / 1e3) / 1e9,
                         "kernel": "bwdc_kernel" if args.bwd_schedule == "chunked" else "bwd_kernel"},
            "clocks": clk.summary(), "gpu_launches": launches * args.steps}), flush=True)
    return 0


def run_config_bench(args, world, rank, local):
    """Throughput of kda_fwd on one of the five parity workloads (same seeded inputs as
    the tests), device-resident inputs, CUDA-event timing."""
    import kda_inputs as ki
    import linear_attention_09_b200 as kda
    from linear_attention_09_b200 import build as kbuild
    kbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = ki.WORKLOADS[args.config_id]
    kda.kda_set_schedule(args.schedule)
    inp = ki.make_inputs(args.config_id)
    d = lambda t: None if t is None else t.to(device)
    call = dict(q=d(inp.q), k=d(inp.k), v=d(inp.v), g=d(inp.g), beta=d(inp.beta), scale=inp.scale,
                A_log=d(inp.A_log), dt_bias=d(inp.dt_bias), lower_bound=inp.lower_bound,
                initial_state=d(inp.initial_state), cu_seqlens=d(inp.cu_seqlens))
    out = torch.empty_like(call["v"])
    N, H = inp.num_seqs, inp.H
    fin = torch.empty((N, H, 128, 128), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    step = lambda: kda.kda_fwd(**call, out=out, final_state=fin, stream=stream)
    for _ in range(args.warmup):
        step()
    launches = kda.kda_last_launch_count()
    kernel = "chunk_kernel_split" if kda.kda_last_schedule() == "split" else KERNEL
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    tokens = inp.tokens
    init_bytes = 0 if inp.initial_state is None else inp.initial_state.element_size() * 128 * 128
    bytes_launch = tokens * H * BYTES_PER_TOKEN_HEAD + N * H * (STATE_BYTES + init_bytes) + H * 516
    peak, peak_src = peaks()
    achieved = bytes_launch / (ms / args.steps / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": f"KDA fwd prefill tokens/s, workload {wl.name}", "value": tokens * world * args.steps / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
            "config": {"workload": wl.name, "tokens": tokens, "sequences": N, "heads": H,
                       "schedule": args.schedule},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "peak_source": peak_src,
                         "alg_bytes_per_launch": bytes_launch, "kernel": kernel},
            "clocks": clk.summary(), "gpu_launches": launches * args.steps}), flush=True)
    return 0


def strong_scaling(args, world, rank, device):
    """One fixed global batch (the headline shape) split across the ranks by heads
    (``partition.plan_heads``): each rank runs kda_fwd on its heads, then the outputs are
    all-gathered (NCCL) so that every rank holds the global out.  Device time, max over
    ranks, both without and with the gather (tensor-parallel attention keeps the output
    head-sharded, so the first is the operator's own cost)."""
    import torch.distributed as dist
    import linear_attention_09_b200 as kda
    from linear_attention_09_b200 import partition
    w = WORKLOAD
    B, T, H = w["B"], w["T"], w["H"]
    plan = partition.plan_heads(H, world)[rank]
    Hr = plan.heads[1] - plan.heads[0]
    saved = WORKLOAD["H"]
    WORKLOAD["H"] = Hr
    try:
        inp = device_inputs(args.seed + 7 * rank, device)  # this rank's heads of the batch
    finally:
        WORKLOAD["H"] = saved
    out = torch.empty((B, T, Hr, w["V"]), dtype=torch.bfloat16, device=device)
    fin = torch.empty((B, Hr, w["K"], w["V"]), dtype=torch.float32, device=device)
    Hmax = max(p.heads[1] - p.heads[0] for p in partition.plan_heads(H, world))
    send = torch.zeros((Hmax, B, T, w["V"]), dtype=torch.bfloat16, device=device)
    recv = [torch.empty_like(send) for _ in range(world)]
    stream = torch.cuda.current_stream(device)

    def step(gather):
        kda.kda_fwd(**inp, out=out, final_state=fin, stream=stream)
        if gather:
            send[:Hr].copy_(out.permute(2, 0, 1, 3))
            dist.all_gather(recv, send)

    res = {}
    for gather in (False, True):
        for _ in range(args.warmup):
            step(gather)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step(gather)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
        res["with_gather" if gather else "kernel"] = {"ms_per_step": ms,
                                                       "value": B * T / (ms / 1e3)}
    return {"scaling": "strong", "plan": "heads", "global_batch": B, "seq_len": T, "heads": H,
            "unit": UNIT, "value": res["kernel"]["value"], "ms_per_step": res["kernel"]["ms_per_step"],
            "with_all_gather": res["with_gather"]}


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    if args.config_id is not None and args.impl == "ours":
        rc = run_config_bench(args, world, rank, local)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc
    if args.op in ("decode", "backward") and args.impl == "ours":
        rc = (run_decode_bench if args.op == "decode" else run_backward_bench)(args, world, rank,
                                                                                local)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import linear_attention_09_b200 as kda
    from linear_attention_09_b200 import build as kbuild
    kbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    kda.kda_set_schedule(args.schedule)
    w = WORKLOAD
    inp = device_inputs(args.seed + 1000 * rank, device)
    B, T, H = w["B"], w["T"], w["H"]
    out = torch.empty((B, T, H, w["V"]), dtype=torch.bfloat16, device=device)
    fin = torch.empty((B, H, w["K"], w["V"]), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        kda.kda_fwd(**inp, out=out, final_state=fin, stream=stream)

    for _ in range(args.warmup):
        step()
    launches_per_step = kda.kda_last_launch_count()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    tokens = B * T
    value = tokens * world * args.steps / (ms / 1e3)
    ms_step = ms / args.steps

    # roofline of the dominant (only) kernel: algorithmic bytes / average launch time
    peak, peak_src = peaks()
    bytes_launch = algorithmic_bytes(B, T, H, B)
    achieved = bytes_launch / (ms_local / args.steps / launches_per_step / 1e3) / 1e9
    traffic, _ = profile_traffic(KERNEL_SRC)

    # end to end: host (pinned) buffers through kda_fwd_host, copies inside the timed region
    host = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "g", "beta")}
    host_alog, host_dt = inp["A_log"].cpu(), inp["dt_bias"].cpu()
    out_h = torch.empty((B, T, H, w["V"]), dtype=torch.bfloat16).pin_memory()
    fin_h = torch.empty((B, H, w["K"], w["V"]), dtype=torch.float32).pin_memory()
    ws = torch.empty(kda.kda_fwd_host_workspace_size(B, T, H, 128, 128, 0, 0, True),
                     dtype=torch.uint8, device=device)

    def e2e_step():
        kda.kda_fwd_host(**host, scale=inp["scale"], A_log=host_alog, dt_bias=host_dt,
                         lower_bound=inp["lower_bound"], out=out_h, final_state=fin_h,
                         workspace=ws, stream=stream)

    e2e_value = None
    if args.e2e_steps > 0:
        e2e_step()
        barrier(world)
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            e2e_step()
        e2e_s = max_over_ranks(time.perf_counter() - t0, world)
        e2e_value = tokens * world * args.e2e_steps / e2e_s
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + host_alog.numel() * 4 + \
        host_dt.numel() * 4
    d2h = out_h.numel() * 2 + fin_h.numel() * 4
    del ws

    strong = strong_scaling(args, world, rank, device) if world > 1 else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
            "config": {"workload": w["name"], "global_batch": B * world, "seq_len": T, "heads": H,
                       "head_dim": 128, "parallelism": f"dp{world}",
                       "l2": "inputs 5.4 GB per step > 126 MB L2 (no flush needed)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": peak_src,
                         "alg_bytes_per_launch": bytes_launch,
                         "kernel": KERNEL},
            "tflops": FLOPS_PER_TOKEN_HEAD * tokens * H * world * args.steps / (ms / 1e3) / 1e12,
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "cpu_baseline": cpu,
        }
        if strong is not None:
            line["strong"] = strong
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
