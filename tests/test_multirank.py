"""Multi-rank host logic of bench.py on the CPU: world size 2 over gloo.

The data path has no collective (the (sequence, head) units are independent), so the
multi-rank part is the harness: process-group setup from the torchrun environment,
the barrier around the timed region, the max-over-ranks time, and the reference arm
where rank 0 alone runs and prints.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    assert (w, r) == (world, rank)
    bench.barrier(w)
    t = bench.max_over_ranks(1.5 * (rank + 1), w)  # ranks report 1.5 and 3.0
    with open(os.path.join(outdir, f"r{rank}.txt"), "w") as f:
        f.write(repr(t))
    bench.barrier(w)
    dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    ctx = mp.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        assert float((tmp_path / f"r{r}.txt").read_text()) == 3.0


def test_reference_arm_two_ranks_prints_once():
    """torchrun with 2 ranks: rank 0 times the oracle and prints one JSON line; rank 1
    exits 0 without work."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--seqlen", "256"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_on_a_parity_workload():
    """--impl reference --config-id N times the oracle on a bounded sample of workload N."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--config-id", "0"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    d = json.loads([l for l in res.stdout.splitlines() if l.startswith("{")][0])
    assert d["impl"] == "reference" and "tiny_B1_T512_H4" in d["metric"]
    assert d["value"] > 0 and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _strong_main(rank, world, port, outdir):
    """bench.strong_scaling over gloo on the CPU, with the kernel and the CUDA timing
    calls replaced by host stand-ins (the collective and the head plan are the real ones)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import time
    import types

    import torch
    import bench
    import linear_attention_09_b200 as kda
    import torch.distributed as dist

    class Ev:
        def __init__(self, **_):
            self.t = 0.0

        def record(self, *_):
            self.t = time.perf_counter()

        def elapsed_time(self, other):
            return (other.t - self.t) * 1e3

    calls = []

    def fake_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, out=None,
                 final_state=None, stream=None, **_):
        calls.append(q.shape)
        out.fill_(float(rank + 1))
        final_state.zero_()
        return out, final_state

    torch.cuda.Event = Ev
    torch.cuda.synchronize = lambda *a, **k: None
    torch.cuda.current_stream = lambda *a, **k: None
    kda.kda_fwd = fake_fwd
    w, r, _ = bench.dist_setup(world)
    bench.WORKLOAD.update(B=1, T=64, H=5)
    args = types.SimpleNamespace(seed=3, warmup=1, steps=2)
    res = bench.strong_scaling(args, w, r, torch.device("cpu"))
    with open(os.path.join(outdir, f"s{rank}.txt"), "w") as f:
        f.write(repr((res["heads"], res["global_batch"], res["value"] > 0,
                      res["with_all_gather"]["value"] > 0, sorted(set(tuple(c) for c in calls)))))
    dist.destroy_process_group()


def test_strong_scaling_line_two_gloo_ranks(tmp_path):
    ctx = mp.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=_strong_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = [eval((tmp_path / f"s{r}.txt").read_text()) for r in range(2)]
    # H = 5 over two ranks: heads 0..2 and 3..4; every step ran the forward on its heads
    assert got[0][0] == 5 and got[0][2] and got[0][3]
    assert got[0][4] == [(1, 64, 3, 128)] and got[1][4] == [(1, 64, 2, 128)]
