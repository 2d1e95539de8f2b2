"""Context-parallel prefill (the batch's sequences split along T).

CPU tests run the algorithm with the fp64 token-by-token oracle as the forward pass,
in one process and as two gloo ranks, and require agreement with the unsplit oracle
to ~1e-10: that checks the segment maps (Z from a zero start, M from v = 0 and an
identity start), the exchange and the exclusive scan.  The GPU test runs the same
split with the CUDA kernel and holds it to the parity bars.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import kda_inputs as ki
import oracle
from linear_attention_09_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def oracle_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lb, init):
    """The oracle with the signature of the kernel call (CPU tensors in and out)."""
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    if init is None:
        idt, arr = oracle.STATE_NONE, None
    elif init.dtype == torch.float64:
        idt, arr = oracle.STATE_F64, init.numpy()
    else:
        idt, arr = oracle.STATE_F32, init.float().numpy()
    out, fin = oracle.forward(bits(q), bits(k), bits(v), bits(g), bits(beta), scale,
                              A_log.numpy(), dt_bias.numpy(), lb, arr, idt)
    return torch.from_numpy(out), torch.from_numpy(fin)


def inputs(T=96, B=2, H=2, init="f32", seed=0, g_std=1.0):
    return ki.make_inputs(ki.Workload("cp", B=B, T=T, H=H, init_state=init, g_std=g_std), seed)


def args_of(inp):
    return (inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale, inp.A_log, inp.dt_bias,
            inp.lower_bound)


def rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(np.asarray(b)))


@pytest.mark.parametrize("segments", [2, 3, 4])
@pytest.mark.parametrize("init", [None, "f32"])
def test_split_equals_unsplit_oracle(segments, init):
    inp = inputs(init=init, seed=segments)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_s, fin_s = cp.kda_fwd_segments(*args_of(inp), initial_state=inp.initial_state,
                                       segments=segments, fwd=oracle_fwd)
    assert rel(out_s, out_r) < 1e-10
    assert rel(fin_s, fin_r) < 1e-10


def test_segment_maps_are_affine():
    """S_end = M S_start + Z for an arbitrary start, with M and Z from the two runs."""
    inp = inputs(T=40, B=1, H=2, init="f32", seed=7, g_std=2.0)
    M, Z = cp.segment_maps(*args_of(inp), fwd=oracle_fwd)
    _, fin = oracle.forward_inputs(inp)
    S0 = inp.initial_state.double()
    assert rel(torch.matmul(M, S0) + Z, fin) < 1e-10


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    inp = inputs(T=64, seed=11)
    Tr = 64 // world
    cut = lambda t: t[:, rank * Tr:(rank + 1) * Tr].contiguous()
    out, fin = cp.kda_fwd_context_parallel(
        cut(inp.q), cut(inp.k), cut(inp.v), cut(inp.g), cut(inp.beta), inp.scale, inp.A_log,
        inp.dt_bias, inp.lower_bound, initial_state=inp.initial_state, fwd=oracle_fwd)
    np.save(os.path.join(outdir, f"out{rank}.npy"), out.numpy())
    np.save(os.path.join(outdir, f"fin{rank}.npy"), fin.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_context_parallel_two_gloo_ranks(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    inp = inputs(T=64, seed=11)
    out_r, fin_r = oracle.forward_inputs(inp)
    out = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(2)], axis=1)
    assert rel(out, out_r) < 1e-10
    assert rel(np.load(tmp_path / "fin1.npy"), fin_r) < 1e-10  # the last rank holds the final state


@pytest.mark.gpu
@pytest.mark.parametrize("segments", [2, 4])
def test_split_on_the_gpu_meets_the_bars(segments):
    """The kernel run as the split (three passes per segment, fp64 scan) against the
    oracle over the whole sequences, under the parity bars."""
    inp = inputs(T=512, B=2, H=3, init="f32", seed=5)
    d = lambda t: t.to("cuda")
    out, fin = cp.kda_fwd_segments(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale,
                                   d(inp.A_log), d(inp.dt_bias), inp.lower_bound,
                                   initial_state=d(inp.initial_state), segments=segments)
    torch.cuda.synchronize()
    out_r, fin_r = oracle.forward_inputs(inp)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(o - out_r).max() <= 3e-2 and rel(o, out_r) <= 5e-3
    assert rel(fin.cpu().numpy().astype(np.float64), fin_r) <= 1e-3
