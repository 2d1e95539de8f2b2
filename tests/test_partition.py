"""Data-parallel split of one global batch across ranks (CPU; the oracle stands in for
the kernel as the forward pass, so the gathered result must equal the one-rank call
exactly: every (sequence, head) unit is computed by the same arithmetic either way)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import kda_inputs as ki
import oracle
from linear_attention_09_b200 import partition as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def oracle_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
               cu_seqlens=None, **_):
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    init, idt = None, oracle.STATE_NONE
    if initial_state is not None:
        init, idt = initial_state.numpy(), oracle.STATE_F32
    out, fin = oracle.forward(bits(q), bits(k), bits(v), bits(g), bits(beta), scale,
                              A_log.numpy(), dt_bias.numpy(), lower_bound, init, idt,
                              None if cu_seqlens is None else cu_seqlens.numpy())
    return torch.from_numpy(out), torch.from_numpy(fin)


def global_inputs(kind):
    if kind == "heads":
        w = ki.Workload("p", B=2, T=150, H=5, init_state="f32", g_std=2.0)
        inp = ki.make_inputs(w, 1)
    else:
        w = ki.Workload("p", B=1, T=0, H=3, init_state="f32")
        inp = ki.make_inputs(w, 2, lengths=[300, 5, 0, 129, 64, 77, 1])
    return inp, dict(q=inp.q, k=inp.k, v=inp.v, g=inp.g, beta=inp.beta, scale=inp.scale,
                     A_log=inp.A_log, dt_bias=inp.dt_bias, lower_bound=inp.lower_bound,
                     initial_state=inp.initial_state, cu_seqlens=inp.cu_seqlens)


def test_head_plan_covers_every_head_once():
    for H, world in [(32, 8), (5, 2), (3, 4), (1, 1)]:
        plans = P.plan_heads(H, world)
        sizes = [p.heads[1] - p.heads[0] for p in plans]
        assert sum(sizes) == H and max(sizes) - min(sizes) <= 1
        assert all(plans[r].heads[1] == plans[r + 1].heads[0] for r in range(world - 1))


def test_sequence_plan_is_lpt_balanced():
    rng = np.random.default_rng(0)
    lengths = rng.integers(64, 513, size=1024).tolist()
    plans = P.plan_sequences(lengths, H=16, world=8)
    got = sorted(s for p in plans for s in p.seqs)
    assert got == list(range(len(lengths)))
    loads = [sum(lengths[s] + P.PER_SEQUENCE_TOKENS for s in p.seqs) for p in plans]
    # LPT: no rank exceeds the mean by more than the largest single sequence
    assert max(loads) - sum(loads) / len(loads) <= max(lengths) + P.PER_SEQUENCE_TOKENS
    # longest first: the two longest sequences land on different ranks
    a, b = sorted(range(len(lengths)), key=lambda s: -lengths[s])[:2]
    assert [a in p.seqs for p in plans].index(True) != [b in p.seqs for p in plans].index(True)


@pytest.mark.parametrize("kind", ["heads", "sequences"])
def test_shards_of_one_rank_equal_slices_of_the_full_result(kind):
    inp, kw = global_inputs(kind)
    full_out, full_fin = oracle_fwd(**kw)
    plans = (P.plan_heads(inp.H, 2) if kind == "heads"
             else P.plan_sequences(inp.cu_seqlens.diff().tolist(), inp.H, 3))
    for p in plans:
        if p.seqs == []:
            continue
        out, fin = oracle_fwd(**P.shard(kw, p))
        h0, h1 = p.heads
        if kind == "heads":
            assert torch.equal(out, full_out[:, :, h0:h1]) and torch.equal(fin, full_fin[:, h0:h1])
        else:
            cu = inp.cu_seqlens
            rows = torch.cat([torch.arange(int(cu[s]), int(cu[s + 1])) for s in p.seqs])
            assert torch.equal(out[0], full_out[0, rows])
            assert torch.equal(fin, full_fin[p.seqs])


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, kind, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    inp, kw = global_inputs(kind)
    plans = (P.plan_heads(inp.H, world) if kind == "heads"
             else P.plan_sequences(inp.cu_seqlens.diff().tolist(), inp.H, world))
    out, fin = P.run_sharded(kw, plans, rank, fwd=oracle_fwd)
    torch.save({"out": out, "fin": fin}, os.path.join(outdir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["heads", "sequences"])
def test_two_gloo_ranks_gather_the_one_rank_result(tmp_path, kind):
    ctx = mp.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, kind, str(tmp_path)))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    inp, kw = global_inputs(kind)
    ref_out, ref_fin = oracle_fwd(**kw)
    rows = torch.ones(ref_out.shape[1], dtype=torch.bool)
    for r in range(2):
        d = torch.load(tmp_path / f"r{r}.pt")
        assert torch.equal(d["out"][:, rows], ref_out[:, rows].to(d["out"].dtype))
        assert torch.equal(d["fin"], ref_fin.to(d["fin"].dtype))
