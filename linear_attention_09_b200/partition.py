"""Data-parallel split of one global KDA batch across ranks (one GPU per rank).

KDA has no term that couples two heads or two sequences (FlashKDA pages,
7minutos.es "¿Qué es la atención Kimi Delta...?": the state is per head, and each
sequence of a cu_seqlens batch starts from its own initial state), so the
(sequence, head) units of a batch can be split across GPUs with no exchange on the
data path.  Two plans:

- ``plan_heads``: contiguous head ranges, sizes within one of each other (the
  tensor-parallel split of attention heads).  Every rank processes every token.
- ``plan_sequences``: whole varlen sequences, assigned longest first to the rank
  with the least work so far (LPT).  The cost of a sequence is its token count plus
  a fixed per-sequence overhead expressed in tokens (set-up, pipeline fill and
  drain of its units).

``shard`` cuts a rank's part out of the global inputs (copies into contiguous
tensors, since the kernel wants contiguous rows); ``run_sharded`` runs the
forward pass on each rank's part and gathers the outputs with one all-gather, so
every rank ends with the same global ``out`` and final states as a single-rank
call.  The forward pass is a parameter (default: ``kda_fwd``, the CUDA kernel);
the CPU tests pass the oracle there.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence

import torch

PER_SEQUENCE_TOKENS = 96  # fixed cost of a sequence, in tokens of work, for LPT


@dataclasses.dataclass
class Plan:
    """A rank's part of the batch: ``heads`` (h0, h1) and ``seqs`` (sorted sequence
    indices; None means every sequence)."""
    mode: str                      # "heads" or "sequences"
    heads: tuple                   # (h0, h1)
    seqs: Optional[List[int]]


def plan_heads(H: int, world: int) -> List[Plan]:
    """Contiguous head ranges; rank r gets H // world heads, plus one for r < H % world."""
    base, extra = divmod(H, world)
    plans, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        plans.append(Plan("heads", (h, h + n), None))
        h += n
    return plans


def plan_sequences(lengths: Sequence[int], H: int, world: int,
                   per_seq: int = PER_SEQUENCE_TOKENS) -> List[Plan]:
    """Longest processing time first: sequences in decreasing length (ties by index)
    go to the rank with the least assigned cost (ties by rank)."""
    order = sorted(range(len(lengths)), key=lambda s: (-int(lengths[s]), s))
    load = [0] * world
    owned: List[List[int]] = [[] for _ in range(world)]
    for s in order:
        r = min(range(world), key=lambda i: (load[i], i))
        owned[r].append(s)
        load[r] += int(lengths[s]) + per_seq
    return [Plan("sequences", (0, H), sorted(o)) for o in owned]


def _rows(cu: torch.Tensor, seqs: List[int]) -> torch.Tensor:
    """Token rows of the listed sequences, in order."""
    parts = [torch.arange(int(cu[s]), int(cu[s + 1]), dtype=torch.long) for s in seqs]
    return torch.cat(parts) if parts else torch.zeros(0, dtype=torch.long)


def shard(inputs: dict, plan: Plan) -> dict:
    """The rank's inputs as contiguous tensors (same keys as ``kda_fwd``'s arguments:
    q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, plus the scalars)."""
    out = dict(inputs)
    h0, h1 = plan.heads
    for name in ("q", "k", "v", "g", "beta"):
        out[name] = inputs[name][:, :, h0:h1].contiguous()
    out["A_log"] = inputs["A_log"][h0:h1].contiguous()
    out["dt_bias"] = inputs["dt_bias"][h0:h1].contiguous()
    init = inputs.get("initial_state")
    if init is not None:
        out["initial_state"] = init[:, h0:h1].contiguous()
    if plan.seqs is not None:
        cu = inputs["cu_seqlens"].cpu()
        rows = _rows(cu, plan.seqs).to(inputs["q"].device)
        for name in ("q", "k", "v", "g", "beta"):
            out[name] = out[name].index_select(1, rows).contiguous()
        lens = [int(cu[s + 1] - cu[s]) for s in plan.seqs]
        local = torch.zeros(len(lens) + 1, dtype=torch.int64)
        local[1:] = torch.tensor(lens, dtype=torch.int64).cumsum(0)
        out["cu_seqlens"] = local.to(inputs["cu_seqlens"].device)
        if init is not None:
            idx = torch.tensor(plan.seqs, dtype=torch.long, device=init.device)
            out["initial_state"] = out["initial_state"].index_select(0, idx).contiguous()
    return out


def _default_fwd(**kw):
    from . import kda_fwd
    return kda_fwd(**kw)


def _all_gather_padded(t: torch.Tensor, group, world: int) -> List[torch.Tensor]:
    """all_gather of tensors whose first dimension differs by rank (padded to the max)."""
    import torch.distributed as dist
    n = torch.tensor([t.shape[0]], dtype=torch.int64, device=t.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n, group=group)
    m = int(max(int(x) for x in sizes))
    buf = torch.zeros((m,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    buf[: t.shape[0]] = t
    bufs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(bufs, buf, group=group)
    return [b[: int(s)] for b, s in zip(bufs, sizes)]


def run_sharded(inputs: dict, plans: List[Plan], rank: int, group=None,
                fwd: Callable = _default_fwd):
    """Forward pass over this rank's part, then one all-gather of every rank's out and
    final states; returns the global (out [B,T,H,V], final [N,H,K,V]) on every rank."""
    import torch.distributed as dist
    world = len(plans)
    plan = plans[rank]
    B, T, H = inputs["q"].shape[:3]
    V = inputs["v"].shape[3]
    if plan.mode == "sequences" and not plan.seqs:  # more ranks than sequences
        dev = inputs["q"].device
        out = torch.zeros((1, 0, H, V), dtype=torch.bfloat16, device=dev)
        fin = torch.zeros((0, H, inputs["q"].shape[3], V), dtype=torch.float32, device=dev)
    else:
        out, fin = fwd(**shard(inputs, plan))
    # heads: [H_r, B, T, V] and [H_r, N, K, V] (head-major, so the gather is along dim 0)
    # sequences: rows of the packed local batch [rows_r, H, V] and states [N_r, H, K, V]
    if plan.mode == "heads":
        o_parts = _all_gather_padded(out.permute(2, 0, 1, 3).contiguous(), group, world)
        f_parts = _all_gather_padded(fin.permute(1, 0, 2, 3).contiguous(), group, world)
        out_g = torch.cat(o_parts, 0).permute(1, 2, 0, 3).contiguous()
        fin_g = torch.cat(f_parts, 0).permute(1, 0, 2, 3).contiguous()
        return out_g, fin_g
    cu = inputs["cu_seqlens"].cpu()
    o_parts = _all_gather_padded(out[0].contiguous(), group, world)
    f_parts = _all_gather_padded(fin.contiguous(), group, world)
    out_g = torch.zeros((1, T, H, V), dtype=out.dtype, device=out.device)
    N = cu.numel() - 1
    fin_g = torch.zeros((N,) + tuple(fin.shape[1:]), dtype=fin.dtype, device=fin.device)
    for p, op, fp in zip(plans, o_parts, f_parts):
        rows = _rows(cu, p.seqs).to(out.device)
        out_g[0].index_copy_(0, rows, op)
        if p.seqs:
            fin_g.index_copy_(0, torch.tensor(p.seqs, dtype=torch.long, device=fin.device), fp)
    return out_g, fin_g
