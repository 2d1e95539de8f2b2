"""Context-parallel prefill: the sequences of a batch split along T across ranks.

The recurrence is affine in the state: over a segment of tokens, the state at its
end is S_end = M S_start + Z, where M (K x K) is the product of the segment's
transitions (I - b k^ k^T) Diag(alpha) and Z is the state the segment reaches from
S_start = 0 (operator: FlashKDA pages, 7minutos.es "¿Qué es la atención Kimi
Delta...?"; the long-context motivation in the same article).  Both come out of the
forward kernel itself: Z is the final state of the segment started from zero, and M
is the final state of the segment run with v = 0 from S_start = I (K = V = 128, so
the identity is a valid state).

Rank r holds tokens [r T_r, (r+1) T_r) of every sequence.  It computes (M_r, Z_r),
the ranks exchange them with one all-gather, every rank forms its true start state
by the exclusive scan S_0 = initial state, S_{j+1} = M_j S_j + Z_j (in fp64), and
reruns its segment from that state, which gives its exact outputs and, on the last
rank, the final state.  Each rank runs three forward passes over its segment, so
the split pays off from about four ranks.

Every forward pass is a ``kda_fwd_ex`` call (the CUDA kernel); the scan is K x K by
K x V products per (sequence, head), done with torch in fp64.  ``fwd`` can be
replaced (the CPU tests pass a token-by-token reference there).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch


def _default_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state):
    from . import kda_fwd_ex
    return kda_fwd_ex(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound,
                      initial_state=initial_state)


def segment_maps(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound,
                 fwd: Callable = _default_fwd):
    """(M, Z) of one segment, each [B, H, 128, 128] fp32: S_end = M S_start + Z."""
    B, _, H, K = q.shape
    _, Z = fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, None)
    eye = torch.eye(K, dtype=torch.float32, device=q.device).expand(B, H, K, K).contiguous()
    _, M = fwd(q, k, torch.zeros_like(v), g, beta, scale, A_log, dt_bias, lower_bound, eye)
    return M, Z


def scan_starts(Ms: Sequence[torch.Tensor], Zs: Sequence[torch.Tensor],
                initial_state: Optional[torch.Tensor]) -> list:
    """Start states of the segments: S_0 = initial state (or 0), S_{j+1} = M_j S_j + Z_j.

    Returns tensors of the dtype of the Z_j (fp32 from the kernel); the products run
    in fp64."""
    S = (torch.zeros_like(Zs[0], dtype=torch.float64) if initial_state is None
         else initial_state.to(torch.float64))
    starts = []
    for M, Z in zip(Ms, Zs):
        starts.append(S.to(Zs[0].dtype))
        S = torch.matmul(M.to(torch.float64), S) + Z.to(torch.float64)
    return starts


def kda_fwd_context_parallel(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound,
                             initial_state=None, group=None, fwd: Callable = _default_fwd):
    """This rank's segment of a context-parallel prefill.

    q, k, g: [B, T_r, H, 128], v: [B, T_r, H, 128], beta: [B, T_r, H] -- the tokens
    [r T_r, (r+1) T_r) of every sequence, r = this rank in ``group``.  initial_state
    ([B, H, 128, 128] or None) is the state before token 0, the same on every rank.
    Returns (out for the segment, state at the end of the segment); on the last rank
    the latter is the final state of the sequences.  One all-gather of 2 B H 64 KB
    per rank crosses the ranks.
    """
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    M, Z = segment_maps(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, fwd)
    both = torch.stack([M, Z]).contiguous()
    gathered = [torch.empty_like(both) for _ in range(world)]
    dist.all_gather(gathered, both, group=group)
    starts = scan_starts([t[0] for t in gathered], [t[1] for t in gathered], initial_state)
    return fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, starts[rank])


def kda_fwd_segments(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
                     segments: int = 2, fwd: Callable = _default_fwd):
    """The context-parallel algorithm run in one process over ``segments`` equal
    pieces of T (T divisible by ``segments``); returns (out, final state) of the whole
    sequences, for checking the split against an unsplit call."""
    B, T, H, K = q.shape
    assert T % segments == 0
    Tr = T // segments
    cut = lambda t, j: t[:, j * Tr:(j + 1) * Tr].contiguous()
    maps = [segment_maps(cut(q, j), cut(k, j), cut(v, j), cut(g, j), cut(beta, j), scale, A_log,
                         dt_bias, lower_bound, fwd) for j in range(segments)]
    starts = scan_starts([m for m, _ in maps], [z for _, z in maps], initial_state)
    outs, fin = [], None
    for j in range(segments):
        o, fin = fwd(cut(q, j), cut(k, j), cut(v, j), cut(g, j), cut(beta, j), scale, A_log,
                     dt_bias, lower_bound, starts[j])
        outs.append(o)
    return torch.cat(outs, dim=1), fin
