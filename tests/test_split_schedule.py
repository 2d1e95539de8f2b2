"""The split schedule (a 4-CTA cluster per (sequence, head): three CTAs prepare every
third chunk, one runs the state pass) against the fused one (one CTA per unit).

Both run the same arithmetic in the same order, and the data that crosses between the
CTAs is copied bit for bit, so out and the final state must be identical; the split
results are also held to the oracle's bars.  Cases of long units also compare the fused
kernel variant whose state warps compute the round-1 gates against the split kernel
(which does not).  Forced splits cover units with fewer
chunks than producing CTAs (some CTAs get none) and empty varlen sequences.
"""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_09_b200 as kda
import oracle

OUT_MAXABS, OUT_REL, FIN_REL = 3e-2, 5e-3, 1e-3


def test_schedule_switch_rejects_unknown_modes():
    prev = kda.kda_set_schedule("auto")
    try:
        with pytest.raises(kda.KDAError):
            kda.kda_set_schedule(7)
        assert kda.kda_set_schedule("fused") == "auto"
        assert kda.kda_set_schedule("split") == "fused"
    finally:
        kda.kda_set_schedule(prev)


def _run(inp, schedule):
    d = lambda t: None if t is None else t.to("cuda")
    prev = kda.kda_set_schedule(schedule)
    try:
        o, f = kda.kda_fwd(q=d(inp.q), k=d(inp.k), v=d(inp.v), g=d(inp.g), beta=d(inp.beta),
                           scale=inp.scale, A_log=d(inp.A_log), dt_bias=d(inp.dt_bias),
                           lower_bound=inp.lower_bound, initial_state=d(inp.initial_state),
                           cu_seqlens=d(inp.cu_seqlens))
        torch.cuda.synchronize()
    finally:
        kda.kda_set_schedule(prev)
    assert kda.kda_device_status(reset=True) == 0, "a bounded wait in the kernel gave up"
    return o.cpu(), f.cpu()


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


CASES = [
    dict(B=1, T=512, H=4, init=None, lengths=None),        # the tiny workload's shape
    dict(B=2, T=700, H=5, init="f32", lengths=None),       # partial last chunk
    dict(B=1, T=64, H=3, init="f32", lengths=None),        # one chunk: two CTAs idle
    dict(B=1, T=130, H=2, init="bf16", lengths=None),      # three chunks, the last partial
    dict(B=1, T=1, H=2, init="f32", lengths=None),
    dict(B=1, T=0, H=2, init="f32", lengths=[300, 0, 65, 1000, 129]),
    # units of >= 1024 tokens on average: the fused schedule runs the kernel whose state
    # warps compute the round-1 gates from chunk 2 on
    dict(B=1, T=1300, H=3, init="f32", lengths=None),
    dict(B=1, T=0, H=2, init="bf16", lengths=[1300, 2, 2000]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}T{c['T']}H{c['H']}{'v' if c['lengths'] else ''}")
def test_split_equals_fused_and_meets_the_bars(case):
    w = ki.Workload("split", B=case["B"], T=max(case["T"], 1), H=case["H"], init_state=case["init"])
    inp = ki.make_inputs(w, 11, lengths=case["lengths"]) if case["lengths"] else ki.make_inputs(w, 11, T=case["T"])
    of, ff = _run(inp, "fused")
    osp, fsp = _run(inp, "split")
    assert torch.equal(of.view(torch.int16), osp.view(torch.int16)), "out differs between schedules"
    assert torch.equal(ff, fsp), "final state differs between schedules"
    out_r, fin_r = oracle.forward_inputs(inp)
    og = osp.float().numpy().astype(np.float64)
    rows = [og[b, t0:t0 + n, :].ravel() for (b, t0, n) in inp.seq_bounds()]
    refs = [out_r[b, t0:t0 + n, :].ravel() for (b, t0, n) in inp.seq_bounds()]
    og, orf = np.concatenate(rows), np.concatenate(refs)
    if og.size:
        assert np.abs(og - orf).max() <= OUT_MAXABS
        assert _rel(og, orf) <= OUT_REL
    assert _rel(fsp.numpy().astype(np.float64), fin_r) <= FIN_REL


@pytest.mark.gpu
@pytest.mark.parametrize("layout,final_dtype", [("vk", torch.float32), ("kv", torch.bfloat16)])
def test_split_state_variants_equal_fused(layout, final_dtype):
    """The state I/O variants (S[v][k] layout, bf16 final state) go through the same
    state pass on CTA 0 of the split kernel: identical bits to the fused schedule."""
    w = ki.Workload("split_ex", B=2, T=300, H=3, init_state="f32")
    inp = ki.make_inputs(w, 13)
    d = lambda t: t.to("cuda")
    init = d(inp.initial_state)
    if layout == "vk":
        init = init.transpose(-1, -2).contiguous()
    res = []
    for sch in ("fused", "split"):
        prev = kda.kda_set_schedule(sch)
        try:
            o, f = kda.kda_fwd_ex(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale,
                                  d(inp.A_log), d(inp.dt_bias), inp.lower_bound, initial_state=init,
                                  state_layout=layout, final_state_dtype=final_dtype)
            torch.cuda.synchronize()
            assert kda.kda_last_schedule() == sch
        finally:
            kda.kda_set_schedule(prev)
        assert kda.kda_device_status(reset=True) == 0
        res.append((o.cpu(), f.cpu()))
    assert torch.equal(res[0][0].view(torch.int16), res[1][0].view(torch.int16))
    assert torch.equal(res[0][1], res[1][1])
