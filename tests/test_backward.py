"""Parity of the CUDA backward pass (``kda_bwd``) against the fp64 oracle backward,
in both schedules: "chunked" (the forward kernel's chunk checkpoints, then the chunked
matrix form in reverse) and "token" (the token recurrence reversed step by step).

Every gradient the call returns is compared element by element with the oracle on
the same seeded bf16 inputs, random bf16 dL/dout and (optionally) fp32 dL/dS_final.
Bars: per gradient tensor rel-L2 <= 1e-3 and max-abs <= 1e-2 of the tensor's largest
entry.  The token schedule is fp32 throughout: sums of at most 128 terms per token and
a reverse recurrence whose factors alpha are <= 1, about 1e-6 relative.  The chunked
schedule is fp32 too, but its chunk states come from the forward kernel, whose fp16 and
tf32 products put about 3e-4 relative error on the state; the gradients are linear in
those states (and in the quantities derived from them), so they carry errors of that
order, still below the bars.

The gate clamp lam = max(lb, z) is a kink: where z = -exp(A_log) softplus(x) sits
within 5e-5 of lb (fp32 evaluates z to within ~3e-6), the kernel (fp32) and the oracle
(fp64) may take different sides, and both gradients are valid there.  At those
elements dg must be 0 or the open-side value -dlam exp(A_log) sigmoid(x) (dlam from
the oracle); ddt_bias and dA_log may differ from the oracle by at most the sum of
those elements' contributions, on top of the bars.
"""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import oracle

pytestmark = pytest.mark.gpu

REL, MAXREL = 1e-3, 1e-2
TIE = 5e-5


def kda():
    import linear_attention_09_b200 as m
    return m


def case(lengths=None, B=2, T=200, H=3, init=None, g_std=1.0, seed=0, dfinal=True):
    w = ki.Workload("bwd", B=B, T=T, H=H, init_state=init, g_std=g_std)
    inp = ki.make_inputs(w, seed, lengths=lengths)
    gen = torch.Generator().manual_seed(seed + 1000)
    Bv, Tv = inp.q.shape[:2]
    dO = torch.randn((Bv, Tv, H, 128), generator=gen).to(torch.bfloat16)
    N = Bv if inp.cu_seqlens is None else inp.cu_seqlens.numel() - 1
    dSf = torch.randn((N, H, 128, 128), generator=gen) * 0.1 if dfinal else None
    return inp, dO, dSf


def gate_terms(inp):
    """z - lb and the factor d(lam)/d(x) on the open side, fp64 [B,T,H,K]."""
    x = inp.g.double() + inp.dt_bias.double()[None, None]
    ea = torch.exp(inp.A_log.double())[None, None, :, None]
    z = -ea * torch.nn.functional.softplus(x, threshold=60.0)
    return (z - inp.lower_bound).numpy(), (-ea * torch.sigmoid(x)).numpy(), z.numpy()


SCHEDULES = ("chunked", "token")


def run_gpu(inp, dO, dSf, on_device=False, schedule="chunked"):
    d = lambda t: None if t is None else t.cuda()
    prev = kda().kda_set_bwd_schedule(schedule)
    try:
        r = _bwd(inp, dO, dSf, d)
    finally:
        kda().kda_set_bwd_schedule(prev)
    if on_device:
        return r
    return {k: v.cpu().double().numpy() for k, v in r.items() if v is not None}


def _bwd(inp, dO, dSf, d):
    r = kda().kda_bwd(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale,
                      d(inp.A_log), d(inp.dt_bias), inp.lower_bound, d(dO),
                      initial_state=d(inp.initial_state), d_final_state=d(dSf),
                      cu_seqlens=d(inp.cu_seqlens))
    torch.cuda.synchronize()
    return r


def rows_in_sequences(inp):
    """Mask of token rows [B, T] that belong to a sequence."""
    B, T = inp.q.shape[:2]
    m = np.zeros((B, T), bool)
    if inp.cu_seqlens is None:
        m[:] = True
    else:
        cu = inp.cu_seqlens.tolist()
        m[0, cu[0]:cu[-1]] = True
    return m


def check(got, ref, inp, names=("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "dS0")):
    rows = rows_in_sequences(inp)
    gap, fac, z = gate_terms(inp)
    tie = (np.abs(gap) < TIE) & rows[:, :, None, None]
    open_dx = ref["dlam"] * fac        # dg on the open side of the kink
    slack = {"dg": np.where(tie, np.abs(open_dx) * 1.01, 0.0),
             "ddt_bias": np.where(tie, np.abs(open_dx), 0.0).sum(axis=(0, 1)),
             "dA_log": np.where(tie, np.abs(ref["dlam"] * z), 0.0).sum(axis=(0, 1, 3)) * 1.01}
    worst = {}
    for n in names:
        a, b = got[n], ref[n]
        extra = slack.get(n)
        if n in ("dq", "dk", "dv", "dg", "dbeta"):
            a, b = a[rows], b[rows]
            if extra is not None:
                extra = extra[rows]
        if b.size == 0:
            continue
        assert np.all(np.isfinite(a)), n
        diff = a - b
        if extra is not None:
            diff = np.sign(diff) * np.maximum(np.abs(diff) - extra, 0.0)
        nb = np.linalg.norm(b)
        rel = np.linalg.norm(diff) / nb if nb > 0 else np.linalg.norm(diff)
        mx = np.abs(diff).max() / max(np.abs(b).max(), 1e-30)
        worst[n] = (rel, mx)
        assert rel <= REL and mx <= MAXREL, (n, rel, mx)
    return worst


@pytest.mark.parametrize("init", [None, "f32", "bf16"])
def test_fixed_length_ragged(init):
    """T = 200: three full 64-token chunks and a ragged one of 8 tokens."""
    inp, dO, dSf = case(init=init, seed={None: 1, "f32": 2, "bf16": 3}[init])
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    for sch in SCHEDULES:
        check(run_gpu(inp, dO, dSf, schedule=sch), ref, inp)


def test_varlen_edge_lengths():
    """Empty, 1-token, sub-chunk-boundary and chunk-boundary sequences in one batch."""
    lengths = [0, 1, 7, 8, 9, 63, 64, 65, 130, 3]
    inp, dO, dSf = case(lengths=lengths, H=2, init="f32", seed=4)
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    for sch in SCHEDULES:
        got = run_gpu(inp, dO, dSf, schedule=sch)
        check(got, ref, inp)
        # an empty sequence passes dL/dS_final through unchanged
        np.testing.assert_array_equal(got["dS0"][0], dSf[0].double().numpy())


def test_long_sequences_many_chunks():
    """Two sequences of 1000 and 700 tokens (16 and 11 chunks, ragged ends): the dS
    hand-off from chunk to chunk over many chunks, with an fp32 initial state."""
    inp, dO, dSf = case(lengths=[1000, 700], H=2, init="f32", seed=11)
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    for sch in SCHEDULES:
        check(run_gpu(inp, dO, dSf, schedule=sch), ref, inp)


def test_no_final_state_gradient_and_strong_decay():
    """dL/dS_final = 0 and g ~ N(0, 2) (the clamp holds on many channels)."""
    inp, dO, _ = case(T=150, H=2, g_std=2.0, seed=6, dfinal=False)
    ref = oracle.backward_inputs(inp, dO, None, want_dlam=True)
    for sch in SCHEDULES:
        check(run_gpu(inp, dO, None, schedule=sch), ref, inp)


def test_more_units_than_resident_ctas():
    """200 (sequence, head) units on a persistent grid of at most 148 CTAs."""
    rng = np.random.default_rng(7)
    lengths = [int(x) for x in rng.integers(1, 40, size=100)]
    inp, dO, dSf = case(lengths=lengths, H=2, init="bf16", seed=7)
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    for sch in SCHEDULES:
        check(run_gpu(inp, dO, dSf, schedule=sch), ref, inp)


def test_decay_at_the_lower_bound():
    """Every token of half the channels at lam = lower_bound = -5 (g far above the clamp),
    the other half with weak decay: the per-block factors of the chunked schedule reach
    their widest range there (e^(+-75) across a 16-token block) and must stay finite."""
    inp, dO, dSf = case(T=300, B=1, H=2, init="f32", seed=12)
    g = inp.g.float()
    g[..., 0::2] = 20.0 + 0.1 * g[..., 0::2]   # softplus ~ 20: z << -5, the clamp holds
    g[..., 1::2] = -6.0 + 0.1 * g[..., 1::2]   # softplus ~ 2.5e-3: weak decay
    inp.g = g.to(torch.bfloat16)
    inp.lower_bound = -5.0
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    for sch in SCHEDULES:
        check(run_gpu(inp, dO, dSf, schedule=sch), ref, inp)


@pytest.mark.parametrize("sch", SCHEDULES)
def test_zero_length(sch):
    """T = 0: every output is the pass-through of dL/dS_final (or zeros)."""
    inp, dO, dSf = case(T=0, B=2, H=2, init="f32", seed=8)
    got = run_gpu(inp, dO, dSf, schedule=sch)
    np.testing.assert_array_equal(got["dS0"], dSf.double().numpy())
    assert np.all(got["dA_log"] == 0) and np.all(got["ddt_bias"] == 0)


def test_adjoint_identity_on_the_gpu():
    """<dO, out> + <dSf, final> = <dv, v> + <dS0, S0> with out and final from the
    forward kernel and dv, dS0 from the backward kernel (the two CUDA paths checked
    against each other through an identity of the operator)."""
    inp, dO, dSf = case(T=256, H=2, init="f32", seed=9)
    d = lambda t: t.cuda()
    out, fin = kda().kda_fwd(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale,
                             d(inp.A_log), d(inp.dt_bias), inp.lower_bound,
                             initial_state=d(inp.initial_state))
    got = run_gpu(inp, dO, dSf)
    lhs = float((out.double().cpu() * dO.double()).sum() + (fin.double().cpu() * dSf.double()).sum())
    rhs = float((torch.from_numpy(got["dv"]) * inp.v.double()).sum()
                + (torch.from_numpy(got["dS0"]) * inp.initial_state.double()).sum())
    # the forward kernel's out carries ~2e-3 relative error (tf32/fp16 products)
    assert abs(lhs - rhs) <= 1e-2 * (abs(lhs) + abs(rhs)), (lhs, rhs)


def test_full_size_sampled_units():
    """The long-context prefill shape (B=4, T=32768, H=32, g ~ N(0, 2)) in the launch
    the benchmark times; two (sequence, head) units against the oracle run on just
    those units."""
    inp = ki.make_inputs(ki.WORKLOADS[3], 3)
    gen = torch.Generator().manual_seed(3)
    dO = torch.randn(inp.v.shape, generator=gen).to(torch.bfloat16)
    got = run_gpu(inp, dO, None, on_device=True)
    for (s, h) in [(0, 0), (3, 31)]:
        cut = lambda t: t[s:s + 1, :, h:h + 1].contiguous()
        sub = ki.KDAInputs(q=cut(inp.q), k=cut(inp.k), v=cut(inp.v), g=cut(inp.g),
                           beta=inp.beta[s:s + 1, :, h:h + 1].contiguous(),
                           A_log=inp.A_log[h:h + 1].contiguous(),
                           dt_bias=inp.dt_bias[h:h + 1].contiguous(), scale=inp.scale,
                           lower_bound=inp.lower_bound, initial_state=None, cu_seqlens=None)
        ref = oracle.backward_inputs(sub, cut(dO), None, want_dlam=True)
        one = {n: got[n][s:s + 1, :, h:h + 1].cpu().double().numpy()
               for n in ("dq", "dk", "dv", "dg", "dbeta")}
        one["dS0"] = got["dS0"][s:s + 1, h:h + 1].cpu().double().numpy()
        check(one, ref, sub, names=("dq", "dk", "dv", "dg", "dbeta", "dS0"))
