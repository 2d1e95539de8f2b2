"""GPU parity of libkda against the fp64 CPU oracle, through the C ABI.

Bars (the operator's stated tolerances): bf16 out has max-abs error <= 3e-2 and
relative L2 error <= 5e-3; the fp32 final state has relative L2 error <= 1e-3.
Small cases compare every element; the full-size workloads compare the
(sequence, head) pairs the oracle computes one by one (a bounded sample).
"""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_09_b200 as kda
import oracle

pytestmark = pytest.mark.gpu

OUT_MAXABS, OUT_REL, FIN_REL = 3e-2, 5e-3, 1e-3


def dev(inp):
    d = "cuda"
    return dict(q=inp.q.to(d), k=inp.k.to(d), v=inp.v.to(d), g=inp.g.to(d), beta=inp.beta.to(d),
                scale=inp.scale, A_log=inp.A_log.to(d), dt_bias=inp.dt_bias.to(d),
                lower_bound=inp.lower_bound,
                initial_state=None if inp.initial_state is None else inp.initial_state.to(d),
                cu_seqlens=None if inp.cu_seqlens is None else inp.cu_seqlens.to(d))


def run_gpu(inp):
    out, fin = kda.kda_fwd(**dev(inp))
    torch.cuda.synchronize()
    assert kda.kda_device_status(reset=True) == 0, "a bounded wait in the kernel gave up"
    return out.float().cpu().numpy().astype(np.float64), fin.cpu().numpy().astype(np.float64)


def rel(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


def gather(inp, out, fin, pairs):
    seqs = inp.seq_bounds()
    o = [out[b, t0:t0 + n, h].ravel() for (s, h) in pairs for (b, t0, n) in [seqs[s]]]
    f = [fin[s, h].ravel() for (s, h) in pairs]
    return np.concatenate(o) if o else np.zeros(0), np.concatenate(f)


def assert_parity(inp, out_g, fin_g, out_r, fin_r, pairs=None, what=""):
    if pairs is None:
        pairs = [(s, h) for s in range(inp.num_seqs) for h in range(inp.H)]
    og, fg = gather(inp, out_g, fin_g, pairs)
    orf, fr = gather(inp, out_r, fin_r, pairs)
    assert np.isfinite(og).all() and np.isfinite(fg).all(), f"{what}: non-finite GPU output"
    if og.size:
        e_max = np.abs(og - orf).max()
        e_rel = rel(og, orf)
        assert e_max <= OUT_MAXABS, f"{what}: out max-abs {e_max:.3e}"
        assert e_rel <= OUT_REL, f"{what}: out rel-L2 {e_rel:.3e}"
    e_fin = rel(fg, fr)
    assert e_fin <= FIN_REL, f"{what}: final-state rel-L2 {e_fin:.3e}"
    return dict(out_rel=rel(og, orf) if og.size else 0.0, fin_rel=e_fin)


def mask_for(inp, pairs):
    m = np.zeros(inp.num_seqs * inp.H, np.uint8)
    for s, h in pairs:
        m[s * inp.H + h] = 1
    return m


# ---------------------------------------------------------------------------
# Small shapes: every element, ragged tails, edge cases.
# ---------------------------------------------------------------------------
def small(T=64, H=3, seed=0, lengths=None, init=None, g_std=1.0, lb=-5.0):
    w = ki.Workload("edge", B=1, T=T, H=H, g_std=g_std, init_state=init, lower_bound=lb)
    return ki.make_inputs(w, seed, lengths=lengths)


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 63, 64, 65, 127, 128, 129, 200, 512])
@pytest.mark.parametrize("lb", [-5.0, 0.0])
def test_fixed_length_edges(T, lb):
    inp = small(T=T, lb=lb, init="f32", seed=T)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what=f"T={T} lb={lb}")


@pytest.mark.parametrize("init", [None, "f32", "bf16"])
def test_batched_and_states(init):
    w = ki.Workload("b3", B=3, T=150, H=2, init_state=init, g_std=2.0)
    inp = ki.make_inputs(w, 42)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what=f"B=3 init={init}")


@pytest.mark.parametrize("lengths", [[0, 1, 63, 64, 65, 130, 2], [5], [0], [1, 0, 0, 300],
                                     [64] * 9, [129, 1, 257]])
def test_varlen_edges(lengths):
    inp = small(lengths=lengths, init="f32", seed=len(lengths))
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what=f"varlen {lengths}")
    # tokens of zero-length sequences are not written; final = initial there
    for s, n in enumerate(lengths):
        if n == 0:
            np.testing.assert_array_equal(fin_g[s], inp.initial_state[s].numpy())


def test_zero_tokens_returns_initial_state():
    inp = small(T=0, init="bf16")
    out_g, fin_g = run_gpu(inp)
    np.testing.assert_array_equal(fin_g, inp.initial_state.float().numpy())
    inp2 = small(T=0, init=None)
    _, fin2 = run_gpu(inp2)
    assert np.all(fin2 == 0)


def test_weak_decay_long_memory():
    """lower_bound = 0 disables decay: errors accumulate over the whole sequence."""
    inp = small(T=1024, H=2, lb=0.0, init="f32", seed=9)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what="no decay T=1024")


def test_deterministic_reruns():
    inp = small(T=300, H=4, init="f32", seed=3)
    a = run_gpu(inp)
    b = run_gpu(inp)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_chaining_through_final_state():
    """One call over T ~ call(T1) -> final_state -> initial_state -> call(T - T1)."""
    inp = small(T=333, H=2, init="f32", seed=4)
    out_full, fin_full = run_gpu(inp)
    T1 = 100
    part = lambda t, a, b: t[:, a:b].contiguous()
    i1 = ki.KDAInputs(**{**inp.__dict__, **{n: part(getattr(inp, n), 0, T1)
                                             for n in ("q", "k", "v", "g", "beta")}})
    o1, f1 = run_gpu(i1)
    i2 = ki.KDAInputs(**{**inp.__dict__, **{n: part(getattr(inp, n), T1, 333)
                                             for n in ("q", "k", "v", "g", "beta")}},)
    i2.initial_state = torch.from_numpy(f1.astype(np.float32))
    o2, f2 = run_gpu(i2)
    assert rel(np.concatenate([o1, o2], axis=1), out_full) < 2e-3
    assert rel(f2, fin_full) < 5e-4


def test_host_entry_point_matches_device_entry_point():
    inp = ki.make_inputs(0)
    out_d, fin_d = run_gpu(inp)
    pin = lambda t: None if t is None else t.pin_memory()
    out_h, fin_h = kda.kda_fwd_host(pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.g), pin(inp.beta),
                                    inp.scale, inp.A_log, inp.dt_bias, inp.lower_bound)
    np.testing.assert_array_equal(out_h.float().numpy(), out_d)
    np.testing.assert_array_equal(fin_h.numpy(), fin_d)


# ---------------------------------------------------------------------------
# The five workloads at their full sizes.
# ---------------------------------------------------------------------------
SAMPLES = {
    0: None,  # every pair
    1: [(0, 0), (0, 7), (0, 13), (0, 31)],
    2: "ends",  # shortest and longest sequences, several heads
    3: [(0, 0), (1, 9), (2, 22), (3, 31)],
    4: "ends",
}


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_workload_parity(cfg):
    inp = ki.make_inputs(cfg)
    pairs = SAMPLES[cfg]
    if pairs == "ends":
        lens = [n for (_, _, n) in inp.seq_bounds()]
        order = np.argsort(lens)
        seqs = [int(order[0]), int(order[1]), int(order[-1]), int(order[len(order) // 2])]
        pairs = [(s, h) for i, s in enumerate(seqs) for h in (i % inp.H, (5 * i + 3) % inp.H)]
    mask = None if pairs is None else mask_for(inp, pairs)
    out_r, fin_r = oracle.forward_inputs(inp, mask=mask)
    out_g, fin_g = run_gpu(inp)
    r = assert_parity(inp, out_g, fin_g, out_r, fin_r, pairs=pairs, what=f"config {cfg}")
    print(f"config {cfg}: {r}")
