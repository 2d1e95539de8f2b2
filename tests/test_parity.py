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


@pytest.mark.parametrize("fill", [0x7FC0, 0x7F80, 0xFF80, 0x7F7F])  # NaN, +Inf, -Inf, bf16 max
def test_rows_after_the_last_sequence_do_not_matter(fill):
    """A varlen batch may end before its buffer does (cu_seqlens[N] < rows).  The last
    sequence's final 64-token tile then also covers rows that belong to no sequence.
    Whatever those rows hold (here NaN, Inf or the largest bf16 in every input), every
    result must be bit-identical to the run with zero rows there, and the rows
    themselves must not be written."""
    lengths, pad = [70, 33, 129], 40
    inp = small(lengths=lengths, init="f32", seed=9)
    rows = int(inp.cu_seqlens[-1])
    d = dev(inp)

    def padded(t, bits):
        extra = torch.full((1, pad) + tuple(t.shape[2:]), bits, dtype=torch.int16,
                           device=t.device).view(torch.bfloat16)
        return torch.cat([t, extra], dim=1).contiguous()

    runs = []
    for bits in (0, fill - 0x10000 if fill >= 0x8000 else fill):
        call = dict(d)
        for name in ("q", "k", "v", "g", "beta"):
            call[name] = padded(d[name], bits)
        out = torch.full((1, rows + pad, inp.H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
        o, f = kda.kda_fwd(**call, out=out)
        torch.cuda.synchronize()
        assert kda.kda_device_status(reset=True) == 0
        runs.append((o.cpu(), f.cpu()))
    (o0, f0), (o1, f1) = runs
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    assert torch.equal(f0, f1)
    assert torch.all(o1[:, rows:] == 7.0), "rows outside every sequence were written"
    out_r, fin_r = oracle.forward_inputs(inp)
    assert_parity(inp, o1[:, :rows].float().numpy().astype(np.float64),
                  f1.numpy().astype(np.float64), out_r, fin_r, what=f"pad fill {fill:#x}")



@pytest.mark.parametrize("fill", [0x7FC0, 0xFF80])  # NaN, -Inf
def test_a_sequence_ignores_the_bits_of_the_next_one(fill):
    """Each sequence's last 64-token tile also covers the first rows of the sequence after
    it.  With every input of sequence 1 set to NaN or -Inf, sequences 0 and 2 must give
    bit-identical out and final states to the run where sequence 1 is clean."""
    lengths = [70, 45, 100]
    inp = small(lengths=lengths, init="f32", seed=21)
    d = dev(inp)
    t0, t1 = lengths[0], lengths[0] + lengths[1]
    bad = dict(d)
    bits = fill - 0x10000 if fill >= 0x8000 else fill
    for name in ("q", "k", "v", "g", "beta"):
        t = d[name].clone()
        t.view(torch.int16)[:, t0:t1] = bits
        bad[name] = t
    runs = []
    for call in (d, bad):
        o, f = kda.kda_fwd(**call)
        torch.cuda.synchronize()
        assert kda.kda_device_status(reset=True) == 0
        runs.append((o.cpu(), f.cpu()))
    (o0, f0), (o1, f1) = runs
    keep = torch.cat([torch.arange(0, t0), torch.arange(t1, sum(lengths))])
    assert torch.equal(o0[:, keep].view(torch.int16), o1[:, keep].view(torch.int16))
    assert torch.equal(f0[[0, 2]], f1[[0, 2]])


def test_many_short_sequences_with_empty_ones():
    """More (sequence, head) units than SMs, most of them a chunk or two long and a
    quarter of them empty: the work is dealt to a persistent grid in decreasing length
    (every unit is compared; empty sequences return their initial state)."""
    rng = np.random.default_rng(77)
    lengths = [int(x) if rng.random() > 0.25 else 0 for x in rng.integers(1, 150, size=400)]
    inp = small(lengths=lengths, H=2, init="bf16", seed=78)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what="400 short sequences")
    for s_, n in enumerate(lengths):
        if n == 0:
            np.testing.assert_array_equal(fin_g[s_], inp.initial_state[s_].float().numpy())


def test_fixed_length_more_units_than_sms():
    """B * H = 200 units of one length (> 148 SMs): a persistent grid takes two units on
    some CTAs, chaining the second unit's start behind the first one's drain."""
    w = ki.Workload("b5h40", B=5, T=130, H=40, init_state="f32", g_std=1.0)
    inp = ki.make_inputs(w, 5)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_g, fin_g = run_gpu(inp)
    assert_parity(inp, out_g, fin_g, out_r, fin_r, what="B=5 H=40")

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
    1: [(0, h) for h in range(32)],  # the one sequence, every head
    2: "ends",  # every head of the longest sequence; shortest and median, several heads
    3: [(b, h) for b in range(4) for h in range(b, 32, 4)],  # every entry x 8 heads (32 pairs)
    4: "ends",
}


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_workload_parity(cfg):
    inp = ki.make_inputs(cfg)
    pairs = SAMPLES[cfg]
    if pairs == "ends":
        lens = [n for (_, _, n) in inp.seq_bounds()]
        order = np.argsort(lens, kind="stable")
        seqs = [int(order[0]), int(order[1]), int(order[len(order) // 2])]
        pairs = [(s, h) for i, s in enumerate(seqs) for h in (i % inp.H, (5 * i + 3) % inp.H)]
        pairs += [(int(order[-1]), h) for h in range(inp.H)]
    mask = None if pairs is None else mask_for(inp, pairs)
    out_r, fin_r = oracle.forward_inputs(inp, mask=mask)
    out_g, fin_g = run_gpu(inp)
    r = assert_parity(inp, out_g, fin_g, out_r, fin_r, pairs=pairs, what=f"config {cfg}")
    print(f"config {cfg}: {r}")


# ---------------------------------------------------------------------------
# State variants (kda_fwd_ex): transposed layout, bf16 final state.
# ---------------------------------------------------------------------------
def bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to bf16 (nearest even), returned as float64."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("init", ["f32", "bf16"])
def test_transposed_state_layout_is_the_transpose(init):
    """S[v][k] in and out gives exactly the transposes of the S[k][v] call, and the same out."""
    w = ki.Workload("vk", B=2, T=200, H=3, init_state=init)
    inp = ki.make_inputs(w, 21)
    d = dev(inp)
    out_kv, fin_kv = kda.kda_fwd(**d)
    d_vk = dict(d, initial_state=d["initial_state"].transpose(-1, -2).contiguous())
    out_vk, fin_vk = kda.kda_fwd_ex(**d_vk, state_layout="vk")
    torch.cuda.synchronize()
    assert kda.kda_device_status(reset=True) == 0
    assert torch.equal(out_vk, out_kv)
    assert torch.equal(fin_vk, fin_kv.transpose(-1, -2))
    out_r, fin_r = oracle.forward_inputs(inp)
    assert_parity(inp, out_vk.float().cpu().numpy().astype(np.float64),
                  fin_vk.transpose(-1, -2).cpu().numpy().astype(np.float64), out_r, fin_r,
                  what=f"VK layout init={init}")


@pytest.mark.parametrize("layout", ["kv", "vk"])
def test_bf16_final_state(layout):
    """The bf16 final state is the fp32 one rounded to nearest even (bit for bit), and
    within the fp32 bar plus one bf16 half-ulp (2^-9 relative) of the oracle."""
    inp = small(T=333, H=2, init="f32", seed=8)
    d = dev(inp)
    if layout == "vk":
        d["initial_state"] = d["initial_state"].transpose(-1, -2).contiguous()
    out32, fin32 = kda.kda_fwd_ex(**d, state_layout=layout)
    out16, fin16 = kda.kda_fwd_ex(**d, state_layout=layout, final_state_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert kda.kda_device_status(reset=True) == 0
    assert fin16.dtype == torch.bfloat16 and torch.equal(out16, out32)
    assert torch.equal(fin16, fin32.to(torch.bfloat16))
    _, fin_r = oracle.forward_inputs(inp)
    f = fin16.double().cpu().numpy()
    if layout == "vk":
        f = np.swapaxes(f, -1, -2)
    assert rel(f, fin_r) <= FIN_REL + 2.0 ** -9


def test_zero_tokens_state_variants():
    """T = 0: the final state is the initial one, converted (both states in the same
    layout, so no transpose)."""
    inp = small(T=0, init="f32")
    d = dev(inp)
    _, fin = kda.kda_fwd_ex(**d, state_layout="vk", final_state_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(fin.cpu(), inp.initial_state.to(torch.bfloat16))


# ---------------------------------------------------------------------------
# Decode step (kda_decode): one token per sequence, state in HBM.
# ---------------------------------------------------------------------------
def decode_inputs(N, H, seed, g_std=1.0):
    w = ki.Workload("decode", B=N, T=1, H=H, init_state="f32", g_std=g_std)
    return ki.make_inputs(w, seed)


def run_decode(inp, in_place=True):
    d = dev(inp)
    sq = lambda t: t[:, 0].contiguous()  # [N,1,H,D] -> [N,H,D]
    state = d["initial_state"].clone()
    out, st = kda.kda_decode(sq(d["q"]), sq(d["k"]), sq(d["v"]), sq(d["g"]), d["beta"][:, 0].contiguous(),
                             d["scale"], d["A_log"], d["dt_bias"], d["lower_bound"], state,
                             state_out=None if in_place else torch.empty_like(state))
    torch.cuda.synchronize()
    return out, st


@pytest.mark.parametrize("N,H,g_std", [(1, 1, 1.0), (5, 3, 1.0), (64, 32, 2.0)])
def test_decode_matches_oracle(N, H, g_std):
    inp = decode_inputs(N, H, seed=N + H, g_std=g_std)
    out, st = run_decode(inp)
    out_r, fin_r = oracle.forward_inputs(inp)
    og = out.float().cpu().numpy().astype(np.float64)[:, None]
    assert_parity(inp, og, st.cpu().numpy().astype(np.float64), out_r, fin_r, what=f"decode N={N}")


def test_decode_in_place_equals_out_of_place():
    inp = decode_inputs(7, 4, seed=3)
    a = run_decode(inp, in_place=True)
    b = run_decode(inp, in_place=False)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("layout,in_dt,out_dt", [("vk", torch.float32, torch.float32),
                                                  ("kv", torch.bfloat16, torch.float32),
                                                  ("vk", torch.bfloat16, torch.bfloat16)])
def test_decode_state_variants(layout, in_dt, out_dt):
    """kda_decode_ex on the state variants equals kda_decode on the fp32 S[k][v] copy of the
    same state: bit for bit with fp32 in and out, the bf16 result being that fp32 state
    rounded to nearest even."""
    inp = decode_inputs(9, 4, seed=31)
    d = dev(inp)
    sq = lambda t: t[:, 0].contiguous()
    args = (sq(d["q"]), sq(d["k"]), sq(d["v"]), sq(d["g"]), d["beta"][:, 0].contiguous(),
            d["scale"], d["A_log"], d["dt_bias"], d["lower_bound"])
    s_kv = d["initial_state"].to(in_dt).float()  # the values the variant call sees
    o_ref, st_ref = kda.kda_decode(*args, s_kv.clone())
    s_in = d["initial_state"].to(in_dt)
    if layout == "vk":
        s_in = s_in.transpose(-1, -2).contiguous()
    o, st = kda.kda_decode_ex(*args, s_in, state_layout=layout, state_out_dtype=out_dt)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    st_kv = st.transpose(-1, -2) if layout == "vk" else st
    assert torch.equal(st_kv, st_ref.to(out_dt))


def test_vk_prefill_chains_into_vk_decode():
    """A prefill in the transposed layout with a bf16 final state hands it to decode in the
    same layout; the result matches the oracle over T + 1 tokens under the bars."""
    full = small(T=130, H=3, init="f32", seed=14)
    d = dev(full)
    part = {n: d[n][:, :129].contiguous() for n in ("q", "k", "v", "g", "beta")}
    init_vk = d["initial_state"].transpose(-1, -2).contiguous()
    _, fin_vk = kda.kda_fwd_ex(**dict(d, **part, initial_state=init_vk), state_layout="vk",
                               final_state_dtype=torch.bfloat16)
    last = lambda t: t[:, 129].contiguous()
    out_dec, st = kda.kda_decode_ex(last(d["q"]), last(d["k"]), last(d["v"]), last(d["g"]),
                                    d["beta"][:, 129].contiguous(), d["scale"], d["A_log"],
                                    d["dt_bias"], d["lower_bound"], fin_vk, state_layout="vk",
                                    state_out_dtype=torch.float32)
    torch.cuda.synchronize()
    out_r, fin_r = oracle.forward_inputs(full)
    od = out_dec.float().cpu().numpy().astype(np.float64)
    assert np.abs(od - out_r[:, 129]).max() <= OUT_MAXABS and rel(od, out_r[:, 129]) <= OUT_REL
    fs = st.transpose(-1, -2).cpu().numpy().astype(np.float64)
    # the handed-over state was rounded to bf16 (about 2^-9 relative), so the final state
    # carries that rounding on top of the kernel's own error
    assert rel(fs, fin_r) <= 4e-3


def test_prefill_then_decode_equals_longer_prefill():
    """kda_fwd over T tokens, then kda_decode of token T+1, matches kda_fwd over T+1."""
    full = small(T=130, H=3, init="f32", seed=12)
    d = dev(full)
    out_full, fin_full = kda.kda_fwd(**d)
    part = {n: d[n][:, :129].contiguous() for n in ("q", "k", "v", "g", "beta")}
    _, fin_129 = kda.kda_fwd(**dict(d, **part))
    last = lambda t: t[:, 129].contiguous()
    out_dec, st = kda.kda_decode(last(d["q"]), last(d["k"]), last(d["v"]), last(d["g"]),
                                 d["beta"][:, 129].contiguous(), d["scale"], d["A_log"],
                                 d["dt_bias"], d["lower_bound"], fin_129)
    torch.cuda.synchronize()
    # each path against the oracle under the stated bars, and the two GPU paths against
    # each other under the same bars (each differs from the oracle by less)
    out_r, fin_r = oracle.forward_inputs(full)
    od = out_dec.float().cpu().numpy().astype(np.float64)
    assert np.abs(od - out_r[:, 129]).max() <= OUT_MAXABS and rel(od, out_r[:, 129]) <= OUT_REL
    assert rel(st.cpu().numpy().astype(np.float64), fin_r) <= FIN_REL
    assert rel(od, out_full[:, 129].float().cpu().numpy()) <= OUT_REL
    assert rel(st.cpu().numpy(), fin_full.cpu().numpy()) <= FIN_REL


@pytest.mark.parametrize("case", ["batch3", "varlen"])
def test_pipelined_host_entry_matches_device_entry(case):
    """The host entry point splits the call into pieces (batch entries / groups of
    sequences) with overlapped copies; the result is bit for bit the device call's."""
    if case == "batch3":
        inp = ki.make_inputs(ki.Workload("h3", B=3, T=200, H=2, init_state="f32"), 31)
    else:
        inp = small(lengths=[70, 0, 1, 130, 64, 257, 3, 90, 33, 200], init="bf16", seed=32)
    out_d, fin_d = run_gpu(inp)
    pin = lambda t: None if t is None else t.pin_memory()
    out_h, fin_h = kda.kda_fwd_host(pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.g), pin(inp.beta),
                                    inp.scale, inp.A_log, inp.dt_bias, inp.lower_bound,
                                    initial_state=pin(inp.initial_state), cu_seqlens=inp.cu_seqlens)
    for (b, t0, nn) in inp.seq_bounds():
        np.testing.assert_array_equal(out_h[b, t0:t0 + nn].float().numpy(), out_d[b, t0:t0 + nn])
    np.testing.assert_array_equal(fin_h.numpy(), fin_d)



def test_host_entry_point_on_a_nan_workspace_with_rows_past_the_last_sequence():
    """kda_fwd_host copies each piece into a caller workspace; the last tile of a piece
    also covers workspace rows that nothing wrote (here all bytes 0xFF, NaN as bf16),
    including rows after the last sequence (cu_seqlens[N] < rows).  The kernel clears
    them on chip, so the result is bit for bit the device call's on clean buffers."""
    lengths, pad = [70, 45, 129], 50
    inp = small(lengths=lengths, init="f32", seed=47)
    rows = int(inp.cu_seqlens[-1])
    out_d, fin_d = run_gpu(inp)
    def padded(t):
        extra = torch.zeros((1, pad) + tuple(t.shape[2:]), dtype=t.dtype)
        return torch.cat([t, extra], dim=1).contiguous().pin_memory()
    H = inp.H
    ws = torch.full((kda.kda_fwd_host_workspace_size(1, rows + pad, H, num_seqs=len(lengths),
                                                     initial_state_dtype=kda.KDA_STATE_F32),),
                    255, dtype=torch.uint8, device="cuda")
    out_h, fin_h = kda.kda_fwd_host(padded(inp.q), padded(inp.k), padded(inp.v), padded(inp.g),
                                    padded(inp.beta), inp.scale, inp.A_log, inp.dt_bias,
                                    inp.lower_bound, initial_state=inp.initial_state.pin_memory(),
                                    cu_seqlens=inp.cu_seqlens, workspace=ws)
    assert kda.kda_device_status(reset=True) == 0
    np.testing.assert_array_equal(out_h[:, :rows].float().numpy(), out_d)
    np.testing.assert_array_equal(fin_h.numpy(), fin_d)

@pytest.mark.gpu
def test_device_offset_check_rejects_bad_cu_seqlens():
    """With checks on, a varlen call whose cu_seqlens is not non-decreasing within
    [0, B*T] returns KDA_ERR_SEQLENS before any kernel runs (outputs untouched); a valid
    one gives the same bits as with checks off."""
    inp = small(lengths=[5, 10, 20], init="f32", seed=41)
    d = lambda t: None if t is None else t.cuda()
    args = (d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale, d(inp.A_log),
            d(inp.dt_bias), inp.lower_bound)
    ref, ref_fin = kda.kda_fwd(*args, initial_state=d(inp.initial_state), cu_seqlens=d(inp.cu_seqlens))
    old = kda.kda_set_checks(1)
    try:
        out, fin = kda.kda_fwd(*args, initial_state=d(inp.initial_state), cu_seqlens=d(inp.cu_seqlens))
        torch.cuda.synchronize()
        assert torch.equal(out, ref) and torch.equal(fin, ref_fin)
        for bad in ([0, 10, 5, 35], [0, 5, 15, 36], [-1, 5, 15, 35]):
            cu = torch.tensor(bad, dtype=torch.int64, device="cuda")
            sentinel = torch.full_like(ref, 7.0)
            with pytest.raises(kda.KDAError) as e:
                kda.kda_fwd(*args, initial_state=d(inp.initial_state), cu_seqlens=cu, out=sentinel)
            assert e.value.code == -14
            dO = torch.zeros_like(ref)
            with pytest.raises(kda.KDAError) as e:
                kda.kda_bwd(*args, dO, initial_state=d(inp.initial_state), cu_seqlens=cu)
            assert e.value.code == -14
            torch.cuda.synchronize()
            assert bool((sentinel == 7.0).all())
    finally:
        kda.kda_set_checks(old)
