"""The chunked (per-64-token matrix) form of the backward equals the oracle's token-by-
token reverse mode (CPU, fp64).  This pins the algebra a tensor-core backward kernel
would run: the per-chunk adjoints of the WY form (dU, dY, dT, dS0, the solve's adjoint
through M^-1, the decay-weighted products) and the reverse pass of dS over chunks."""
import numpy as np
import pytest
import torch

import chunked_bwd_ref as cb
import kda_inputs as ki
import oracle

NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "dS0", "dlam")


def run(lengths=None, T=150, H=2, init="f32", g_std=1.0, seed=0, dfinal=True, C=64):
    inp = ki.make_inputs(ki.Workload("cbwd", B=2, T=T, H=H, init_state=init, g_std=g_std), seed,
                         lengths=lengths)
    gen = torch.Generator().manual_seed(seed + 7)
    dO = torch.randn(inp.v.shape, generator=gen).to(torch.bfloat16)
    N = inp.num_seqs
    dSf = torch.randn((N, H, 128, 128), generator=gen) * 0.1 if dfinal else None
    ref = oracle.backward_inputs(inp, dO, dSf, want_dlam=True)
    got = cb.backward_inputs(inp, dO, dSf, C=C)
    for n in NAMES:
        nb = np.linalg.norm(ref[n])
        err = np.linalg.norm(got[n] - ref[n]) / (nb if nb > 0 else 1.0)
        assert err <= 1e-11, (n, err)


@pytest.mark.parametrize("C", [16, 64])
def test_fixed_length_ragged(C):
    run(C=C, seed=1)


def test_varlen_with_empty_and_boundary_lengths():
    run(lengths=[0, 1, 63, 64, 65, 130], init="bf16", seed=2)


def test_strong_decay_without_state_gradient():
    run(T=200, g_std=2.0, init=None, dfinal=False, seed=3)


# Precision plan for a tensor-core backward, emulated on the CPU (chunked_bwd_ref's
# tiled form with operand rounding): A and P in tf32 (as the forward kernel), their
# adjoints in fp32, every other product operand fp16 with a power-of-two scale per row
# or column (along the non-contracted dimension), T fp16, the solve adjoint tf32.
BWD_PLAN = {"APf": "tf32", "APb": "f32", "F": "f16", "T": "f16", "dM": "tf32", "Minv": "f32"}
BARS = ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "dS0")


def _case(g_std, init, seed):
    inp = ki.make_inputs(ki.Workload("cbp", B=1, T=200, H=2, init_state=init, g_std=g_std), seed)
    gen = torch.Generator().manual_seed(2)
    dO = torch.randn(inp.v.shape, generator=gen).to(torch.bfloat16)
    dSf = torch.randn((1, 2, 128, 128), generator=gen) * 0.1
    return inp, dO, dSf, oracle.backward_inputs(inp, dO, dSf, want_dlam=True)


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_tiled_form_equals_the_oracle():
    """Sub-blocks with mid-block reference tokens (no rounding) change nothing."""
    inp, dO, dSf, ref = _case(2.0, "f32", 5)
    got = cb.backward_inputs(inp, dO, dSf, tiled=True)
    for n in BARS:
        assert _rel(got[n], ref[n]) <= 1e-11, n


@pytest.mark.parametrize("g_std,init,seed", [(2.0, "f32", 5), (1.0, None, 6)])
def test_backward_precision_plan_meets_the_bars(g_std, init, seed):
    inp, dO, dSf, ref = _case(g_std, init, seed)
    got = cb.backward_inputs(inp, dO, dSf, prec=BWD_PLAN)
    for n in BARS:
        assert _rel(got[n], ref[n]) <= 1e-3, (n, _rel(got[n], ref[n]))


def test_tf32_adjoints_of_the_decay_weighted_products_break_the_gate_gradients():
    """Why the plan keeps those products in fp32: with their operands in tf32 the gate
    gradients (sums over the chunk of nearly cancelling terms) miss the bar tenfold."""
    inp, dO, dSf, ref = _case(2.0, "f32", 5)
    got = cb.backward_inputs(inp, dO, dSf, prec=dict(BWD_PLAN, APb="tf32"))
    assert _rel(got["ddt_bias"], ref["ddt_bias"]) > 1e-2
    assert _rel(got["dv"], ref["dv"]) <= 1e-3  # the rest is unaffected


def test_three_tf32_products_recover_the_adjoints():
    """The fp32-grade adjoint products the plan needs, made of tf32 tensor-core products:
    a b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi (halves rounded to tf32) meets the bars."""
    inp, dO, dSf, ref = _case(2.0, "f32", 5)
    got = cb.backward_inputs(inp, dO, dSf, prec=dict(BWD_PLAN, APb="tf32x3"))
    for n in BARS:
        assert _rel(got[n], ref[n]) <= 1e-3, (n, _rel(got[n], ref[n]))


def _split_factors_f32(G, ref_of_j_block, clamp=120.0):
    """e^(G_i - G_j) for j <= i as the product of two float32 factors split at the
    reference token r = ref(block of j or i), in base 2 with the exponent clamped as the
    chunked backward kernel does; returns the [C, C] products in float64."""
    L2E = np.float32(1.4426950408889634)
    G2 = (G.astype(np.float32) * L2E).astype(np.float32)
    C = G.shape[0]
    out = np.zeros((C, C))
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        for i in range(C):
            for j in range(i + 1):
                r = ref_of_j_block(i, j)
                a = np.exp2(np.minimum(np.float32(G2[i] - G2[r]), np.float32(clamp)), dtype=np.float32)
                b = np.exp2(np.minimum(np.float32(G2[r] - G2[j]), np.float32(clamp)), dtype=np.float32)
                out[i, j] = float(np.float32(a * b))
    return out


@pytest.mark.parametrize("side", ["row", "column"])
def test_block_reference_split_stays_in_fp32_range(side):
    """The chunked backward kernel splits e^(G_i - G_j) at a reference token of a 16-token
    block (row side and A/P: the last token of j's block; column side: the first token of
    i's block).  At the steepest decay the operator allows (lam = lower_bound = -5 on
    every token) both factors must stay finite and their product must match e^(G_i - G_j)
    to float32 accuracy wherever it is above float32's normal range; below it, the
    product may flush to zero.  A wrong reference (e.g. a chunk-wide one) overflows."""
    C = 64
    lam = np.full(C, -5.0)
    G = np.cumsum(lam)
    exact = np.exp(G[:, None] - G[None, :])
    if side == "row":
        ref = lambda i, j: (j // 16) * 16 + 15
    else:
        ref = lambda i, j: (i // 16) * 16
    got = _split_factors_f32(G, ref)
    lower = np.tril(np.ones((C, C), bool))
    assert np.all(np.isfinite(got[lower]))
    big = lower & (exact > 1e-30)
    rel = np.abs(got[big] - exact[big]) / exact[big]
    # the exponent G*log2(e) is rounded to float32 (|G| <= 320): ~2e-5 relative at most
    assert rel.max() < 1e-4, rel.max()
    small = lower & (exact <= 1e-30)
    assert np.all(got[small] <= 1e-29)
    # a chunk-wide reference (token 0) is what the blocks avoid: its factors overflow
    chunk_ref = _split_factors_f32(G, lambda i, j: 0, clamp=1e9)
    assert not np.all(np.isfinite(chunk_ref[lower]))
