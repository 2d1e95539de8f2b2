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
