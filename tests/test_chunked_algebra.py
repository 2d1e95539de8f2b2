"""The chunked (WY/UT) form the CUDA kernel computes, checked on the CPU.

``tests/chunked_ref.py`` restates the chunk algorithm in NumPy fp64.  These tests pin
it to the token-by-token oracle: the derivation (intra-chunk decay-weighted products,
the unit-triangular solve, U = u - w S, the state update), the inclusive cumulative
sum, partial last chunks, and the 32-token sub-blocks with a mid-block reference
token that keep every decay factor inside the fp32 exponent range.  With the kernel's
operand formats emulated (tf32 for A and P, fp16 for the other products with a
power-of-two per-column scale on S and U), they also show that the precision plan
meets the parity bars on the CPU, before any kernel runs.
"""
import numpy as np
import pytest

import kda_inputs as ki
import oracle
from chunked_ref import chunk_forward_inputs


def rel(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


def small(T, H=2, lb=-5.0, g_std=1.0, init="f32", seed=0, lengths=None):
    w = ki.Workload("chunk", B=1, T=T, H=H, g_std=g_std, init_state=init, lower_bound=lb)
    return ki.make_inputs(w, seed, lengths=lengths)


@pytest.mark.parametrize("C", [16, 64])
@pytest.mark.parametrize("T", [1, 15, 63, 64, 65, 200])
@pytest.mark.parametrize("lb", [-5.0, 0.0])
def test_chunked_form_equals_oracle(C, T, lb):
    inp = small(T, lb=lb, seed=T + C)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_c, fin_c = chunk_forward_inputs(inp, C=C, sub=C // 2)
    assert rel(out_c, out_r) < 1e-10
    assert rel(fin_c, fin_r) < 1e-10


def test_chunked_form_under_clamped_decay():
    """g ~ N(0, 4): most channels sit at lambda = -5, so exp(G) spans e^-320 in a chunk.
    The sub-block references keep each factor within e^+-80; fp64 must still agree."""
    inp = small(300, H=2, g_std=4.0, seed=11)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_c, fin_c = chunk_forward_inputs(inp)
    assert np.isfinite(out_c).all() and np.isfinite(fin_c).all()
    assert rel(out_c, out_r) < 1e-10
    assert rel(fin_c, fin_r) < 1e-10


def test_chunked_form_varlen():
    inp = small(0, lengths=[0, 1, 64, 65, 130], seed=5)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_c, fin_c = chunk_forward_inputs(inp)
    assert rel(out_c, out_r) < 1e-10
    assert rel(fin_c, fin_r) < 1e-10


def test_dropping_the_sub_blocks_overflows():
    """Planted mistake, on the CPU: one reference token for the whole 64-token chunk
    puts factors near e^+-320 (outside fp32) into the products; in fp32 emulation the
    result is no longer finite or no longer accurate, which is why the kernel blocks."""
    inp = small(128, H=1, g_std=4.0, seed=2)
    out_r, _ = oracle.forward_inputs(inp)
    with np.errstate(all="ignore"):
        out_c, _ = chunk_forward_inputs(inp, prec={"Akk": "f32", "Pqk": "f32"}, sub=64)
    bad = (not np.isfinite(out_c).all()) or rel(out_c, out_r) > 1e-3
    assert bad


KERNEL_PREC = {"Akk": "tf32", "Pqk": "tf32", "T": "f16", "kg": "f16", "qg": "f16", "w": "f16",
               "S": "f16", "U": "f16", "kp": "f16", "P": "f16", "v": "bf16"}


@pytest.mark.parametrize("case", ["tiny", "clamped", "nodecay"])
def test_kernel_precision_plan_meets_the_bars(case):
    """Operand rounding of the kernel (T emulated in fp16 for both w and u, which is
    coarser than the kernel's bf16 hi + lo pair for u) against the fp64 oracle, with
    the bf16 rounding of the output, under the parity bars."""
    if case == "tiny":
        inp = ki.make_inputs(0)
    elif case == "clamped":
        inp = small(512, H=2, g_std=2.0, init=None, seed=3)
    else:
        inp = small(1024, H=1, lb=0.0, seed=9)
    out_r, fin_r = oracle.forward_inputs(inp)
    out_c, fin_c = chunk_forward_inputs(inp, prec=KERNEL_PREC)
    out_b = out_c.astype(np.float32)
    out_b = (out_b.view(np.uint32) + 0x7FFF + ((out_b.view(np.uint32) >> 16) & 1)) >> 16 << 16
    out_b = out_b.astype(np.uint32).view(np.float32).astype(np.float64)
    assert np.abs(out_b - out_r).max() <= 3e-2
    assert rel(out_b, out_r) <= 5e-3
    assert rel(fin_c, fin_r) <= 1e-3
