"""Pins of the oracle's bf16 initial-state input (CPU).

The operator takes its initial state in bf16 or fp32 (FlashKDA de código abierto de
Moonshot AI, 7minutos.es, section "Debajo del capó": initial and final states in
bf16 or fp32).  A bf16 state is promoted exactly, so the oracle fed a bf16 state must
behave exactly as when fed the same values in fp32 (whose path the other oracle pins
cover), and with no tokens to process its final state is the promoted input itself.
Distinct states per (sequence, head) make a wrong element offset visible, and values
that are not bf16 patterns of small integers make a wrong element type visible.
"""
import numpy as np
import pytest

import oracle

K = V = 128


def _bf16_bits(rng, shape, std):
    """Random normals rounded to bf16 (round to nearest even), as uint16 bits."""
    x = rng.normal(0.0, std, size=shape).astype(np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def _inputs(rng, B, T, H):
    q, k, g = (_bf16_bits(rng, (B, T, H, K), 1.0) for _ in range(3))
    v = _bf16_bits(rng, (B, T, H, V), 1.0)
    beta = _bf16_bits(rng, (B, T, H), 1.0)
    A_log = np.log(rng.uniform(1.0, 16.0, H)).astype(np.float32)
    dt_bias = rng.normal(0.0, 0.1, (H, K)).astype(np.float32)
    return q, k, v, g, beta, A_log, dt_bias


def _run(args, init, dtype, cu=None):
    q, k, v, g, beta, A_log, dt_bias = args
    return oracle.forward(q, k, v, g, beta, 1.0 / np.sqrt(K), A_log, dt_bias, -5.0,
                          initial_state=init, init_dtype=dtype, cu_seqlens=cu)


@pytest.mark.parametrize("T", [1, 70])
def test_bf16_state_equals_fp32_state_of_the_same_values(T):
    rng = np.random.default_rng(40 + T)
    B, H = 2, 3
    args = _inputs(rng, B, T, H)
    s_bits = _bf16_bits(rng, (B, H, K, V), 0.05)
    out16, fin16 = _run(args, s_bits, oracle.STATE_BF16)
    out32, fin32 = _run(args, _bits_to_f32(s_bits), oracle.STATE_F32)
    assert np.array_equal(out16, out32) and np.array_equal(fin16, fin32)
    # and the state matters: the run without it differs everywhere
    out0, _ = _run(args, None, oracle.STATE_NONE)
    assert np.all(np.abs(out16 - out0).max(axis=(1, 3)) > 0)


def test_bf16_state_varlen_with_an_empty_sequence():
    rng = np.random.default_rng(7)
    H, lens = 2, [33, 0, 70, 1]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    args = _inputs(rng, 1, int(cu[-1]), H)
    s_bits = _bf16_bits(rng, (len(lens), H, K, V), 0.05)
    out16, fin16 = _run(args, s_bits, oracle.STATE_BF16, cu)
    out32, fin32 = _run(args, _bits_to_f32(s_bits), oracle.STATE_F32, cu)
    assert np.array_equal(out16, out32) and np.array_equal(fin16, fin32)
    # the empty sequence returns its own initial state, promoted exactly
    assert np.array_equal(fin16[1], _bits_to_f32(s_bits[1]).astype(np.float64))


def test_bf16_state_with_no_tokens_is_returned_exactly():
    rng = np.random.default_rng(3)
    B, H = 3, 2
    args = _inputs(rng, B, 0, H)
    s_bits = _bf16_bits(rng, (B, H, K, V), 0.05)
    _, fin = _run(args, s_bits, oracle.STATE_BF16)
    assert np.array_equal(fin, _bits_to_f32(s_bits).astype(np.float64))


def test_bf16_state_one_token_closed_form():
    """T = 1 from a bf16 state S0: S1 = Diag(a) S0 + b k^ (v - S0^T Diag(a) k^)^T and
    out = scale S1^T q^, written out here in NumPy from the operator statement."""
    rng = np.random.default_rng(11)
    H = 2
    args = _inputs(rng, 1, 1, H)
    q, k, v, g, beta, A_log, dt_bias = args
    s_bits = _bf16_bits(rng, (1, H, K, V), 0.05)
    out, fin = _run(args, s_bits, oracle.STATE_BF16)
    scale = 1.0 / np.sqrt(K)
    for h in range(H):
        qv = _bits_to_f32(q[0, 0, h]).astype(np.float64)
        kv = _bits_to_f32(k[0, 0, h]).astype(np.float64)
        vv = _bits_to_f32(v[0, 0, h]).astype(np.float64)
        x = _bits_to_f32(g[0, 0, h]).astype(np.float64) + dt_bias[h].astype(np.float64)
        sp = np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))
        a = np.exp(np.maximum(-5.0, -np.exp(np.float64(A_log[h])) * sp))
        b = 1.0 / (1.0 + np.exp(-np.float64(_bits_to_f32(beta[0, 0, h]))))
        qh = qv / np.sqrt(qv @ qv + oracle.EPS)
        kh = kv / np.sqrt(kv @ kv + oracle.EPS)
        S0 = _bits_to_f32(s_bits[0, h]).astype(np.float64)
        Sa = a[:, None] * S0
        S1 = Sa + b * np.outer(kh, vv - Sa.T @ kh)
        assert np.allclose(fin[0, h], S1, rtol=1e-12, atol=1e-14)
        assert np.allclose(out[0, 0, h], scale * S1.T @ qh, rtol=1e-12, atol=1e-14)
