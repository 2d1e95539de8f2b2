"""Pins of the oracle's backward pass (CPU, fp64).

The backward differentiates L = <dO, out> + <dS_final, final> of the operator (the
recurrence of the FlashKDA pages, 7minutos.es "¿Qué es la atención Kimi Delta...?").
It is pinned by things other than itself:
  * central finite differences of the raw-fp64 forward twin, one input at a time
    (a dropped term or a wrong sign in any gradient fails its own case);
  * the exact adjoint identity of the map (v, S0) -> (out, final), which is linear:
    <dO, out> + <dS_final, final> = <dv, v> + <dS0, S0>;
  * the closed form of a single token from a zero state;
  * invariants: dq is orthogonal to q and dk to k when eps = 0 (the outputs do not
    change when q or k is rescaled); with beta -> -inf nothing is written, so dv,
    dk, dbeta vanish; with A_log = -inf the decay is exactly 1, so the gate
    gradients vanish;
  * chaining: the backward over [0, T) equals the backward over [T1, T) fed into
    the backward over [0, T1) through the state gradient at T1.
The forward twin itself is pinned to the pinned bf16-input forward: on bf16 values
the two agree bit for bit.
"""
import zlib

import numpy as np
import pytest
import torch

import kda_inputs as ki
import oracle

LB = -5.0


def rand_case(rng, B=2, T=7, H=2, K=4, V=4, s0=True, g_mu=0.0, g_std=1.0, cu=None):
    N = B if cu is None else len(cu) - 1
    c = dict(q=rng.standard_normal((B, T, H, K)), k=rng.standard_normal((B, T, H, K)),
             v=rng.standard_normal((B, T, H, V)), g=rng.normal(g_mu, g_std, (B, T, H, K)),
             beta=rng.standard_normal((B, T, H)), A_log=np.log(rng.uniform(1, 16, H)),
             dt_bias=rng.normal(0, 0.1, (H, K)),
             S0=rng.standard_normal((N, H, K, V)) * 0.3 if s0 else None)
    c["dO"] = rng.standard_normal((B, T, H, V))
    c["dSf"] = rng.standard_normal((N, H, K, V))
    c["cu"] = None if cu is None else np.asarray(cu, np.int64)
    return c


def loss(c, scale=0.5, **over):
    a = dict(c)
    a.update(over)
    out, fin = oracle.forward_f64(a["q"], a["k"], a["v"], a["g"], a["beta"], scale, a["A_log"],
                                  a["dt_bias"], LB, a["S0"], a["cu"])
    return float((out * a["dO"]).sum() + (fin * a["dSf"]).sum())


def grads(c, scale=0.5, eps=oracle.EPS):
    return oracle.backward(c["q"], c["k"], c["v"], c["g"], c["beta"], scale, c["A_log"],
                           c["dt_bias"], LB, c["dO"], c["S0"], c["dSf"], c["cu"], eps)


def min_clamp_margin(c):
    """Smallest |z - lb| over the case, z = -exp(A_log) softplus(g + dt_bias)."""
    x = c["g"] + c["dt_bias"][None, None]
    sp = np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))
    z = -np.exp(c["A_log"])[None, None, :, None] * sp
    return float(np.abs(z - LB).min())


INPUTS = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("beta", "dbeta"),
          ("A_log", "dA_log"), ("dt_bias", "ddt_bias"), ("S0", "dS0")]


@pytest.mark.parametrize("name,gname", INPUTS)
@pytest.mark.parametrize("layout", ["fixed", "varlen"])
def test_finite_differences(name, gname, layout):
    """<grad, d> equals the central difference of L along a random direction d."""
    rng = np.random.default_rng(zlib.crc32(f"{name}-{layout}".encode()))
    if layout == "fixed":
        c = rand_case(rng, B=2, T=9, H=2, K=4, V=3)
    else:
        c = rand_case(rng, B=1, T=13, H=2, K=5, V=4, cu=[0, 4, 4, 13])
    # the clamp is a kink: keep every z well away from the lower bound
    assert min_clamp_margin(c) > 1e-4
    r = grads(c)
    d = rng.standard_normal(c[name].shape)
    h = 1e-6
    fd = (loss(c, **{name: c[name] + h * d}) - loss(c, **{name: c[name] - h * d})) / (2 * h)
    an = float((r[gname] * d).sum())
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


def test_finite_differences_with_the_clamp_active():
    """Large positive g drives z far below lb on some channels: those channels get zero
    gate gradient, the others still match finite differences."""
    rng = np.random.default_rng(5)
    c = rand_case(rng, B=1, T=8, H=2, K=6, V=3, g_mu=1.5, g_std=3.0)
    assert min_clamp_margin(c) > 1e-4
    x = c["g"] + c["dt_bias"][None, None]
    sp = np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))
    clamped = -np.exp(c["A_log"])[None, None, :, None] * sp < LB
    assert clamped.any() and (~clamped).any()
    r = grads(c)
    assert np.all(r["dg"][clamped] == 0.0)
    for name, gname in [("g", "dg"), ("A_log", "dA_log"), ("dt_bias", "ddt_bias")]:
        d = rng.standard_normal(c[name].shape)
        h = 1e-6
        fd = (loss(c, **{name: c[name] + h * d}) - loss(c, **{name: c[name] - h * d})) / (2 * h)
        an = float((r[gname] * d).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_adjoint_identity_full_head_size():
    """(v, S0) -> (out, final) is linear at fixed q, k, g, beta, so the backward is its
    exact adjoint: <dO, out> + <dSf, final> = <dv, v> + <dS0, S0>."""
    rng = np.random.default_rng(11)
    c = rand_case(rng, B=1, T=70, H=2, K=128, V=128, cu=[0, 30, 70])
    out, fin = oracle.forward_f64(c["q"], c["k"], c["v"], c["g"], c["beta"], 0.3, c["A_log"],
                                  c["dt_bias"], LB, c["S0"], c["cu"])
    r = grads(c, scale=0.3)
    lhs = (out * c["dO"]).sum() + (fin * c["dSf"]).sum()
    rhs = (r["dv"] * c["v"]).sum() + (r["dS0"] * c["S0"]).sum()
    assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + 1.0), (lhs, rhs)


def test_single_token_closed_form():
    """T = 1 from S0 = 0: out = scale b (kh.qh) v, final = b kh v^T, so
    dv = scale b (kh.qh) dO + b dSf^T kh, db = scale (kh.qh)(v.dO) + kh^T dSf v,
    dqh = scale b (v.dO) kh, dkh = scale b (v.dO) qh + b dSf v, and no gate gradient."""
    rng = np.random.default_rng(3)
    K = V = 8
    c = rand_case(rng, B=1, T=1, H=1, K=K, V=V, s0=False)
    scale = 0.7
    r = grads(c, scale=scale)
    q, k, v = c["q"][0, 0, 0], c["k"][0, 0, 0], c["v"][0, 0, 0]
    dO, dSf = c["dO"][0, 0, 0], c["dSf"][0, 0]
    rq, rk = 1 / np.sqrt(q @ q + oracle.EPS), 1 / np.sqrt(k @ k + oracle.EPS)
    qh, kh = q * rq, k * rk
    b = 1 / (1 + np.exp(-c["beta"][0, 0, 0]))
    kq, vd = kh @ qh, v @ dO
    dv = scale * b * kq * dO + b * dSf.T @ kh
    db = scale * kq * vd + kh @ dSf @ v
    dqh = scale * b * vd * kh
    dkh = scale * b * vd * qh + b * dSf @ v
    np.testing.assert_allclose(r["dv"][0, 0, 0], dv, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["dbeta"][0, 0, 0], db * b * (1 - b), rtol=1e-13)
    np.testing.assert_allclose(r["dq"][0, 0, 0], rq * (dqh - qh * (qh @ dqh)), rtol=1e-12,
                               atol=1e-14)
    np.testing.assert_allclose(r["dk"][0, 0, 0], rk * (dkh - kh * (kh @ dkh)), rtol=1e-12,
                               atol=1e-14)
    assert np.all(r["dg"] == 0) and np.all(r["dA_log"] == 0) and np.all(r["ddt_bias"] == 0)
    # dS0 = Diag(alpha) (dS_1 - kh dr^T), dS_1 = dSf + scale qh dO^T, dr = b dS_1^T kh
    alpha = np.exp(np.maximum(LB, -np.exp(c["A_log"][0]) * np.logaddexp(
        0, c["g"][0, 0, 0] + c["dt_bias"][0])))
    dS1 = dSf + scale * np.outer(qh, dO)
    dS0 = alpha[:, None] * (dS1 - np.outer(kh, b * (dS1.T @ kh)))
    np.testing.assert_allclose(r["dS0"][0, 0], dS0, rtol=1e-12, atol=1e-14)


def test_normalisation_gradients_are_orthogonal():
    """With eps = 0, q -> c q and k -> c k leave the result unchanged, so dq.q = dk.k = 0
    per token."""
    rng = np.random.default_rng(9)
    c = rand_case(rng, B=2, T=6, H=2, K=16, V=8)
    r = grads(c, eps=0.0)
    for x, dx in [(c["q"], r["dq"]), (c["k"], r["dk"])]:
        dots = (x * dx).sum(-1)
        assert np.abs(dots).max() <= 1e-12 * np.abs(dx).max() * np.abs(x).max() * 16


def test_no_write_when_beta_is_minus_infinity():
    rng = np.random.default_rng(4)
    c = rand_case(rng, B=1, T=5, H=2, K=6, V=5)
    c["beta"] = np.full_like(c["beta"], -np.inf)
    r = grads(c)
    assert np.all(r["dv"] == 0) and np.all(r["dk"] == 0) and np.all(r["dbeta"] == 0)


def test_no_gate_gradient_when_decay_is_one():
    rng = np.random.default_rng(6)
    c = rand_case(rng, B=1, T=5, H=2, K=6, V=5)
    c["A_log"] = np.full_like(c["A_log"], -np.inf)
    r = grads(c)
    assert np.all(r["dg"] == 0) and np.all(r["ddt_bias"] == 0) and np.all(r["dA_log"] == 0)


def test_chaining_through_the_state_gradient():
    rng = np.random.default_rng(8)
    K = V = 16
    T, T1 = 150, 67  # crosses checkpoint blocks of 64 in both halves
    c = rand_case(rng, B=1, T=T, H=2, K=K, V=V)
    full = grads(c)
    first = {k: (v[:, :T1] if k in ("q", "k", "v", "g", "beta", "dO") else v)
             for k, v in c.items()}
    second = {k: (v[:, T1:] if k in ("q", "k", "v", "g", "beta", "dO") else v)
              for k, v in c.items()}
    _, mid = oracle.forward_f64(first["q"], first["k"], first["v"], first["g"], first["beta"],
                                0.5, c["A_log"], c["dt_bias"], LB, c["S0"])
    second["S0"] = mid
    r2 = grads(second)
    first["dSf"] = r2["dS0"]
    r1 = grads(first)
    for key in ("dq", "dk", "dv", "dg", "dbeta"):
        np.testing.assert_array_equal(np.concatenate([r1[key], r2[key]], axis=1), full[key])
    np.testing.assert_array_equal(r1["dS0"], full["dS0"])
    np.testing.assert_allclose(r1["dA_log"] + r2["dA_log"], full["dA_log"], rtol=1e-12)
    np.testing.assert_allclose(r1["ddt_bias"] + r2["ddt_bias"], full["ddt_bias"], rtol=1e-12,
                               atol=1e-15)


@pytest.mark.parametrize("varlen", [False, True])
def test_forward_twin_equals_bf16_forward(varlen):
    """On bf16 values (promoted exactly) the raw-fp64 twin is the pinned forward."""
    wl = ki.Workload("twin", B=2, T=75, H=2, init_state="f32")
    inp = ki.make_inputs(wl, 1, lengths=[40, 0, 110] if varlen else None)
    out_b, fin_b = oracle.forward_inputs(inp)
    d = lambda t: t.to(torch.float64).numpy()
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    out_f, fin_f = oracle.forward_f64(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta),
                                      inp.scale, d(inp.A_log), d(inp.dt_bias), inp.lower_bound,
                                      d(inp.initial_state), cu)
    np.testing.assert_array_equal(out_f, out_b)
    np.testing.assert_array_equal(fin_f, fin_b)


def test_dlam_is_the_gate_gradient_before_the_activation():
    """dg = -dlam exp(A_log) sigmoid(x) where the clamp is open, 0 where it holds
    (dg itself is pinned by finite differences above)."""
    rng = np.random.default_rng(12)
    c = rand_case(rng, B=1, T=6, H=2, K=6, V=3, g_mu=1.0, g_std=3.0)
    r = oracle.backward(c["q"], c["k"], c["v"], c["g"], c["beta"], 0.5, c["A_log"], c["dt_bias"],
                        LB, c["dO"], c["S0"], c["dSf"], None, want_dlam=True)
    x = c["g"] + c["dt_bias"][None, None]
    ea = np.exp(c["A_log"])[None, None, :, None]
    z = -ea * np.logaddexp(0, x)
    want = np.where(z >= LB, -r["dlam"] * ea / (1 + np.exp(-x)), 0.0)
    np.testing.assert_allclose(r["dg"], want, rtol=1e-12, atol=1e-15)
    assert np.any(r["dlam"][z < LB] != 0)  # the kink cuts a nonzero gradient
