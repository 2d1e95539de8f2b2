"""Chunked form of the KDA backward pass in NumPy fp64 -- test-side only.

This is NOT the oracle (the oracle differentiates the token recurrence directly).  It
restates the backward in the per-chunk matrix form a tensor-core kernel would run, so
that the algebra can be checked against the oracle's gradients before any kernel of
that shape exists.

Forward of one chunk of L tokens from state S0 (K x V), on activations q^, k^, b,
lam, with G the inclusive cumulative sum of lam and Gam = exp(G), GL = G[L-1]
(the chunked form of the recurrence of the FlashKDA pages, 7minutos.es "¿Qué es la
atención Kimi Delta...?"):
  A_ij = sum_c k^_i k^_j exp(G_i - G_j)   (j < i),   P_ij = same with q^_i (j <= i)
  M = I + Diag(b) A,  T = M^-1 Diag(b)
  Y = v - (k^ Gam) S0,  U = T Y
  O = scale [(q^ Gam) S0 + P U]
  S_end = Diag(exp GL) S0 + (k^ exp(GL - G))^T U
Reverse of the chunk, given dO and dS_end (written as dS):
  dU = scale P^T dO + K' dS          (K' = k^ exp(GL - G))
  dY = T^T dU;  dv = dY;  dT = dU Y^T
  dS0 = scale (q^ Gam)^T dO + Diag(exp GL) dS - (k^ Gam)^T dY
  d(k^ Gam) = -dY S0^T;  d(q^ Gam) = scale dO S0^T;  dP = scale dO U^T (j <= i)
  dK' = U dS^T;  d(exp GL) = rowsum(dS o S0)
  dMinv = dT Diag(b);  db_j += sum_i dT_ij Minv_ij
  dM = -Minv^T dMinv Minv^T;  dA = Diag(b) dM (j < i);  db_i += sum_j dM_ij A_ij
then through the decay-weighted products into dq^, dk^ and dG, and dlam is the
reverse cumulative sum of dG.  The chunks are visited in reverse, dS passing from
each chunk's dS0 to the chunk before it.
"""
from __future__ import annotations

import numpy as np


def _gram(x, k, G, strict):
    """M_ij = sum_c x_i k_j exp(G_i - G_j) on the lower triangle; also E_ijc."""
    E = np.exp(G[:, None, :] - G[None, :, :])  # [L, L, K]; only the lower part is used
    L = G.shape[0]
    mask = np.tril(np.ones((L, L)), -1 if strict else 0)
    E = E * mask[:, :, None]
    return np.einsum("ic,jc,ijc->ij", x, k, E), E


def chunk_backward(qh, kh, v, b, lam, scale, dO, S0=None, dSf=None, C=64):
    """Gradients w.r.t. the activations of ONE (sequence, head).

    Returns (dqh, dkh, dv, db, dlam, dS0) in fp64 for L = <dO, out> + <dSf, S_final>.
    """
    T_, K = qh.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    starts = []
    for c0 in range(0, T_, C):  # forward: the state before every chunk
        starts.append(S.copy())
        L = min(C, T_ - c0)
        sl = slice(c0, c0 + L)
        G = np.cumsum(lam[sl], axis=0)
        A, _ = _gram(kh[sl], kh[sl], G, True)
        Tm = np.linalg.solve(np.eye(L) + b[sl, None] * A, np.diag(b[sl]))
        U = Tm @ (v[sl] - (kh[sl] * np.exp(G)) @ S)
        S = np.exp(G[L - 1])[:, None] * S + (kh[sl] * np.exp(G[L - 1][None] - G)).T @ U
    dqh, dkh = np.zeros_like(qh), np.zeros_like(kh)
    dv, db, dlam = np.zeros_like(v), np.zeros_like(b), np.zeros_like(lam)
    dS = np.zeros((K, V)) if dSf is None else np.array(dSf, dtype=np.float64)
    for n in reversed(range(len(starts))):
        c0 = n * C
        L = min(C, T_ - c0)
        sl = slice(c0, c0 + L)
        q_, k_, v_, b_, S0n, dO_ = qh[sl], kh[sl], v[sl], b[sl], starts[n], dO[sl]
        G = np.cumsum(lam[sl], axis=0)
        Gam, GL = np.exp(G), G[L - 1]
        A, EA = _gram(k_, k_, G, True)
        P, EP = _gram(q_, k_, G, False)
        Minv = np.linalg.inv(np.eye(L) + b_[:, None] * A)
        Tm = Minv * b_[None, :]
        KG, QG = k_ * Gam, q_ * Gam
        Kp = k_ * np.exp(GL[None] - G)
        Y = v_ - KG @ S0n
        U = Tm @ Y
        # reverse of the chunk
        dU = scale * P.T @ dO_ + Kp @ dS
        dY = Tm.T @ dU
        dT = np.tril(dU @ Y.T)
        dS0 = scale * QG.T @ dO_ + np.exp(GL)[:, None] * dS - KG.T @ dY
        dKG = -dY @ S0n.T
        dQG = scale * dO_ @ S0n.T
        dP = np.tril(scale * dO_ @ U.T)
        dKp = U @ dS.T
        dGL = (dS * S0n).sum(1) * np.exp(GL)
        dv[sl] = dY
        dMinv = dT * b_[None, :]
        db_ = (dT * Minv).sum(0)
        dM = -Minv.T @ dMinv @ Minv.T
        dA = np.tril(b_[:, None] * dM, -1)
        db_ += (np.tril(dM, -1) * A).sum(1)
        # decay-weighted products -> dq^, dk^, dG
        dG = np.zeros_like(G)
        tA_i = np.einsum("ij,jc,ijc->ic", dA, k_, EA)   # sum_j dA_ij k_j E_ij
        tA_j = np.einsum("ij,ic,ijc->jc", dA, k_, EA)   # sum_i dA_ij k_i E_ij
        tP_i = np.einsum("ij,jc,ijc->ic", dP, k_, EP)
        tP_j = np.einsum("ij,ic,ijc->jc", dP, q_, EP)
        dk_ = tA_i + tA_j + tP_j + dKG * Gam + dKp * np.exp(GL[None] - G)
        dq_ = tP_i + dQG * Gam
        dG += k_ * tA_i - k_ * tA_j + q_ * tP_i - k_ * tP_j
        dG += dKG * KG + dQG * QG
        dG -= dKp * Kp
        dG[L - 1] += (dKp * Kp).sum(0) + dGL
        dqh[sl], dkh[sl], db[sl] = dq_, dk_, db_
        dlam[sl] = np.cumsum(dG[::-1], axis=0)[::-1]  # dlam_s = sum_{i >= s} dG_i
        dS = dS0
    return dqh, dkh, dv, db, dlam, dS


def backward_inputs(inp, dO, dSf=None, C=64, eps=1e-6, prec=None, tiled=False):
    """``chunk_backward`` (or, with ``tiled`` or ``prec``, ``chunk_backward_tiled``) over a
    ``kda_inputs.KDAInputs``, chained through the norms, the sigmoid and the gate to
    the raw inputs; returns the dict of ``oracle.backward`` (plus dlam)."""
    q, k, v, g = (t.double().numpy() for t in (inp.q, inp.k, inp.v, inp.g))
    beta = inp.beta.double().numpy()
    A_log, dt = inp.A_log.double().numpy(), inp.dt_bias.double().numpy()
    init = None if inp.initial_state is None else inp.initial_state.double().numpy()
    dOn = dO.double().numpy()
    dSn = None if dSf is None else dSf.double().numpy()
    B, Tt, H, K = q.shape
    seqs = inp.seq_bounds()
    r = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dg=np.zeros_like(g),
             dbeta=np.zeros_like(beta), dA_log=np.zeros(H), ddt_bias=np.zeros((H, K)),
             dS0=np.zeros((len(seqs), H, K, v.shape[3])), dlam=np.zeros_like(g))
    for s, (bi, t0, n) in enumerate(seqs):
        sl = slice(t0, t0 + n)
        for h in range(H):
            qq, kk, gg = q[bi, sl, h], k[bi, sl, h], g[bi, sl, h]
            rq = 1 / np.sqrt((qq * qq).sum(-1, keepdims=True) + eps)
            rk = 1 / np.sqrt((kk * kk).sum(-1, keepdims=True) + eps)
            qh, kh = qq * rq, kk * rk
            bb = 1 / (1 + np.exp(-beta[bi, sl, h]))
            x = gg + dt[h][None]
            z = -np.exp(A_log[h]) * (np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x))))
            lam = np.maximum(inp.lower_bound, z)
            args = (qh, kh, v[bi, sl, h], bb, lam, inp.scale, dOn[bi, sl, h],
                    None if init is None else init[s, h], None if dSn is None else dSn[s, h], C)
            if tiled or prec:
                dqh, dkh, dvv, dbb, dlam, dS0 = chunk_backward_tiled(*args, prec=prec)
            else:
                dqh, dkh, dvv, dbb, dlam, dS0 = chunk_backward(*args)
            r["dq"][bi, sl, h] = rq * (dqh - qh * (qh * dqh).sum(-1, keepdims=True))
            r["dk"][bi, sl, h] = rk * (dkh - kh * (kh * dkh).sum(-1, keepdims=True))
            r["dv"][bi, sl, h] = dvv
            r["dbeta"][bi, sl, h] = dbb * bb * (1 - bb)
            openm = z >= inp.lower_bound
            dx = np.where(openm, -dlam * np.exp(A_log[h]) / (1 + np.exp(-x)), 0.0)
            r["dg"][bi, sl, h] = dx
            r["dlam"][bi, sl, h] = dlam
            r["ddt_bias"][h] += dx.sum(0)
            r["dA_log"][h] += np.where(openm, dlam * z, 0.0).sum()
            r["dS0"][s, h] = dS0
    return r


# ---------------------------------------------------------------------------------
# Tiled form with operand rounding (for sizing a tensor-core precision plan).
#
# The decay-weighted products and their adjoints run in 32-token sub-blocks with a
# mid-block reference token r (so every factor exp(+-(G - G_r)) stays inside the fp32
# range, as in the forward): for row block I and column block J <= I,
#   exp(G_i - G_j) = rho_i sigma_j,  rho = exp(G_I - G_r),  sigma = exp(G_r - G_J).
# Every other product has fp16 operands with a power-of-two scale per row or column,
# chosen along the dimension that is NOT contracted, so the scale factors out.
# ``prec`` maps operand groups to rounding kinds (see ``round_to``); missing = exact.
# ---------------------------------------------------------------------------------

def _scaled(x, kind, axis):
    """Round x to ``kind`` after dividing by a power of two per slice along ``axis``
    (axis=0: per column, axis=1: per row); None/"f64" leaves x exact."""
    if kind in (None, "f64"):
        return x
    from chunked_ref import pow2_scale, round_to
    s = pow2_scale(x, axis)
    return round_to(x / s, kind) * s


def _blocks(L, sub):
    out = []
    for I0 in range(0, L, sub):
        I1 = min(L, I0 + sub)
        out.append((I0, I1, min(I1 - 1, I0 + sub // 2 - 1)))
    return out


def chunk_backward_tiled(qh, kh, v, b, lam, scale, dO, S0=None, dSf=None, C=64, sub=32,
                         prec=None):
    """``chunk_backward`` with the decay-weighted products in sub-blocks and the
    tensor-core operands rounded per ``prec``.  Operand groups:
      "APf"  factors of the decay-weighted products A and P,
      "APb"  operands of their adjoints (dA, dP and the k^ / q^ factors); "tf32x3"
             emulates the three-product split of each operand into tf32 halves,
      "Minv" the solve result, "dM" the solve adjoint products,
      "T"    T as a product operand, "F"  the other fp16 operands (k^Gam, q^Gam, K',
      P, S0, dS, dO, U, Y, dU, dY with per-slice scales).
    """
    from chunked_ref import round_to
    prec = prec or {}
    R = lambda g, x: round_to(x, prec.get(g))
    F = lambda x, axis: _scaled(x, prec.get("F"), axis)
    T_, K = qh.shape
    V = v.shape[1]

    def gram(x, k, G, strict):
        L = G.shape[0]
        M = np.zeros((L, L))
        for I0, I1, r in _blocks(L, sub):
            rho = np.exp(G[I0:I1] - G[r])
            for J0, J1, _ in _blocks(L, sub):
                if J0 >= I1:
                    continue
                sig = np.exp(G[r] - G[J0:J1])
                M[I0:I1, J0:J1] = R("APf", x[I0:I1] * rho) @ R("APf", k[J0:J1] * sig).T
        return np.tril(M, -1 if strict else 0)

    def mm(a, b_):
        """Product of the adjoint operands: rounded per "APb", or with "tf32x3" the
        three-term split a_hi b_hi + a_hi b_lo + a_lo b_hi of tf32 halves."""
        if prec.get("APb") == "tf32x3":
            ah, bh = round_to(a, "tf32"), round_to(b_, "tf32")
            al, bl = round_to(a - ah, "tf32"), round_to(b_ - bh, "tf32")
            return ah @ bh + ah @ bl + al @ bh
        return R("APb", a) @ R("APb", b_)

    def gram_adjoint(dM, x, k, G):
        """(sum_j dM_ij k_j e^{G_i-G_j}, sum_i dM_ij x_i e^{G_i-G_j}) per channel."""
        L = G.shape[0]
        ti, tj = np.zeros_like(x), np.zeros_like(k)
        for I0, I1, r in _blocks(L, sub):
            rho = np.exp(G[I0:I1] - G[r])
            for J0, J1, _ in _blocks(L, sub):
                if J0 >= I1:
                    continue
                sig = np.exp(G[r] - G[J0:J1])
                blk, ks, xr = dM[I0:I1, J0:J1], k[J0:J1] * sig, x[I0:I1] * rho
                ti[I0:I1] += rho * mm(blk, ks)
                tj[J0:J1] += sig * mm(blk.T, xr)
        return ti, tj

    def solve(A, b_):
        L = A.shape[0]
        Minv = R("Minv", np.linalg.inv(np.eye(L) + b_[:, None] * A))
        return Minv

    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    starts, Us = [], []
    for c0 in range(0, T_, C):
        starts.append(S.copy())
        L = min(C, T_ - c0)
        sl = slice(c0, c0 + L)
        G = np.cumsum(lam[sl], axis=0)
        Minv = solve(gram(kh[sl], kh[sl], G, True), b[sl])
        Tm = Minv * b[sl][None, :]
        Y = v[sl] - F(kh[sl] * np.exp(G), 0) @ F(S, 0)
        U = Tm @ Y
        S = np.exp(G[L - 1])[:, None] * S + F(kh[sl] * np.exp(G[L - 1][None] - G), 0).T @ F(U, 0)
    dqh, dkh = np.zeros_like(qh), np.zeros_like(kh)
    dv, db, dlam = np.zeros_like(v), np.zeros_like(b), np.zeros_like(lam)
    dS = np.zeros((K, V)) if dSf is None else np.array(dSf, dtype=np.float64)
    for n in reversed(range(len(starts))):
        c0 = n * C
        L = min(C, T_ - c0)
        sl = slice(c0, c0 + L)
        q_, k_, v_, b_, S0n, dO_ = qh[sl], kh[sl], v[sl], b[sl], starts[n], dO[sl]
        G = np.cumsum(lam[sl], axis=0)
        Gam, GL = np.exp(G), G[L - 1]
        A = gram(k_, k_, G, True)
        P = gram(q_, k_, G, False)
        Minv = solve(A, b_)
        Tm = Minv * b_[None, :]
        KG, QG = k_ * Gam, q_ * Gam
        Kp = k_ * np.exp(GL[None] - G)
        Y = v_ - F(KG, 0) @ F(S0n, 0)
        U = Tm @ Y
        # products over tokens (scale per value column) and over k (scale per column)
        dU = scale * F(P, 0).T @ F(dO_, 0) + F(Kp, 0) @ F(dS, 0)
        Tq = R("T", Tm)
        dY = Tq.T @ F(dU, 0)
        dS0 = (scale * F(QG, 0).T @ F(dO_, 0) + np.exp(GL)[:, None] * dS
               - F(KG, 0).T @ F(dY, 0))
        # products over v (scale per row)
        dKG = -F(dY, 1) @ F(S0n, 1).T
        dQG = scale * F(dO_, 1) @ F(S0n, 1).T
        dKp = F(U, 1) @ F(dS, 1).T
        dP = np.tril(scale * F(dO_, 1) @ F(U, 1).T)
        dT = np.tril(F(dU, 1) @ F(Y, 1).T)
        dGL = (dS * S0n).sum(1) * np.exp(GL)
        dv[sl] = dY
        dMinv = dT * b_[None, :]
        db_ = (dT * Minv).sum(0)
        Mq = R("dM", Minv)
        dM = -Mq.T @ R("dM", R("dM", dMinv) @ Mq.T)
        dA = np.tril(b_[:, None] * dM, -1)
        db_ += (np.tril(dM, -1) * A).sum(1)
        tA_i, tA_j = gram_adjoint(dA, k_, k_, G)
        tP_i, tP_j = gram_adjoint(dP, q_, k_, G)
        dk_ = tA_i + tA_j + tP_j + dKG * Gam + dKp * np.exp(GL[None] - G)
        dq_ = tP_i + dQG * Gam
        dG = k_ * tA_i - k_ * tA_j + q_ * tP_i - k_ * tP_j + dKG * KG + dQG * QG - dKp * Kp
        dG[L - 1] += (dKp * Kp).sum(0) + dGL
        dqh[sl], dkh[sl], db[sl] = dq_, dk_, db_
        dlam[sl] = np.cumsum(dG[::-1], axis=0)[::-1]
        dS = dS0
    return dqh, dkh, dv, db, dlam, dS
