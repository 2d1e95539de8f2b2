"""Chunked (WY/UT) form of the KDA forward pass in NumPy fp64 -- test-side only.

This is NOT the oracle.  It restates, in plain NumPy, the chunk algorithm the CUDA
kernel runs, so that the derivation (intra-chunk decay-weighted products, the
unit-triangular solve, the inter-chunk state pass, the 32-token sub-blocks with
mid-block reference points that keep every decay factor inside the fp32 exponent
range) can be checked against the token-by-token oracle to ~1e-10, and so that
the rounding of each tensor-core operand can be emulated to size the precision
of every product before any kernel exists.

Per chunk of C tokens starting from state S0 (K x V), with q^, k^ normalised,
b = sigmoid(beta), lam = log-decay and G the inclusive in-chunk cumsum of lam:
  A_ij = sum_c k^_i k^_j exp(G_i - G_j)      (j < i)
  P_ij = sum_c q^_i k^_j exp(G_i - G_j)      (j <= i)
  T    = (I + Diag(b) A)^-1 Diag(b)
  w    = T (k^ * exp(G)),   u = T v
  U    = u - w S0
  O    = scale * [(q^ * exp(G)) S0 + P U]
  S    = Diag(exp(G_last)) S0 + (k^ * exp(G_last - G))^T U
"""
from __future__ import annotations

import numpy as np

LOG2E = 1.4426950408889634


def round_to(x: np.ndarray, kind: str | None) -> np.ndarray:
    """Round float64 values to the named operand format (None/"f64": untouched)."""
    if kind in (None, "f64"):
        return x
    x = np.asarray(x, dtype=np.float64)
    if kind == "f32":
        return x.astype(np.float32).astype(np.float64)
    f = x.astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    if kind == "bf16":  # round to nearest even on the upper 16 bits
        lsb = (u >> 16) & 1
        u = ((u + 0x7FFF + lsb) >> 16) << 16
        return (u.astype(np.uint32)).view(np.float32).astype(np.float64)
    if kind == "tf32":  # round half away from zero to 10 stored mantissa bits
        u = ((u + 0x1000) >> 13) << 13
        return (u.astype(np.uint32)).view(np.float32).astype(np.float64)
    if kind == "f16":
        return x.astype(np.float16).astype(np.float64)
    raise ValueError(kind)


def activations(q, k, g, beta, A_log_h, dt_bias_h, lb, eps=1e-6):
    """Per-token activations of one head: q^, k^, b, lam (fp64)."""
    qh = q / np.sqrt((q * q).sum(-1, keepdims=True) + eps)
    kh = k / np.sqrt((k * k).sum(-1, keepdims=True) + eps)
    b = 1.0 / (1.0 + np.exp(-beta))
    x = g + dt_bias_h[None, :]
    sp = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))
    lam = np.maximum(lb, -np.exp(A_log_h) * sp)
    return qh, kh, b, lam


def pow2_scale(x: np.ndarray, axis: int) -> np.ndarray:
    """Power-of-two scale per slice so that max |x / s| lies in [1, 2) (1 if all zero)."""
    m = np.abs(x).max(axis=axis, keepdims=True)
    e = np.where(m > 0, np.floor(np.log2(np.where(m > 0, m, 1.0))), 0.0)
    return np.exp2(e)


def chunk_forward(qh, kh, v, b, lam, scale, S0=None, C=64, sub=32, prec=None):
    """Chunked KDA for ONE (sequence, head) on activations; returns (out, S_final).

    ``prec`` maps operand names to rounding kinds (emulating the tensor-core inputs):
      "Akk" (both factors of A), "Pqk" (both factors of P), "T" (T in w and u),
      "kg" (k^*exp(G)), "qg" (q^*exp(G)), "w", "S" (state operand), "U",
      "kp" (k^*exp(G_last - G)), "P" (P in P U), "v".
    Operands "S" and "U" are scaled by a power of two per value column before
    rounding (as the kernel does for fp16 operands), and unscaled after.
    """
    prec = prec or {}
    R = lambda name, x: round_to(x, prec.get(name))
    T_, K = qh.shape
    V = v.shape[1]
    S = np.zeros((K, V)) if S0 is None else np.array(S0, dtype=np.float64)
    out = np.zeros((T_, V))
    for c0 in range(0, T_, C):
        L = min(C, T_ - c0)
        sl = slice(c0, c0 + L)
        q_, k_, v_, b_, lam_ = qh[sl], kh[sl], v[sl], b[sl], lam[sl]
        G = np.cumsum(lam_, axis=0)  # inclusive
        # decay-weighted Gram matrices in sub-blocks with a mid-block reference
        A = np.zeros((L, L))
        P = np.zeros((L, L))
        for I0 in range(0, L, sub):
            I1 = min(L, I0 + sub)
            r = min(I1 - 1, I0 + sub // 2 - 1)  # reference token of block I
            rho = np.exp(G[I0:I1] - G[r])       # <= e^{80} for 32-token blocks, lb >= -5
            for J0 in range(0, I1, sub):
                J1 = min(L, J0 + sub)
                sig = np.exp(G[r] - G[J0:J1])   # exact for J = I; <= 1 for J < I
                kr = R("Akk", k_[I0:I1] * rho)
                qr = R("Pqk", q_[I0:I1] * rho)
                kc_a = R("Akk", k_[J0:J1] * sig)
                kc_p = R("Pqk", k_[J0:J1] * sig)
                A[I0:I1, J0:J1] = kr @ kc_a.T
                P[I0:I1, J0:J1] = qr @ kc_p.T
        A = np.tril(A, -1)
        P = np.tril(P, 0)
        Tm = np.linalg.solve(np.eye(L) + b_[:, None] * A, np.diag(b_))
        Gam = np.exp(G)
        w = R("T", Tm) @ R("kg", k_ * Gam)
        u = R("T", Tm) @ R("v", v_)
        sS = pow2_scale(S, 0)  # per value column
        Sop = R("S", S / sS) * sS
        U = u - R("w", w) @ Sop
        sU = pow2_scale(U, 0)
        Uop = R("U", U / sU) * sU
        out[sl] = scale * (R("qg", q_ * Gam) @ Sop + R("P", P) @ Uop)
        gl = G[L - 1]
        S = np.exp(gl)[:, None] * S + R("kp", k_ * np.exp(gl[None, :] - G)).T @ Uop
    return out, S


def chunk_forward_inputs(inp, prec=None, C=64, sub=32, pairs=None, eps=1e-6):
    """Run ``chunk_forward`` over a ``kda_inputs.KDAInputs``; returns (out, final) fp64.

    ``pairs`` restricts to a list of (sequence, head) indices (others stay zero)."""
    q = inp.q.double().numpy()
    k = inp.k.double().numpy()
    v = inp.v.double().numpy()
    g = inp.g.double().numpy()
    beta = inp.beta.double().numpy()
    A_log = inp.A_log.double().numpy()
    dt = inp.dt_bias.double().numpy()
    init = None if inp.initial_state is None else inp.initial_state.double().numpy()
    B, Tt, H, K = q.shape
    V = v.shape[3]
    seqs = inp.seq_bounds()
    out = np.zeros((B, Tt, H, V))
    fin = np.zeros((len(seqs), H, K, V))
    todo = pairs if pairs is not None else [(s, h) for s in range(len(seqs)) for h in range(H)]
    for s, h in todo:
        bi, t0, n = seqs[s]
        sl = slice(t0, t0 + n)
        qh, kh, bb, lam = activations(q[bi, sl, h], k[bi, sl, h], g[bi, sl, h], beta[bi, sl, h],
                                      A_log[h], dt[h], inp.lower_bound, eps)
        S0 = None if init is None else init[s, h]
        o, Sf = chunk_forward(qh, kh, v[bi, sl, h], bb, lam, inp.scale, S0, C, sub, prec)
        out[bi, sl, h] = o
        fin[s, h] = Sf
    return out, fin
