"""CPU fp64 oracle of the KDA forward and backward passes -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never calls it and shares no code with it.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, token by token); this
file only builds it with gcc and marshals arguments through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

STATE_NONE, STATE_F32, STATE_BF16, STATE_F64 = 0, 1, 2, 3
EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` (gcc, -O2, OpenMP, IEEE math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, D, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int
            lib.kda_oracle_fwd.argtypes = [P, P, P, P, P, D, P, P, D, P, I, P, P, I64, P,
                                           I64, I64, I64, I64, I64, D, P]
            lib.kda_oracle_fwd.restype = I
            lib.kda_oracle_core.argtypes = [I64, I64, I64, P, P, P, P, P, D, P, P, P]
            lib.kda_oracle_core.restype = I
            lib.kda_oracle_fwd_f64.argtypes = [P, P, P, P, P, D, P, P, D, P, P, P, I64, P,
                                               I64, I64, I64, I64, I64, D]
            lib.kda_oracle_fwd_f64.restype = I
            lib.kda_oracle_bwd_f64.argtypes = [P, P, P, P, P, D, P, P, D, P, P, P, P, I64,
                                               P, P, P, P, P, P, P, P, P,
                                               I64, I64, I64, I64, I64, D]
            lib.kda_oracle_bwd_f64.restype = I
            lib.kda_oracle_threads.argtypes = []
            lib.kda_oracle_threads.restype = I
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().kda_oracle_threads())


def core(qh, kh, v, b, lam, scale, S0=None):
    """Recurrence on post-activation values for one (sequence, head).

    qh, kh, lam: [T,K]; v: [T,V]; b: [T]; S0: [K,V] or None.  Returns (out [T,V],
    S_final [K,V]) in fp64.
    """
    qh = np.ascontiguousarray(qh, dtype=np.float64)
    kh = np.ascontiguousarray(kh, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    lam = np.ascontiguousarray(lam, dtype=np.float64)
    T, K = qh.shape
    V = v.shape[1]
    S0c = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    out = np.zeros((T, V), np.float64)
    Sf = np.zeros((K, V), np.float64)
    rc = _load().kda_oracle_core(T, K, V, _ptr(qh), _ptr(kh), _ptr(v), _ptr(b), _ptr(lam),
                                 float(scale), _ptr(S0c), _ptr(out), _ptr(Sf))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_core failed: {rc}")
    return out, Sf


def forward(q_bits, k_bits, v_bits, g_bits, beta_bits, scale, A_log, dt_bias, lower_bound,
            initial_state=None, init_dtype=STATE_NONE, cu_seqlens=None, eps=EPS,
            want_out=True, want_final=True, mask=None):
    """Full forward pass on raw inputs.

    q_bits..beta_bits: uint16 bf16 bit patterns with shapes [B,T,H,K] / [B,T,H,V] /
    [B,T,H]; A_log fp32 [H]; dt_bias fp32 [H,K]; initial_state: fp32 array,
    uint16 bf16 bits or fp64 array [N,H,K,V] (init_dtype says which); cu_seqlens int64 [N+1].
    ``mask`` (uint8 [N*H]) restricts the computed (sequence, head) pairs.
    Returns (out fp64 [B,T,H,V] or None, final fp64 [N,H,K,V] or None).
    """
    B, T, H, K = q_bits.shape
    V = v_bits.shape[3]
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q_bits, k_bits, v_bits, g_bits,
                                                               beta_bits)]
    A_log = np.ascontiguousarray(A_log, dtype=np.float32)
    dt_bias = np.ascontiguousarray(dt_bias, dtype=np.float32)
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = B if cu is None else cu.size - 1
    if initial_state is not None:
        want = {STATE_F32: np.float32, STATE_BF16: np.uint16, STATE_F64: np.float64}[init_dtype]
        initial_state = np.ascontiguousarray(initial_state, dtype=want)
    else:
        init_dtype = STATE_NONE
    out = np.zeros((B, T, H, V), np.float64) if want_out else None
    fin = np.zeros((N, H, K, V), np.float64) if want_final else None
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    rc = _load().kda_oracle_fwd(*[_ptr(a) for a in arrs], float(scale), _ptr(A_log),
                                _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                                int(init_dtype), _ptr(fin), _ptr(cu), int(N if cu is not None else 0),
                                _ptr(out), B, T, H, K, V, float(eps), _ptr(m))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_fwd failed: {rc}")
    return out, fin


def forward_inputs(inp, eps=EPS, want_out=True, want_final=True, mask=None):
    """``forward`` on a ``kda_inputs.KDAInputs`` (CPU tensors)."""
    import torch  # local: only for dtype checks / views

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    init, idt = None, STATE_NONE
    if inp.initial_state is not None:
        if inp.initial_state.dtype == torch.float32:
            init, idt = inp.initial_state.numpy(), STATE_F32
        else:
            init, idt = bits(inp.initial_state), STATE_BF16
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return forward(bits(inp.q), bits(inp.k), bits(inp.v), bits(inp.g), bits(inp.beta), inp.scale,
                   inp.A_log.numpy(), inp.dt_bias.numpy(), inp.lower_bound, init, idt, cu, eps,
                   want_out, want_final, mask)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def forward_f64(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, S0=None, cu_seqlens=None,
                eps=EPS):
    """Forward pass on raw fp64 inputs (the twin of ``forward`` that finite differences
    can be taken of).  Shapes as in ``forward``; S0 fp64 [N,H,K,V] or None.
    Returns (out [B,T,H,V], final [N,H,K,V]), fp64."""
    q, k, v, g, beta, A_log, dt_bias, S0 = map(_f64, (q, k, v, g, beta, A_log, dt_bias, S0))
    B, T, H, K = q.shape
    V = v.shape[3]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = B if cu is None else cu.size - 1
    out = np.zeros((B, T, H, V), np.float64)
    fin = np.zeros((N, H, K, V), np.float64)
    rc = _load().kda_oracle_fwd_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                    _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(S0),
                                    _ptr(fin), _ptr(cu), int(N if cu is not None else 0),
                                    _ptr(out), B, T, H, K, V, float(eps))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_fwd_f64 failed: {rc}")
    return out, fin


def backward(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, dO, S0=None, dS_final=None,
             cu_seqlens=None, eps=EPS, want_dlam=False):
    """Gradients of L = <dO, out> + <dS_final, final> (fp64, token by token in reverse).

    Inputs are raw fp64 values with the shapes of ``forward``; dO [B,T,H,V];
    dS_final [N,H,K,V] or None (zero).  Returns a dict with dq, dk, dg [B,T,H,K],
    dv [B,T,H,V], dbeta [B,T,H], dA_log [H], ddt_bias [H,K], dS0 [N,H,K,V], and with
    ``want_dlam`` dlam [B,T,H,K] = dL/dlam (the gate's log-decay).
    Tokens outside every sequence get zeros."""
    q, k, v, g, beta, A_log, dt_bias, S0, dO, dSf = map(
        _f64, (q, k, v, g, beta, A_log, dt_bias, S0, dO, dS_final))
    B, T, H, K = q.shape
    V = v.shape[3]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = B if cu is None else cu.size - 1
    r = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), dg=np.zeros_like(g),
             dbeta=np.zeros_like(beta), dA_log=np.zeros(H), ddt_bias=np.zeros((H, K)),
             dS0=np.zeros((N, H, K, V)), dlam=np.zeros_like(g) if want_dlam else None)
    rc = _load().kda_oracle_bwd_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(A_log), _ptr(dt_bias),
        float(lower_bound), _ptr(S0), _ptr(dO), _ptr(dSf), _ptr(cu),
        int(N if cu is not None else 0), _ptr(r["dq"]), _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dg"]),
        _ptr(r["dbeta"]), _ptr(r["dA_log"]), _ptr(r["ddt_bias"]), _ptr(r["dS0"]),
        _ptr(r["dlam"]), B, T, H, K, V, float(eps))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_bwd_f64 failed: {rc}")
    return r


def backward_inputs(inp, dO, dS_final=None, eps=EPS, want_dlam=False):
    """``backward`` on a ``kda_inputs.KDAInputs`` (CPU tensors; bf16 values and a bf16
    or fp32 initial state promoted exactly to fp64); dO and dS_final are CPU tensors
    (any float dtype, promoted exactly)."""
    import torch

    d = lambda t: None if t is None else t.detach().to(torch.float64).numpy()
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return backward(d(inp.q), d(inp.k), d(inp.v), d(inp.g), d(inp.beta), inp.scale,
                    d(inp.A_log), d(inp.dt_bias), inp.lower_bound, d(dO), d(inp.initial_state),
                    d(dS_final), cu, eps, want_dlam)
