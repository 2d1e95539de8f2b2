"""Python binding of libkda.so, the B200 (sm_100a) Kimi Delta Attention forward and backward passes.

Argument marshalling only: every step of the pass runs in the CUDA kernels of
``libkda.so``.  PyTorch provides device memory and streams.  There is no CPU or
PyTorch fallback: if the library cannot be loaded, the calls raise.

The functions mirror the C ABI in ``include/kda.h``:
  kda_fwd, kda_fwd_ex, kda_decode, kda_bwd, kda_bwd_workspace_size, kda_fwd_host,
  kda_fwd_host_workspace_size, kda_set_checks, kda_strerror, kda_last_launch_count,
  kda_device_status.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

KDA_STATE_NONE, KDA_STATE_F32, KDA_STATE_BF16 = 0, 1, 2
KDA_LAYOUT_KV, KDA_LAYOUT_VK = 0, 1
_LAYOUTS = {"kv": KDA_LAYOUT_KV, "vk": KDA_LAYOUT_VK}
HEAD = 128

_lib = None
_lock = threading.Lock()


class KDAError(RuntimeError):
    """A libkda call returned a negative code."""

    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {kda_strerror(code)} (code {code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libkda.so (built in-tree by ``linear_attention_09_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: run `python -m linear_attention_09_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I64, F, I, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int,
                                ctypes.c_size_t)
            L.kda_fwd.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, I64, P, I64, I64, I64,
                                  I64, I64, P]
            L.kda_fwd.restype = I
            L.kda_fwd_ex.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, I, I, P, I64, P, I64,
                                     I64, I64, I64, I64, P]
            L.kda_fwd_ex.restype = I
            L.kda_decode.argtypes = [P, P, P, P, P, F, P, P, F, P, P, P, I64, I64, I64, I64, P]
            L.kda_decode.restype = I
            L.kda_fwd_host.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, I64, P, I64, I64,
                                       I64, I64, I64, P, SZ, P]
            L.kda_fwd_host.restype = I
            L.kda_fwd_host_workspace_size.argtypes = [I64, I64, I64, I64, I64, I64, I, I]
            L.kda_fwd_host_workspace_size.restype = SZ
            L.kda_bwd.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, P, I64, P, P, P, P, P,
                                  P, P, P, P, SZ, I64, I64, I64, I64, I64, P]
            L.kda_bwd.restype = I
            L.kda_bwd_workspace_size.argtypes = [I64, I64, I64, I64, I64, I64]
            L.kda_bwd_workspace_size.restype = SZ
            L.kda_set_checks.argtypes = [I]
            L.kda_set_checks.restype = I
            L.kda_strerror.argtypes = [I]
            L.kda_strerror.restype = ctypes.c_char_p
            L.kda_last_launch_count.argtypes = []
            L.kda_last_launch_count.restype = I
            L.kda_device_status.argtypes = [I]
            L.kda_device_status.restype = I
            _lib = L
    return _lib


def kda_strerror(code: int) -> str:
    return lib().kda_strerror(int(code)).decode()


def kda_set_checks(level: int) -> int:
    """Debug checks of device arguments (1: cu_seqlens checked on the device before each
    varlen call, synchronously); returns the previous level."""
    return int(lib().kda_set_checks(int(level)))


def kda_last_launch_count() -> int:
    return int(lib().kda_last_launch_count())


def kda_device_status(reset: bool = False) -> int:
    """Error word of the last kernels (0 = every bounded wait completed)."""
    return int(lib().kda_device_status(int(bool(reset))))


def kda_fwd_host_workspace_size(B, T, H, K=HEAD, V=HEAD, num_seqs=0,
                                initial_state_dtype=KDA_STATE_NONE, want_final_state=True) -> int:
    return int(lib().kda_fwd_host_workspace_size(B, T, H, K, V, num_seqs, initial_state_dtype,
                                                 int(bool(want_final_state))))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _state_dtype(t: Optional[torch.Tensor]) -> int:
    if t is None:
        return KDA_STATE_NONE
    if t.dtype == torch.float32:
        return KDA_STATE_F32
    if t.dtype == torch.bfloat16:
        return KDA_STATE_BF16
    return -1  # rejected by the library


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def kda_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
            final_state=None, cu_seqlens=None, out=None, output_final_state=True, stream=None):
    """Run the KDA forward pass on CUDA tensors; returns (out, final_state or None).

    q, k, g: bf16 [B,T,H,128]; v: bf16 [B,T,H,128]; beta: bf16 [B,T,H];
    A_log: fp32 [H]; dt_bias: fp32 [H,128]; initial_state: fp32/bf16 [N,H,128,128]
    or None; cu_seqlens: int64 [N+1] or None.  ``out`` / ``final_state`` may be
    given (then they are written), else they are allocated on q's device.  The
    call is asynchronous on ``stream`` (default: the current stream).
    """
    B, T, H, K = q.shape
    V = v.shape[3]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    if out is None:
        out = torch.empty((B, T, H, V), dtype=torch.bfloat16, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, K, V), dtype=torch.float32, device=q.device)
    rc = lib().kda_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(A_log),
                       _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                       _state_dtype(initial_state), _ptr(final_state), _ptr(cu_seqlens), num_seqs,
                       _ptr(out), B, T, H, K, V, _stream_handle(stream, q.device))
    if rc != 0:
        raise KDAError(rc, "kda_fwd")
    return out, final_state


def kda_fwd_ex(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
               final_state=None, cu_seqlens=None, out=None, output_final_state=True,
               state_layout="kv", final_state_dtype=torch.float32, stream=None):
    """``kda_fwd`` with the state variants: ``state_layout`` "kv" (S[k][v]) or "vk"
    (S[v][k], the transposed layout) for both states, and a bf16 or fp32 final state
    (``final_state_dtype``, or the dtype of a given ``final_state``)."""
    B, T, H, K = q.shape
    V = v.shape[3]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    layout = _LAYOUTS.get(state_layout, -1) if isinstance(state_layout, str) else int(state_layout)
    if out is None:
        out = torch.empty((B, T, H, V), dtype=torch.bfloat16, device=q.device)
    if final_state is None and output_final_state:
        shape = (N, H, K, V) if layout != KDA_LAYOUT_VK else (N, H, V, K)
        final_state = torch.empty(shape, dtype=final_state_dtype, device=q.device)
    rc = lib().kda_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                          _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                          _state_dtype(initial_state), _ptr(final_state),
                          _state_dtype(final_state) if final_state is not None else KDA_STATE_F32,
                          layout, _ptr(cu_seqlens), num_seqs, _ptr(out), B, T, H, K, V,
                          _stream_handle(stream, q.device))
    if rc != 0:
        raise KDAError(rc, "kda_fwd_ex")
    return out, final_state


def kda_decode(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, state, state_out=None,
               out=None, stream=None):
    """One decode step on CUDA tensors: q, k, g bf16 [N,H,128], v bf16 [N,H,128], beta
    bf16 [N,H]; ``state`` fp32 [N,H,128,128] (S[k][v]) is updated in place unless
    ``state_out`` is given.  Returns (out [N,H,128] bf16, new state)."""
    N, H, K = q.shape
    V = v.shape[2]
    if state_out is None:
        state_out = state
    if out is None:
        out = torch.empty((N, H, V), dtype=torch.bfloat16, device=q.device)
    rc = lib().kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                          _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(state),
                          _ptr(state_out), _ptr(out), N, H, K, V, _stream_handle(stream, q.device))
    if rc != 0:
        raise KDAError(rc, "kda_decode")
    return out, state_out


def kda_bwd_workspace_size(B, T, H, K=HEAD, V=HEAD, num_seqs=0) -> int:
    """Workspace bytes of ``kda_bwd`` (0 for an invalid shape)."""
    return int(lib().kda_bwd_workspace_size(B, T, H, K, V, num_seqs))


def kda_bwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, d_out, initial_state=None,
            d_final_state=None, cu_seqlens=None, want_d_initial_state=True, workspace=None,
            stream=None):
    """Backward pass on CUDA tensors (the inputs of ``kda_fwd`` plus d_out bf16
    [B,T,H,V] and d_final_state fp32 [N,H,128,128] or None).

    Returns a dict of fp32 tensors: dq, dk, dg [B,T,H,128], dv [B,T,H,128], dbeta
    [B,T,H], dA_log [H], ddt_bias [H,128] and dS0 [N,H,128,128] (None unless
    ``want_d_initial_state``).  ``workspace`` is a CUDA uint8 tensor of at least
    ``kda_bwd_workspace_size`` bytes (allocated here if None).
    """
    B, T, H, K = q.shape
    V = v.shape[3]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    g_ = dict(dq=torch.empty((B, T, H, K), **f32), dk=torch.empty((B, T, H, K), **f32),
              dv=torch.empty((B, T, H, V), **f32), dg=torch.empty((B, T, H, K), **f32),
              dbeta=torch.empty((B, T, H), **f32), dA_log=torch.empty((H,), **f32),
              ddt_bias=torch.empty((H, K), **f32),
              dS0=torch.empty((N, H, K, V), **f32) if want_d_initial_state else None)
    need = kda_bwd_workspace_size(B, T, H, K, V, num_seqs)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    rc = lib().kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(A_log),
                       _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                       _state_dtype(initial_state), _ptr(d_out), _ptr(d_final_state),
                       _ptr(cu_seqlens), num_seqs, _ptr(g_["dq"]), _ptr(g_["dk"]), _ptr(g_["dv"]),
                       _ptr(g_["dg"]), _ptr(g_["dbeta"]), _ptr(g_["dA_log"]), _ptr(g_["ddt_bias"]),
                       _ptr(g_["dS0"]), _ptr(workspace), workspace.numel(), B, T, H, K, V,
                       _stream_handle(stream, dev))
    if rc != 0:
        raise KDAError(rc, "kda_bwd")
    return g_


def kda_fwd_raw(*args) -> int:
    """The C entry point with raw arguments (pointers as ints); returns the code."""
    return int(lib().kda_fwd(*args))


def kda_fwd_host(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
                 cu_seqlens=None, out=None, final_state=None, workspace=None, stream=None,
                 output_final_state=True):
    """Host-buffer entry point: CPU tensors in (pinned for async copies), CPU tensors out.

    ``workspace`` is a CUDA uint8 tensor of at least ``kda_fwd_host_workspace_size``
    bytes (allocated here if None).  Returns (out, final_state or None); both are
    ready when the call returns.
    """
    B, T, H, K = q.shape
    V = v.shape[3]
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else num_seqs
    if out is None:
        out = torch.empty((B, T, H, V), dtype=torch.bfloat16)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, K, V), dtype=torch.float32)
    need = kda_fwd_host_workspace_size(B, T, H, K, V, num_seqs, _state_dtype(initial_state),
                                       final_state is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    rc = lib().kda_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                            _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                            _state_dtype(initial_state), _ptr(final_state), _ptr(cu_seqlens),
                            num_seqs, _ptr(out), B, T, H, K, V, _ptr(workspace), workspace.numel(),
                            _stream_handle(stream, workspace.device))
    if rc != 0:
        raise KDAError(rc, "kda_fwd_host")
    return out, final_state
