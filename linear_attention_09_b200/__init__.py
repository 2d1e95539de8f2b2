"""Python binding of libkda.so, the B200 (sm_100a) Kimi Delta Attention forward and backward passes.

Argument marshalling only: every step of the pass runs in the CUDA kernels of
``libkda.so``.  PyTorch provides device memory and streams.  There is no CPU or
PyTorch fallback: if the library cannot be loaded, the calls raise.

The functions mirror the C ABI in ``include/kda.h``:
  kda_fwd, kda_fwd_ex, kda_decode, kda_decode_ex, kda_bwd, kda_bwd_noalloc,
  kda_bwd_workspace_size,
  kda_fwd_host,
  kda_fwd_host_workspace_size, kda_set_checks, kda_strerror, kda_last_launch_count,
  kda_device_status, kda_inject_error, kda_set_schedule, kda_last_schedule,
  kda_set_bwd_schedule.
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
            L.kda_decode_ex.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, I, I, P, I64, I64, I64,
                                        I64, P]
            L.kda_decode_ex.restype = I
            L.kda_fwd_host.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, I64, P, I64, I64,
                                       I64, I64, I64, P, SZ, P]
            L.kda_fwd_host.restype = I
            L.kda_fwd_host_workspace_size.argtypes = [I64, I64, I64, I64, I64, I64, I, I]
            L.kda_fwd_host_workspace_size.restype = SZ
            L.kda_bwd.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, P, I64, P, P, P, P, P,
                                  P, P, P, P, SZ, I64, I64, I64, I64, I64, P]
            L.kda_bwd.restype = I
            L.kda_bwd_noalloc.argtypes = [P, P, P, P, P, F, P, P, F, P, I, P, P, P, I64, P, P, P,
                                          P, P, P, P, P, I64, I64, I64, I64, I64, P]
            L.kda_bwd_noalloc.restype = I
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
            L.kda_inject_error.argtypes = [I]
            L.kda_inject_error.restype = I
            L.kda_set_schedule.argtypes = [I]
            L.kda_set_schedule.restype = I
            L.kda_last_schedule.argtypes = []
            L.kda_last_schedule.restype = I
            L.kda_set_bwd_schedule.argtypes = [I]
            L.kda_set_bwd_schedule.restype = I
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


KDA_SCHEDULE_AUTO, KDA_SCHEDULE_FUSED, KDA_SCHEDULE_SPLIT = 0, 1, 2
_SCHEDULES = {"auto": KDA_SCHEDULE_AUTO, "fused": KDA_SCHEDULE_FUSED, "split": KDA_SCHEDULE_SPLIT}


def kda_set_schedule(mode) -> str:
    """Forward kernel schedule, process-wide: "auto" (default), "fused" (one CTA per
    (sequence, head)) or "split" (a 4-CTA cluster per unit whenever all units fit the
    device); returns the previous one.  Results are identical under every schedule."""
    rc = lib().kda_set_schedule(_SCHEDULES[mode] if isinstance(mode, str) else int(mode))
    if rc < 0:
        raise KDAError(rc, "kda_set_schedule")
    return {v: k for k, v in _SCHEDULES.items()}[rc]


def kda_last_schedule() -> str:
    """Schedule ("fused" or "split") of this thread's last forward launch."""
    return {v: k for k, v in _SCHEDULES.items()}[int(lib().kda_last_schedule())]


KDA_BWD_CHUNKED, KDA_BWD_TOKEN = 0, 1
_BWD_SCHEDULES = {"chunked": KDA_BWD_CHUNKED, "token": KDA_BWD_TOKEN}


def kda_set_bwd_schedule(mode) -> str:
    """Backward pass schedule, process-wide: "chunked" (default: the forward kernel's
    chunk checkpoints, then the chunked matrix form in reverse) or "token" (the token
    recurrence reversed step by step); returns the previous one."""
    rc = lib().kda_set_bwd_schedule(_BWD_SCHEDULES[mode] if isinstance(mode, str) else int(mode))
    if rc < 0:
        raise KDAError(rc, "kda_set_bwd_schedule")
    return {v: k for k, v in _BWD_SCHEDULES.items()}[rc]


def kda_inject_error(code: int) -> None:
    """Testing hook: the next forward launch starts as if one of its CTAs had given up
    with ``code`` (1..255); its CTAs return at once and kda_device_status reports it.
    Code 0 cancels a pending injection."""
    rc = lib().kda_inject_error(int(code))
    if rc != 0:
        raise KDAError(rc, "kda_inject_error")


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


def _check_form(t, name, dtypes, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected "
                        + " or ".join(str(d) for d in dtypes))
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major, no strides)")


def _check_place(t, name, device, host):
    if host:
        if t.device.type != "cpu":
            raise ValueError(f"{name} must be a host (CPU) tensor, got {t.device}")
    elif t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor, got {t.device}")
    elif device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (the device of q)")


def _check_all(specs, device=None, host=False):
    """Reject tensors the library cannot take: wrong shape, dtype or memory layout
    (checked for every tensor first), then wrong device.  Nothing is launched on a bad
    argument: a host pointer handed to a kernel would fault the GPU, and a strided view
    or another dtype would be read as something else.  ``specs``: (tensor or None,
    name, allowed dtypes, shape or None); None tensors are optional and skipped."""
    specs = [sp for sp in specs if sp[0] is not None]
    for t, name, dtypes, shape in specs:
        _check_form(t, name, dtypes, shape)
    for t, name, _, _ in specs:
        _check_place(t, name, device, host)


_BF16, _F32, _I64, _U8 = (torch.bfloat16,), (torch.float32,), (torch.int64,), (torch.uint8,)
_STATE = (torch.float32, torch.bfloat16)


def _check_call(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, extra=(),
                host=False, state_shape=None):
    """Shapes, dtypes, layouts and devices of the common arguments and of ``extra``
    specs (q decides B, T, H, K and the device).  Returns (B, T, H, K, V, N)."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a 4-D tensor [B, T, H, K]")
    if not isinstance(v, torch.Tensor) or v.dim() != 4:
        raise ValueError("v must be a 4-D tensor [B, T, H, V]")
    if cu_seqlens is not None and (not isinstance(cu_seqlens, torch.Tensor)
                                   or cu_seqlens.dim() != 1):
        raise ValueError("cu_seqlens must be a 1-D tensor [num_seqs + 1]")
    B, T, H, K = q.shape
    V = v.shape[3]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    dims = dict(B=B, T=T, H=H, K=K, V=V, N=N)
    specs = [(q, "q", _BF16, (B, T, H, K)), (k, "k", _BF16, (B, T, H, K)),
             (g, "g", _BF16, (B, T, H, K)), (v, "v", _BF16, (B, T, H, V)),
             (beta, "beta", _BF16, (B, T, H)), (A_log, "A_log", _F32, (H,)),
             (dt_bias, "dt_bias", _F32, (H, K)), (cu_seqlens, "cu_seqlens", _I64, None),
             (initial_state, "initial_state", _STATE, state_shape or (N, H, K, V))]
    specs += [(t, n, d, (sh(dims) if callable(sh) else sh)) for t, n, d, sh in extra]
    _check_all(specs, None if host else q.device, host)
    return B, T, H, K, V, N


def kda_fwd(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, initial_state=None,
            final_state=None, cu_seqlens=None, out=None, output_final_state=True, stream=None):
    """Run the KDA forward pass on CUDA tensors; returns (out, final_state or None).

    q, k, g: bf16 [B,T,H,128]; v: bf16 [B,T,H,128]; beta: bf16 [B,T,H];
    A_log: fp32 [H]; dt_bias: fp32 [H,128]; initial_state: fp32/bf16 [N,H,128,128]
    or None; cu_seqlens: int64 [N+1] or None.  ``out`` / ``final_state`` may be
    given (then they are written), else they are allocated on q's device.  The
    call is asynchronous on ``stream`` (default: the current stream).
    """
    B, T, H, K, V, N = _check_call(
        q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens,
        extra=[(out, "out", _BF16, lambda d: (d["B"], d["T"], d["H"], d["V"])),
               (final_state, "final_state", _F32, lambda d: (d["N"], d["H"], d["K"], d["V"]))])
    num_seqs = 0 if cu_seqlens is None else N
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
    layout = _LAYOUTS.get(state_layout, -1) if isinstance(state_layout, str) else int(state_layout)
    vk = layout == KDA_LAYOUT_VK
    B, T, H, K, V, N = _check_call(
        q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens,
        extra=[(out, "out", _BF16, lambda d: (d["B"], d["T"], d["H"], d["V"])),
               (final_state, "final_state", _STATE,
                lambda d: (d["N"], d["H"]) + ((d["V"], d["K"]) if vk else (d["K"], d["V"])))])
    num_seqs = 0 if cu_seqlens is None else N
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
    if not isinstance(q, torch.Tensor) or q.dim() != 3 or not isinstance(v, torch.Tensor) \
            or v.dim() != 3:
        raise ValueError("q and v must be 3-D tensors [N, H, K] / [N, H, V]")
    N, H, K = q.shape
    V = v.shape[2]
    if state is None:
        raise ValueError("state is required")
    _check_all([(q, "q", _BF16, (N, H, K)), (k, "k", _BF16, (N, H, K)), (g, "g", _BF16, (N, H, K)),
                (v, "v", _BF16, (N, H, V)), (beta, "beta", _BF16, (N, H)),
                (A_log, "A_log", _F32, (H,)), (dt_bias, "dt_bias", _F32, (H, K)),
                (state, "state", _F32, (N, H, K, V)), (state_out, "state_out", _F32, (N, H, K, V)),
                (out, "out", _BF16, (N, H, V))], q.device)
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


def kda_decode_ex(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, state, state_out=None,
                  out=None, state_layout="kv", state_out_dtype=None, stream=None):
    """``kda_decode`` with the state variants of ``kda_fwd_ex``: ``state`` fp32 or bf16 in
    the "kv" (S[k][v], [N,H,K,V]) or "vk" (S[v][k], [N,H,V,K]) layout; the new state goes
    to ``state_out`` (default: in place, which needs ``state_out_dtype`` equal to the
    input's) with ``state_out_dtype`` (default: the input's, or that of a given
    ``state_out``).  Returns (out [N,H,128] bf16, new state)."""
    if not isinstance(q, torch.Tensor) or q.dim() != 3 or not isinstance(v, torch.Tensor) \
            or v.dim() != 3:
        raise ValueError("q and v must be 3-D tensors [N, H, K] / [N, H, V]")
    N, H, K = q.shape
    V = v.shape[2]
    layout = _LAYOUTS.get(state_layout, -1) if isinstance(state_layout, str) else int(state_layout)
    shp = (N, H, V, K) if layout == KDA_LAYOUT_VK else (N, H, K, V)
    if state is None:
        raise ValueError("state is required")
    if state_out is None:
        want = state.dtype if state_out_dtype is None else state_out_dtype
        state_out = state if want == state.dtype else torch.empty(shp, dtype=want, device=q.device)
    _check_all([(q, "q", _BF16, (N, H, K)), (k, "k", _BF16, (N, H, K)), (g, "g", _BF16, (N, H, K)),
                (v, "v", _BF16, (N, H, V)), (beta, "beta", _BF16, (N, H)),
                (A_log, "A_log", _F32, (H,)), (dt_bias, "dt_bias", _F32, (H, K)),
                (state, "state", _STATE, shp), (state_out, "state_out", _STATE, shp),
                (out, "out", _BF16, (N, H, V))], q.device)
    if out is None:
        out = torch.empty((N, H, V), dtype=torch.bfloat16, device=q.device)
    rc = lib().kda_decode_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                             _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(state),
                             _state_dtype(state), _ptr(state_out), _state_dtype(state_out), layout,
                             _ptr(out), N, H, K, V, _stream_handle(stream, q.device))
    if rc != 0:
        raise KDAError(rc, "kda_decode_ex")
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
    ``kda_bwd_workspace_size`` bytes (allocated here if None).  The schedule is the
    process-wide one of ``kda_set_bwd_schedule`` ("chunked" by default: three kernel
    launches, the forward kernel's chunk checkpoints, the chunked reverse and a
    parameter reduction).
    """
    if d_out is None:
        raise ValueError("d_out is required")
    B, T, H, K, V, N = _check_call(
        q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens,
        extra=[(d_out, "d_out", _BF16, lambda d: (d["B"], d["T"], d["H"], d["V"])),
               (d_final_state, "d_final_state", _F32, lambda d: (d["N"], d["H"], d["K"], d["V"])),
               (workspace, "workspace", _U8, None)])
    num_seqs = 0 if cu_seqlens is None else N
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


KDA_BWD_NOALLOC_MAX_BYTES = 64 << 20


def kda_bwd_noalloc(q, k, v, g, beta, scale, A_log, dt_bias, lower_bound, d_out,
                    initial_state=None, d_final_state=None, cu_seqlens=None,
                    want_d_initial_state=True, grads=None, stream=None):
    """``kda_bwd`` through the entry point that allocates no device memory: its
    workspace is the library's own fixed 64 MiB device array (shapes that need more
    are rejected with KDA_ERR_WORKSPACE).  For callers that cannot allocate, pass
    ``grads``, a dict of preallocated fp32 outputs with the keys and shapes ``kda_bwd``
    returns; otherwise they are allocated here.  Calls that overlap on the GPU share
    the array and race."""
    if d_out is None:
        raise ValueError("d_out is required")
    gr = grads or {}
    if grads is not None and any(grads.get(n) is None for n in
                                 ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias")):
        raise ValueError("grads must hold dq, dk, dv, dg, dbeta, dA_log and ddt_bias")
    shp = lambda *ks: (lambda d: tuple(d[x] for x in ks))
    B, T, H, K, V, N = _check_call(
        q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens,
        extra=[(d_out, "d_out", _BF16, shp("B", "T", "H", "V")),
               (d_final_state, "d_final_state", _F32, shp("N", "H", "K", "V")),
               (gr.get("dq"), "dq", _F32, shp("B", "T", "H", "K")),
               (gr.get("dk"), "dk", _F32, shp("B", "T", "H", "K")),
               (gr.get("dv"), "dv", _F32, shp("B", "T", "H", "V")),
               (gr.get("dg"), "dg", _F32, shp("B", "T", "H", "K")),
               (gr.get("dbeta"), "dbeta", _F32, shp("B", "T", "H")),
               (gr.get("dA_log"), "dA_log", _F32, shp("H")),
               (gr.get("ddt_bias"), "ddt_bias", _F32, shp("H", "K")),
               (gr.get("dS0"), "dS0", _F32, shp("N", "H", "K", "V"))])
    num_seqs = 0 if cu_seqlens is None else N
    if grads is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        grads = dict(dq=torch.empty((B, T, H, K), **f32), dk=torch.empty((B, T, H, K), **f32),
                     dv=torch.empty((B, T, H, V), **f32), dg=torch.empty((B, T, H, K), **f32),
                     dbeta=torch.empty((B, T, H), **f32), dA_log=torch.empty((H,), **f32),
                     ddt_bias=torch.empty((H, K), **f32),
                     dS0=torch.empty((N, H, K, V), **f32) if want_d_initial_state else None)
    rc = lib().kda_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                               _ptr(A_log), _ptr(dt_bias), float(lower_bound), _ptr(initial_state),
                               _state_dtype(initial_state), _ptr(d_out), _ptr(d_final_state),
                               _ptr(cu_seqlens), num_seqs, _ptr(grads["dq"]), _ptr(grads["dk"]),
                               _ptr(grads["dv"]), _ptr(grads["dg"]), _ptr(grads["dbeta"]),
                               _ptr(grads["dA_log"]), _ptr(grads["ddt_bias"]),
                               _ptr(grads.get("dS0")), B, T, H, K, V,
                               _stream_handle(stream, q.device))
    if rc != 0:
        raise KDAError(rc, "kda_bwd_noalloc")
    return grads


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
    B, T, H, K, V, N = _check_call(
        q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, host=True,
        extra=[(out, "out", _BF16, lambda d: (d["B"], d["T"], d["H"], d["V"])),
               (final_state, "final_state", _F32, lambda d: (d["N"], d["H"], d["K"], d["V"]))])
    num_seqs = 0 if cu_seqlens is None else N
    if workspace is not None:
        _check_all([(workspace, "workspace", _U8, None)])
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
