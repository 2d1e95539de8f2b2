"""Host-side tests of the C ABI: exported symbols and argument validation.

These run without a GPU: every invalid argument is rejected on the host before
any CUDA call, so fake (never dereferenced) pointers are enough.
"""
import ctypes
import os
import re

import pytest

import linear_attention_09_b200 as kda
from linear_attention_09_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kda.lib()


def header_functions():
    txt = open(os.path.join(ROOT, "include", "kda.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol(L):
    names = header_functions()
    assert {"kda_fwd", "kda_fwd_host", "kda_strerror"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/kda.h but not exported"


A16 = 0x10000  # fake 16-byte aligned addresses (never dereferenced)


def call(**over):
    args = dict(q=A16, k=A16 + 0x100, v=A16 + 0x200, g=A16 + 0x300, beta=A16 + 0x400, scale=0.1,
                A_log=A16 + 0x500, dt_bias=A16 + 0x600, lb=-5.0, init=None, init_dtype=0,
                final=None, cu=None, num_seqs=0, out=A16 + 0x700, B=1, T=64, H=2, K=128, V=128,
                stream=None)
    args.update(over)
    a = args
    return kda.kda_fwd_raw(a["q"], a["k"], a["v"], a["g"], a["beta"], ctypes.c_float(a["scale"]),
                           a["A_log"], a["dt_bias"], ctypes.c_float(a["lb"]), a["init"],
                           a["init_dtype"], a["final"], a["cu"], a["num_seqs"], a["out"], a["B"],
                           a["T"], a["H"], a["K"], a["V"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(K=64), -1), (dict(V=256), -1),
    (dict(q=None), -2), (dict(out=None), -2), (dict(A_log=None), -2), (dict(beta=None), -2),
    (dict(cu=A16 + 0x800, num_seqs=2, B=2), -3),
    (dict(cu=A16 + 0x800, num_seqs=0), -4),
    (dict(lb=-5.5), -5), (dict(lb=0.25), -5), (dict(lb=float("nan")), -5),
    (dict(init=A16 + 0x900, init_dtype=0), -6), (dict(init=None, init_dtype=1), -6),
    (dict(init=A16 + 0x900, init_dtype=7), -6),
    (dict(q=A16 + 8), -7), (dict(out=A16 + 2), -7), (dict(final=A16 + 4), -7),
    (dict(cu=A16 + 0x804, num_seqs=1), -7), (dict(beta=A16 + 1), -7),
    (dict(B=0), -8), (dict(T=-1), -8), (dict(H=0), -8),
    (dict(scale=float("inf")), -12),
])
def test_invalid_arguments_rejected_on_host(L, over, code):
    assert call(**over) == code


def test_error_strings(L):
    for c in range(-13, 1):
        s = kda.kda_strerror(c)
        assert isinstance(s, str) and s
    assert kda.kda_strerror(0) == "ok"
    assert "unknown" in kda.kda_strerror(-99)


def test_valid_arguments_without_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; the GPU tests cover valid calls")
    assert call() == -11  # no usable sm_100 device


def test_host_workspace_size(L):
    n = kda.kda_fwd_host_workspace_size(1, 64, 2, 128, 128, 0, 1, True)
    toks = 64 * 2
    assert n >= 3 * toks * 256 + 2 * toks * 256 + toks * 2 + 2 * 128 * 128 * 4 * 2
    assert kda.kda_fwd_host_workspace_size(1, 64, 2, 64, 128, 0, 0, True) == 0


def test_binding_has_no_fallback():
    src = open(os.path.join(ROOT, "linear_attention_09_b200", "__init__.py")).read()
    assert "oracle" not in src and "import numpy" not in src


def call_ex(final_dtype=1, layout=0, **over):
    args = dict(q=A16, k=A16 + 0x100, v=A16 + 0x200, g=A16 + 0x300, beta=A16 + 0x400, scale=0.1,
                A_log=A16 + 0x500, dt_bias=A16 + 0x600, lb=-5.0, init=None, init_dtype=0,
                final=A16 + 0xA00, cu=None, num_seqs=0, out=A16 + 0x700, B=1, T=64, H=2, K=128,
                V=128, stream=None)
    args.update(over)
    a = args
    return int(kda.lib().kda_fwd_ex(a["q"], a["k"], a["v"], a["g"], a["beta"],
                                    ctypes.c_float(a["scale"]), a["A_log"], a["dt_bias"],
                                    ctypes.c_float(a["lb"]), a["init"], a["init_dtype"], a["final"],
                                    final_dtype, layout, a["cu"], a["num_seqs"], a["out"], a["B"],
                                    a["T"], a["H"], a["K"], a["V"], a["stream"]))


@pytest.mark.parametrize("kw,code", [
    (dict(layout=2), -13), (dict(layout=-1), -13),
    (dict(final_dtype=0), -6), (dict(final_dtype=3), -6),
    (dict(K=64), -1), (dict(lb=1.0), -5), (dict(final=A16 + 4), -7),
])
def test_ex_invalid_arguments_rejected_on_host(L, kw, code):
    assert call_ex(**kw) == code


def test_ex_valid_arguments_without_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; the GPU tests cover valid calls")
    for layout in (0, 1):
        for fd in (1, 2):
            assert call_ex(final_dtype=fd, layout=layout) == -11
    # no final state: its dtype is not looked at
    assert call_ex(final=None, final_dtype=0) == -11


def call_decode(**over):
    a = dict(q=A16, k=A16 + 0x100, v=A16 + 0x200, g=A16 + 0x300, beta=A16 + 0x400, scale=0.1,
             A_log=A16 + 0x500, dt_bias=A16 + 0x600, lb=-5.0, sin=A16 + 0x800, sout=A16 + 0x800,
             out=A16 + 0x700, N=4, H=2, K=128, V=128, stream=None)
    a.update(over)
    return int(kda.lib().kda_decode(a["q"], a["k"], a["v"], a["g"], a["beta"],
                                    ctypes.c_float(a["scale"]), a["A_log"], a["dt_bias"],
                                    ctypes.c_float(a["lb"]), a["sin"], a["sout"], a["out"], a["N"],
                                    a["H"], a["K"], a["V"], a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(K=64), -1), (dict(V=64), -1), (dict(q=None), -2), (dict(sin=None), -2),
    (dict(sout=None), -2), (dict(out=None), -2), (dict(lb=-6.0), -5),
    (dict(sin=A16 + 0x804), -7), (dict(q=A16 + 1), -7), (dict(A_log=A16 + 2), -7),
    (dict(N=-1), -8), (dict(H=0), -8), (dict(scale=float("nan")), -12),
])
def test_decode_invalid_arguments_rejected_on_host(L, over, code):
    assert call_decode(**over) == code


def test_decode_empty_and_valid_without_device(L):
    import torch
    assert call_decode(N=0, q=None) == 0  # nothing to do
    if not torch.cuda.is_available():
        assert call_decode() == -11


def call_decode_ex(**over):
    a = dict(q=A16, k=A16 + 0x100, v=A16 + 0x200, g=A16 + 0x300, beta=A16 + 0x400, scale=0.1,
             A_log=A16 + 0x500, dt_bias=A16 + 0x600, lb=-5.0, sin=A16 + 0x800, sind=1,
             sout=A16 + 0x900, soutd=2, layout=1, out=A16 + 0x700, N=4, H=2, K=128, V=128,
             stream=None)
    a.update(over)
    return int(kda.lib().kda_decode_ex(a["q"], a["k"], a["v"], a["g"], a["beta"],
                                       ctypes.c_float(a["scale"]), a["A_log"], a["dt_bias"],
                                       ctypes.c_float(a["lb"]), a["sin"], a["sind"], a["sout"],
                                       a["soutd"], a["layout"], a["out"], a["N"], a["H"], a["K"],
                                       a["V"], a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(layout=2), -13), (dict(sind=0), -6), (dict(soutd=3), -6),
    (dict(sout=A16 + 0x800), -6),  # in place with two element types
    (dict(K=64), -1), (dict(sin=None), -2), (dict(sout=A16 + 0x908), -7),
])
def test_decode_ex_invalid_arguments_rejected_on_host(L, over, code):
    assert call_decode_ex(**over) == code


def test_decode_ex_valid_without_device(L):
    import torch
    assert call_decode_ex(N=0, q=None) == 0
    if not torch.cuda.is_available():
        assert call_decode_ex() == -11
        assert call_decode_ex(sout=A16 + 0x800, soutd=1) == -11  # in place, one dtype


WS = 0x4000000  # fake 256-byte aligned workspace address


def call_bwd(**over):
    a = dict(q=A16, k=A16 + 0x100, v=A16 + 0x200, g=A16 + 0x300, beta=A16 + 0x400, scale=0.1,
             A_log=A16 + 0x500, dt_bias=A16 + 0x600, lb=-5.0, init=None, init_dtype=0,
             dout=A16 + 0x700, dfin=None, cu=None, num_seqs=0, dq=A16 + 0x1000,
             dk=A16 + 0x1100, dv=A16 + 0x1200, dg=A16 + 0x1300, dbeta=A16 + 0x1400,
             dA=A16 + 0x1500, ddt=A16 + 0x1600, dinit=None, ws=WS, ws_bytes=None, B=1, T=64,
             H=2, K=128, V=128, stream=None)
    a.update(over)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = kda.kda_bwd_workspace_size(a["B"], a["T"], a["H"], a["K"], a["V"],
                                                   a["num_seqs"])
    return int(kda.lib().kda_bwd(
        a["q"], a["k"], a["v"], a["g"], a["beta"], ctypes.c_float(a["scale"]), a["A_log"],
        a["dt_bias"], ctypes.c_float(a["lb"]), a["init"], a["init_dtype"], a["dout"], a["dfin"],
        a["cu"], a["num_seqs"], a["dq"], a["dk"], a["dv"], a["dg"], a["dbeta"], a["dA"], a["ddt"],
        a["dinit"], a["ws"], a["ws_bytes"], a["B"], a["T"], a["H"], a["K"], a["V"], a["stream"]))


@pytest.mark.parametrize("over,code", [
    (dict(K=64), -1), (dict(q=None), -2), (dict(dout=None), -2), (dict(dq=None), -2),
    (dict(dbeta=None), -2), (dict(dA=None), -2), (dict(ddt=None), -2),
    (dict(cu=A16 + 0x800, num_seqs=2, B=2), -3), (dict(cu=A16 + 0x800, num_seqs=0), -4),
    (dict(lb=1.0), -5), (dict(init=A16 + 0x900, init_dtype=0), -6),
    (dict(dq=A16 + 4), -7), (dict(dbeta=A16 + 2), -7), (dict(dfin=A16 + 2), -7),
    (dict(ws=WS + 16), -7), (dict(T=-1), -8), (dict(ws=None), -10), (dict(ws_bytes=1024), -10),
    (dict(scale=float("inf")), -12),
])
def test_bwd_invalid_arguments_rejected_on_host(L, over, code):
    assert call_bwd(**over) == code


def test_bwd_workspace_size():
    """64 KB per 64-token chunk and head (plus one slot per sequence), per-CTA scratch
    and the per-(sequence, head) parameter partials."""
    one = kda.kda_bwd_workspace_size(1, 64, 1)
    assert one >= 2 * 65536 + 8 * 65536
    big = kda.kda_bwd_workspace_size(4, 32768, 32)
    assert big >= (4 * 32768 // 64 + 4) * 32 * 65536
    assert kda.kda_bwd_workspace_size(1, 64, 1, K=64) == 0
    assert kda.kda_bwd_workspace_size(1, 1000, 2, num_seqs=3) >= (1000 // 64 + 3) * 2 * 65536


def test_bwd_schedule_switch(L):
    """Backward schedule: "chunked" by default, "token" on request; unknown modes are
    rejected without changing the setting."""
    prev = kda.kda_set_bwd_schedule("chunked")
    try:
        assert prev == "chunked"
        assert L.kda_set_bwd_schedule(5) == -15
        assert kda.kda_set_bwd_schedule("token") == "chunked"
        assert kda.kda_set_bwd_schedule(kda.KDA_BWD_CHUNKED) == "token"
    finally:
        kda.kda_set_bwd_schedule(prev)


def test_bwd_valid_arguments_without_device(L):
    import torch
    if not torch.cuda.is_available():
        assert call_bwd() == -11
        assert call_bwd(T=0, q=None, dout=None, dq=None) == -11  # T = 0 still writes dA_log


def test_checks_level_and_message(L):
    old = kda.kda_set_checks(1)
    try:
        assert kda.kda_set_checks(1) == 1
    finally:
        kda.kda_set_checks(old)
    assert kda.kda_set_checks(old) == old
    assert "cu_seqlens" in kda.kda_strerror(-14)


def test_host_entry_checks_host_offsets_before_copying(L):
    """kda_fwd_host reads cu_seqlens on the host (it plans the copies from it), so bad
    offsets are refused with KDA_ERR_SEQLENS before any device work."""
    import numpy as np
    T, H = 100, 2
    hb = lambda *shape: np.zeros(shape, np.uint16)
    q, k, v, g = (hb(1, T, H, 128) for _ in range(4))
    beta = hb(1, T, H)
    A_log, dt = np.zeros(H, np.float32), np.zeros((H, 128), np.float32)
    out = hb(1, T, H, 128)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    for bad in ([0, 60, 50, 100], [0, 40, 101], [-1, 50, 100]):
        cu = np.asarray(bad, np.int64)
        rc = L.kda_fwd_host(p(q), p(k), p(v), p(g), p(beta), ctypes.c_float(0.1), p(A_log), p(dt),
                            ctypes.c_float(-5.0), None, 0, None, p(cu), len(bad) - 1, p(out), 1, T,
                            H, 128, 128, ctypes.c_void_p(A16), 1 << 30, None)
        assert rc == -14, bad
