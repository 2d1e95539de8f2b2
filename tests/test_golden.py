"""The C ABI's host-side validation against the interface facts the pages state
(``tests/golden/operator_contract.txt``, each line cited).  No GPU needed: every call
here is either rejected on the host or, when valid, stops at the device check
(KDA_ERR_DEVICE) on a machine without an sm_100 device."""
import ctypes
import os

import numpy as np
import pytest
import torch

import linear_attention_09_b200 as kda
from linear_attention_09_b200 import build as kbuild

HERE = os.path.dirname(os.path.abspath(__file__))
A16 = 0x10000


def contract():
    out = {}
    for line in open(os.path.join(HERE, "golden", "operator_contract.txt"), encoding="utf-8"):
        if line.startswith("#") or not line.strip():
            continue
        key, value, cite = (x.strip() for x in line.split("|", 2))
        assert cite, key
        out[key] = value
    return out


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kda.lib()


def fwd(**over):
    a = dict(init=None, init_dtype=0, final=None, cu=None, num_seqs=0, B=1, T=64, H=2, K=128,
             V=128, lb=-5.0)
    a.update(over)
    return kda.kda_fwd_raw(A16, A16 + 0x100, A16 + 0x200, A16 + 0x300, A16 + 0x400,
                           ctypes.c_float(0.1), A16 + 0x500, A16 + 0x600, ctypes.c_float(a["lb"]),
                           a["init"], a["init_dtype"], a["final"], a["cu"], a["num_seqs"],
                           A16 + 0x700, a["B"], a["T"], a["H"], a["K"], a["V"], None)


def valid_code():
    return -11 if not torch.cuda.is_available() else 0


def test_head_dims(L):
    c = contract()
    K, V = int(c["head_dim_K"]), int(c["head_dim_V"])
    if valid_code() == -11:
        assert fwd(K=K, V=V) == -11
    for bad in (64, 96, 127, 129, 256):
        assert fwd(K=bad, V=V) == -1 and fwd(K=K, V=bad) == -1


def test_lower_bound_range(L):
    c = contract()
    lo, hi = float(c["lower_bound_min"]), float(c["lower_bound_max"])
    if valid_code() == -11:
        for lb in (lo, hi, (lo + hi) / 2):
            assert fwd(lb=lb) == -11
    for lb in (np.nextafter(np.float32(lo), np.float32(-10)), np.nextafter(np.float32(hi), np.float32(1)),
               float("nan"), float("inf")):
        assert fwd(lb=float(lb)) == -5


def test_state_dtypes(L):
    c = contract()
    assert c["state_dtypes"].split(",") == ["bf16", "fp32"]
    if valid_code() == -11:
        assert fwd(init=A16 + 0x900, init_dtype=kda.KDA_STATE_BF16) == -11
        assert fwd(init=A16 + 0x900, init_dtype=kda.KDA_STATE_F32) == -11
    for bad in (3, 4, -1):
        assert fwd(init=A16 + 0x900, init_dtype=bad) == -6


def test_varlen_offsets_are_int64(L):
    """cu_seqlens is int64: the ABI takes int64_t* and wants 8-byte alignment."""
    assert contract()["cu_seqlens_dtype"] == "int64"
    assert fwd(cu=A16 + 0x804, num_seqs=1) == -7
    if valid_code() == -11:
        assert fwd(cu=A16 + 0x808, num_seqs=1) == -11


def test_binding_dtypes_follow_the_contract():
    """The binding allocates bf16 outputs and passes fp32 gate parameters through."""
    c = contract()
    assert c["qkvg_dtype"] == c["out_dtype"] == "bf16" and c["gate_param_dtype"] == "fp32"
    import inspect
    src = inspect.getsource(kda.kda_fwd)
    assert "torch.bfloat16" in src
    assert kda._state_dtype(torch.zeros(1, dtype=torch.bfloat16)) == kda.KDA_STATE_BF16
    assert kda._state_dtype(torch.zeros(1, dtype=torch.float32)) == kda.KDA_STATE_F32
    assert kda._state_dtype(torch.zeros(1, dtype=torch.float64)) == -1
