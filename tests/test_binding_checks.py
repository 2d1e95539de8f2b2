"""The Python binding rejects tensors the library cannot take, before any call (CPU).

A host tensor passed where a device pointer is expected would make a kernel read a
host address; a strided view or another dtype would be read as something else.  The
binding checks shape, dtype, contiguity and device first, raising ValueError or
TypeError, so these cases never reach libkda (which would answer with KDAError).
"""
import pytest
import torch

import linear_attention_09_b200 as kda

B, T, H, K = 1, 16, 2, 128


def args(**over):
    a = dict(q=torch.zeros(B, T, H, K, dtype=torch.bfloat16),
             k=torch.zeros(B, T, H, K, dtype=torch.bfloat16),
             v=torch.zeros(B, T, H, K, dtype=torch.bfloat16),
             g=torch.zeros(B, T, H, K, dtype=torch.bfloat16),
             beta=torch.zeros(B, T, H, dtype=torch.bfloat16), scale=0.1,
             A_log=torch.zeros(H), dt_bias=torch.zeros(H, K), lower_bound=-5.0)
    a.update(over)
    return a


@pytest.mark.parametrize("over,exc,what", [
    (dict(q=torch.zeros(B, T, H, K)), TypeError, "q has dtype"),
    (dict(k=torch.zeros(B, T + 1, H, K, dtype=torch.bfloat16)), ValueError, "k has shape"),
    (dict(g=torch.zeros(B, T, K, H, dtype=torch.bfloat16).transpose(2, 3)), ValueError,
     "g must be contiguous"),
    (dict(beta=torch.zeros(B, T, H)), TypeError, "beta has dtype"),
    (dict(A_log=torch.zeros(H, dtype=torch.float64)), TypeError, "A_log has dtype"),
    (dict(dt_bias=torch.zeros(H, K + 1)), ValueError, "dt_bias has shape"),
    (dict(initial_state=torch.zeros(B, H, K, K, dtype=torch.float16)), TypeError,
     "initial_state has dtype"),
    (dict(cu_seqlens=torch.tensor([0, T], dtype=torch.int32)), TypeError, "cu_seqlens has dtype"),
    (dict(), ValueError, "must be a CUDA tensor"),
])
def test_fwd_rejects_bad_tensors_before_the_call(over, exc, what):
    with pytest.raises(exc, match=what):
        kda.kda_fwd(**args(**over))


def test_fwd_rejects_bad_outputs():
    with pytest.raises(TypeError, match="final_state has dtype"):
        kda.kda_fwd(**args(), final_state=torch.zeros(B, H, K, K, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="out has shape"):
        kda.kda_fwd(**args(), out=torch.zeros(B, T, H, K - 1, dtype=torch.bfloat16))


def test_ex_decode_and_backward_reject_bad_tensors():
    with pytest.raises(ValueError, match="final_state has shape"):
        kda.kda_fwd_ex(**args(), final_state=torch.zeros(2, H, K, K), state_layout="vk")
    with pytest.raises(ValueError, match="must be 3-D"):
        kda.kda_decode(*[torch.zeros(B, T, H, K, dtype=torch.bfloat16)] * 5, 0.1,
                       torch.zeros(H), torch.zeros(H, K), -5.0, torch.zeros(B, H, K, K))
    q = torch.zeros(4, H, K, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="state has dtype"):
        kda.kda_decode(q, q, q, q, torch.zeros(4, H, dtype=torch.bfloat16), 0.1, torch.zeros(H),
                       torch.zeros(H, K), -5.0, torch.zeros(4, H, K, K, dtype=torch.float64))
    with pytest.raises(TypeError, match="d_out has dtype"):
        kda.kda_bwd(**args(), d_out=torch.zeros(B, T, H, K))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        kda.kda_bwd_noalloc(**args(), d_out=torch.zeros(B, T, H, K, dtype=torch.bfloat16))


def test_host_entry_point_wants_contiguous_host_tensors():
    bad = torch.zeros(B, T, K, H, dtype=torch.bfloat16).transpose(2, 3)
    with pytest.raises(ValueError, match="q must be contiguous"):
        kda.kda_fwd_host(**args(q=bad))
    with pytest.raises(TypeError, match="cu_seqlens has dtype"):
        kda.kda_fwd_host(**args(cu_seqlens=torch.tensor([0, T], dtype=torch.int32)))
