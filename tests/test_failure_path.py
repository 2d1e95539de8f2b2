"""The forward kernel's failure path, exercised without a GPU fault.

A bounded wait that gives up records (launch epoch << 8) | code in the device error
word; every CTA of the same launch that starts afterwards sees its epoch there and
returns before doing any work.  ``kda_inject_error`` makes a launch start in that
state, so the path runs on the GPU with nothing hung: the launch must return
promptly, write neither output, report the code, and leave the next launch intact.
"""
import time

import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_09_b200 as kda
import oracle


def test_inject_rejects_codes_outside_a_byte():
    for bad in (-1, 256, 1 << 20):
        with pytest.raises(kda.KDAError) as e:
            kda.kda_inject_error(bad)
        assert e.value.code == -15  # KDA_ERR_ARG
    kda.kda_inject_error(0)  # cancelling with nothing pending is fine


@pytest.mark.gpu
def test_launch_that_starts_failed_returns_at_once_and_the_next_one_works():
    w = ki.Workload("fail", B=2, T=300, H=6, init_state="f32")
    inp = ki.make_inputs(w, 3)
    d = lambda t: t.to("cuda")
    call = dict(q=d(inp.q), k=d(inp.k), v=d(inp.v), g=d(inp.g), beta=d(inp.beta), scale=inp.scale,
                A_log=d(inp.A_log), dt_bias=d(inp.dt_bias), lower_bound=inp.lower_bound,
                initial_state=d(inp.initial_state))
    kda.kda_device_status(reset=True)
    out = torch.full((2, 300, 6, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    fin = torch.full((2, 6, 128, 128), 5.0, dtype=torch.float32, device="cuda")
    kda.kda_inject_error(42)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    kda.kda_fwd(**call, out=out, final_state=fin)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert kda.kda_device_status(reset=True) == 42
    assert elapsed < 0.5, f"a launch that starts failed took {elapsed:.3f} s"
    assert torch.all(out == 3.0) and torch.all(fin == 5.0), "a failed launch wrote results"
    # the injection is consumed: the next launch runs normally
    o, f = kda.kda_fwd(**call)
    torch.cuda.synchronize()
    assert kda.kda_device_status(reset=True) == 0
    out_r, fin_r = oracle.forward_inputs(inp)
    og = o.float().cpu().numpy().astype(np.float64)
    assert np.abs(og - out_r).max() <= 3e-2
    fg = f.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(fg - fin_r) / np.linalg.norm(fin_r) <= 1e-3
