"""Failure detection without a GPU fault: every wait inside the kernels is
bounded.  With the limit forced down to one SM cycle the pipelines give up
at once; the kernels must record SWITCH_ERR_TIMEOUT in the workspace's
error word, drain, and return -- and the context must stay usable (the next
call with the default limit is exact)."""
import numpy as np
import pytest
import torch

from switch_inputs import Workload, make_inputs
from gpu_util import dev_float

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


@pytest.mark.parametrize("flags", [0, 32, 64, 512])
def test_forced_timeouts_report_and_recover(sm, flags):
    wl = Workload("f", T=4096, d_model=256, d_ff=512, n_experts=16, capacity_factor=1.0,
                  dtype="bf16", seed=91)
    inp = make_inputs(wl)
    x, wr = dev_float(inp.x), dev_float(inp.w_r)
    w1, w2 = dev_float(inp.w1), dev_float(inp.w2)

    def run(spin):
        cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, 1.0, flags=flags,
                        spin_limit=spin)
        ws = sm.workspace(cfg)
        out = torch.empty_like(x)
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        sm.switch_layer_forward(cfg, x, wr, None, w1, w2, out, None, None, None, loss, ws)
        return sm.switch_get_device_error(ws), out

    (st, where, info), _ = run(1)
    assert st == 5, f"expected SWITCH_ERR_TIMEOUT, got {st}"      # SWITCH_ERR_TIMEOUT
    assert where in (1, 2, 3, 4, 5, 6, 9)
    (st2, _, _), out_a = run(0)
    (st3, _, _), out_b = run(0)
    assert st2 == 0 and st3 == 0
    assert torch.equal(out_a, out_b)          # deterministic again after the failure


@pytest.mark.parametrize("flags", [0, 32], ids=["pair_weight_grads", "one_cta"])
def test_backward_forced_timeouts_report_and_recover(sm, flags):
    """The backward's kernels under a one-cycle wait limit: the forward runs
    normally with SWITCH_FLAG_TRAINING, so only the backward's own pipelines
    (dH, weight gradients, dW_r, dX) give up; afterwards the same workspace
    gives the exact gradients of a clean recomputing call."""
    wl = Workload("fb", T=4096, d_model=256, d_ff=512, n_experts=16, capacity_factor=1.0,
                  dtype="bf16", seed=93)
    inp = make_inputs(wl)
    from switch_inputs import make_dout
    x, wr = dev_float(inp.x), dev_float(inp.w_r)
    w1, w2 = dev_float(inp.w1), dev_float(inp.w2)
    g = dev_float(make_dout(wl))

    def cfg(f, spin=0):
        return sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, 1.0, flags=f, spin_limit=spin)

    def backward(c, ws):
        outs = [torch.zeros_like(x), torch.zeros_like(wr), torch.zeros_like(w1),
                torch.zeros_like(w2)]
        sm.switch_layer_backward(c, x, wr, None, w1, w2, g, 1.0, outs[0], outs[1], None,
                                 outs[2], outs[3], None, ws)
        return sm.switch_get_device_error(ws), outs

    ct = cfg(flags | sm.FLAG_TRAINING)
    ws = sm.backward_workspace(ct)
    out = torch.empty_like(x)
    sm.switch_layer_forward(ct, x, wr, None, w1, w2, out, None, None, None, None, ws)
    assert sm.switch_get_device_error(ws)[0] == 0
    (st, where, info), _ = backward(cfg(flags | sm.FLAG_TRAINING, spin=1), ws)
    assert st == 5, f"expected SWITCH_ERR_TIMEOUT, got {st}"
    assert where in (1, 2, 3, 9)
    (st2, _, _), a = backward(ct, ws)
    (st3, _, _), b = backward(ct, ws)
    wsr = sm.backward_workspace(cfg(flags))
    (st4, _, _), r = backward(cfg(flags), wsr)
    assert st2 == 0 and st3 == 0 and st4 == 0
    for u, v, w in zip(a, b, r):
        assert torch.equal(u, v) and torch.equal(u, w)
