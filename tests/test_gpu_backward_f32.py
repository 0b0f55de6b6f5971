"""Parity of switch_layer_backward in fp32 (dtype SWITCH_F32) against the
oracle's backward passes, top-1 and top-2.

The fp32 path keeps every operand and output in fp32, so the bounds are
fp32's, not bf16's: max |GPU - oracle| <= 1e-4 and RMS(GPU - oracle) <= 2e-5
of RMS(oracle) per gradient.  Derivation: a gradient element is the end of a
chain of at most three fp32 dot products (dY W2 -> dA, dA W1 -> dx; dA^T x ->
dW1), each over at most a few thousand terms, whose rounding error is about
2^-24 sqrt(K) of the terms' magnitude (3e-6 at K = 3000); the chain and the
largest of 10^5 elements stay below 1e-4, and the RMS below 2e-5.  As in the
bf16 tests, hidden units whose pre-activation lies within the accumulation
error of zero may take either ReLU branch; their whole contribution is
allowed on top of the max bound (the RMS bound is not relaxed), and the
oracle is re-based on the GPU's routing.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import Workload, WORKLOADS, make_inputs, make_dout
from gpu_util import check_routing
from test_gpu_backward import run_backward, relu_ambiguity
from test_gpu_backward_top2 import run_backward_top2
from test_gpu_top2 import check_top2_routing

pytestmark = pytest.mark.gpu

F32_MAX_TOL = 1e-4
F32_RMS_TOL = 2e-5


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def grad_ok32(got, want, name, allow=None):
    want = np.asarray(want, np.float64)
    err = np.asarray(got, np.float64) - want
    rms = max(float(np.sqrt(np.mean(want * want))), 1e-30)
    excess = np.abs(err) if allow is None else np.maximum(np.abs(err) - allow, 0.0)
    mx = float(np.max(excess)) / rms
    rm = float(np.sqrt(np.mean(err * err))) / rms
    assert mx <= F32_MAX_TOL and rm <= F32_RMS_TOL, \
        f"{name}: max err / rms = {mx:.3g}, rms err / rms = {rm:.3g}"
    return mx, rm


def allowances(inp, want, idx_routes, gates, dout):
    """ReLU-margin allowances for dW1 [N, F, d] and dx [T, d] from every
    kept (token, expert) pair."""
    N = inp.w1.shape[0]
    a_w1 = np.zeros(inp.w1.shape)
    a_dx = np.zeros(inp.x.shape)
    for e in range(N):
        for r, (idx, g) in enumerate(zip(idx_routes, gates)):
            toks = np.nonzero((idx == e) & ~want["drops"][r])[0]
            if toks.size == 0:
                continue
            aw, ax, _ = relu_ambiguity(inp.x[toks], inp.w1[e], inp.w2[e], g[toks], dout[toks])
            a_w1[e] += aw
            a_dx[toks] += ax
    return a_w1, a_dx


def check_f32(sm, wl, dloss=1.0, flags=0):
    inp = make_inputs(wl)
    dout = make_dout(wl)
    residual = not (flags & sm.FLAG_NO_RESIDUAL)
    if flags & sm.FLAG_TOP2:
        idx2, got = run_backward_top2(sm, wl, inp, dout, dloss, flags & ~sm.FLAG_TOP2, inp.b_r)
        check_top2_routing(idx2, orc.router_top2(inp.x, inp.w_r, inp.b_r))
        want = orc.layer_backward_top2(inp.x, inp.w_r, inp.b_r, inp.w1, inp.w2,
                                       wl.capacity_factor, dout, dloss=dloss, alpha=wl.alpha,
                                       residual=residual, idx2=idx2)
        got["dgate"] = got["dgate"].reshape(2, -1)
        p = orc.router(inp.x, inp.w_r, inp.b_r)["probs"]
        gates = [p[np.arange(wl.T), idx2[r]] for r in range(2)]
        want["drops"] = want["drop2"]
        a_w1, a_dx = allowances(inp, want, [idx2[0], idx2[1]], gates, dout)
    else:
        idx, got = run_backward(sm, wl, inp, dout, dloss, flags)
        r = orc.router(inp.x, inp.w_r, inp.b_r)
        check_routing(idx, r)
        want = orc.layer_backward(inp.x, inp.w_r, inp.b_r, inp.w1, inp.w2, wl.capacity_factor,
                                  dout, dloss=dloss, alpha=wl.alpha, residual=residual, idx=idx)
        want["drops"] = want["drop"][None, :]
        gates = [r["probs"][np.arange(wl.T), idx]]
        a_w1, a_dx = allowances(inp, want, [idx], gates, dout)
    for name, allow in (("dx", a_dx), ("dw1", a_w1), ("dw2", None), ("dw_r", None),
                        ("dgate", None), ("db_r", None)):
        assert np.isfinite(got[name]).all(), name
        print(wl.name, name, "max/rms err ratios %.3g %.3g" % grad_ok32(got[name], want[name],
                                                                         name, allow))
    return got, want


TINY = WORKLOADS["tiny"]


def test_backward_f32_tiny(sm):
    """The pages' fp32 configuration: T 512, d 64, d_ff 256, N 4, cf 1.25."""
    got, want = check_f32(sm, TINY)
    assert not np.any(got["dgate"][want["drop"]])


@pytest.mark.parametrize("flags", [16, 1], ids=["no_residual", "simt_router"])
def test_backward_f32_flags(sm, flags):
    check_f32(sm, TINY, dloss=0.5, flags=flags)


def test_backward_f32_drops_ragged(sm):
    """Capacity factor 0.5 (about half the tokens dropped) and sizes that are
    not multiples of any tile (d 36, d_ff 100, N 5, T 777)."""
    wl = Workload("f32_drop", T=777, d_model=36, d_ff=100, n_experts=5, capacity_factor=0.5,
                  dtype="f32", seed=41)
    got, want = check_f32(sm, wl, dloss=2.0)
    assert want["drop"].mean() > 0.3


def test_backward_f32_top2(sm):
    got, want = check_f32(sm, Workload("f32_top2", T=600, d_model=64, d_ff=128, n_experts=4,
                                       capacity_factor=1.0, dtype="f32", seed=43),
                          flags=sm.FLAG_TOP2)
    d = want["drop2"]
    assert d[1].any() and (~d).all(axis=0).any()


def test_backward_f32_saved_state(sm):
    """SWITCH_FLAG_TRAINING in fp32: the kept-state backward equals the
    recomputing one bit for bit."""
    wl = TINY
    inp = make_inputs(wl)
    dout = make_dout(wl)
    _, a = run_backward(sm, wl, inp, dout)
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor, dtype="f32",
                    alpha=wl.alpha, flags=sm.FLAG_TRAINING)
    ws = sm.backward_workspace(cfg)
    _, b = run_backward(sm, wl, inp, dout, flags=sm.FLAG_TRAINING, reuse_ws=ws)
    _, c = run_backward(sm, wl, inp, dout, flags=sm.FLAG_TRAINING, reuse_ws=ws)
    for k in a:
        assert np.array_equal(a[k], b[k], equal_nan=True) and \
            np.array_equal(b[k], c[k], equal_nan=True), k
