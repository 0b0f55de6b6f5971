"""Parity of switch_layer_backward with top-2 routing (SWITCH_FLAG_TOP2)
against the oracle's layer_backward_top2.

The oracle is re-based on the GPU's two choices per token (read from a
forward call on the same inputs; the backward recomputes the same routing),
then every gradient is compared element by element with the top-1 backward's
bounds (max |GPU - oracle| <= 4e-2 and RMS(GPU - oracle) <= 5e-3 of the
oracle's RMS; the derivation is the same: each route's terms pass through
the same bf16 roundings, and a token's two routes' dx rows are added in fp32
before the one bf16 rounding of dx).  The gate gradient is compared per
route, [2, T].  Routing flips follow the top-2 forward tests' rule.

At full size (Base: T = 65536, N = 128, capacity 1280 over the 2T
assignments) the oracle computes sampled tokens' dx and both routes' gate
gradients, and three experts' weight gradients, one by one.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import Workload, WORKLOADS, make_inputs, make_dout, as_f64
from gpu_util import dev_float, host_f64
from test_gpu_backward import grad_ok, relu_ambiguity
from test_gpu_top2 import check_top2_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _cfg(sm, wl, flags=0):
    return sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                     dtype=wl.dtype, alpha=wl.alpha, flags=sm.FLAG_TOP2 | flags)


def _ok(sm, ws):
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"


def _forward_idx2(sm, cfg, dev, ws):
    x, w_r, b_r, w1, w2 = dev
    out = torch.empty_like(x)
    idx = torch.empty(2 * cfg.T, dtype=torch.int32, device="cuda")
    sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx, None, None, None, ws)
    _ok(sm, ws)
    return idx.cpu().numpy().astype(np.int64).reshape(2, -1)


def run_backward_top2(sm, wl, inp, dout, dloss=1.0, flags=0, b_r=None, to_host=True):
    cfg = _cfg(sm, wl, flags)
    ws = sm.backward_workspace(cfg)
    dev = (dev_float(inp.x), dev_float(inp.w_r), None if b_r is None else dev_float(b_r),
           dev_float(inp.w1), dev_float(inp.w2))
    idx2 = _forward_idx2(sm, cfg, dev, ws)
    x, w_r, b_d, w1, w2 = dev
    g = dev_float(dout)
    res = {"dx": torch.full_like(x, float("nan")), "dw_r": torch.full_like(w_r, float("nan")),
           "db_r": torch.full((wl.n_experts,), float("nan"), device="cuda"),
           "dw1": torch.full_like(w1, float("nan")), "dw2": torch.full_like(w2, float("nan")),
           "dgate": torch.full((2 * wl.T,), float("nan"), device="cuda")}
    sm.switch_layer_backward(cfg, x, w_r, b_d, w1, w2, g, dloss, res["dx"], res["dw_r"],
                             res["db_r"], res["dw1"], res["dw2"], res["dgate"], ws)
    _ok(sm, ws)
    if to_host:
        res = {k: host_f64(v) for k, v in res.items()}
    return idx2, res


def check_backward_top2(sm, wl, dloss=1.0, flags=0, b_r=None):
    inp = make_inputs(wl)
    dout = make_dout(wl)
    b_np = inp.b_r if b_r is None else b_r
    idx2, got = run_backward_top2(sm, wl, inp, dout, dloss, flags, b_np)
    r = orc.router_top2(inp.x, inp.w_r, b_np)
    check_top2_routing(idx2, r)
    residual = not (flags & sm.FLAG_NO_RESIDUAL)
    want = orc.layer_backward_top2(inp.x, inp.w_r, b_np, inp.w1, inp.w2, wl.capacity_factor,
                                   dout, dloss=dloss, alpha=wl.alpha, residual=residual,
                                   idx2=idx2)
    got["dgate"] = got["dgate"].reshape(2, -1)
    for name in ("dx", "dw1", "dw2", "dw_r", "dgate"):
        assert np.isfinite(got[name]).all(), name
        print(wl.name, name, "max/rms err ratios %.3g %.3g" % grad_ok(got[name], want[name], name))
    if b_np is not None:
        grad_ok(got["db_r"], want["db_r"], "db_r")
    # a dropped route's gate gradient is exactly zero
    assert np.all(got["dgate"][want["drop2"]] == 0)
    return got, want


SMALL2 = Workload("bwd2_small", T=3000, d_model=320, d_ff=576, n_experts=8, capacity_factor=1.0,
                  dtype="bf16", seed=93)


def test_backward_top2_small(sm):
    """Capacity factor 1 over the 2T assignments: some second choices are
    dropped, tokens with one and with two kept routes both occur."""
    got, want = check_backward_top2(sm, SMALL2)
    d = want["drop2"]
    assert d[1].any() and (~d[1]).any() and (~d).all(axis=0).any()


@pytest.mark.parametrize("flags", [1, 16, 64, 2048, 32],
                         ids=["simt_router", "no_residual", "gemm1_pairs", "gemm1_rows_pairs",
                              "gemm_1sm"])
def test_backward_top2_flags(sm, flags):
    check_backward_top2(sm, SMALL2, dloss=0.5, flags=flags)


def test_backward_top2_heavy_drop_and_bias(sm):
    """Capacity factor 0.3: many tokens lose both routes (their dx is the
    residual plus the router term only) or keep only their first; a router
    bias and dloss = 3."""
    wl = Workload("bwd2_drop", T=2048, d_model=256, d_ff=512, n_experts=16,
                  capacity_factor=0.3, dtype="bf16", seed=19)
    rng = np.random.default_rng(8)
    bias = (0.05 * rng.standard_normal(wl.n_experts)).astype(np.float32)
    got, want = check_backward_top2(sm, wl, dloss=3.0, b_r=bias)
    both = want["drop2"].all(axis=0)
    assert both.mean() > 0.2 and (want["drop2"][1] & ~want["drop2"][0]).any()


def test_backward_top2_two_experts_no_drops_ragged(sm):
    """N = 2 (every kept token uses both experts) with every assignment kept,
    and sizes that are ragged in every tile dimension."""
    wl = Workload("bwd2_two", T=1000, d_model=192, d_ff=320, n_experts=2,
                  capacity_factor=2.0, dtype="bf16", seed=25)
    got, want = check_backward_top2(sm, wl)
    assert not want["drop2"].any()


def test_backward_top2_many_experts_tiny_batch(sm):
    """N = 100 (bf16 planes padded to 128 columns) and a batch smaller than
    one 128-token tile."""
    for wl in (Workload("bwd2_n100", T=2500, d_model=128, d_ff=192, n_experts=100,
                        capacity_factor=1.0, dtype="bf16", seed=27),
               Workload("bwd2_tiny", T=37, d_model=64, d_ff=128, n_experts=4,
                        capacity_factor=1.0, dtype="bf16", seed=39)):
        check_backward_top2(sm, wl, dloss=2.0)


def test_backward_top2_wide_router(sm):
    """N = 300 with top-2: the FMA router (the CTA-pair router's top-2 form
    takes N <= 128), planes padded to 320 columns; about 40 kept assignments
    per expert."""
    wl = Workload("bwd2_n300", T=6000, d_model=128, d_ff=128, n_experts=300,
                  capacity_factor=1.5, dtype="bf16", seed=35)
    check_backward_top2(sm, wl, dloss=1.5)


def _all_grads(sm, cfg, dev, g, ws):
    x, w_r, b_r, w1, w2 = dev
    outs = [torch.empty_like(x), torch.empty_like(w_r),
            torch.empty(cfg.n_experts, device="cuda"), torch.empty_like(w1),
            torch.empty_like(w2), torch.empty(2 * cfg.T, device="cuda")]
    sm.switch_layer_backward(cfg, x, w_r, b_r, w1, w2, g, 1.0, *outs, ws)
    _ok(sm, ws)
    return [t.cpu() for t in outs]


def _forward_all(sm, cfg, dev, ws):
    x, w_r, b_r, w1, w2 = dev
    outs = [torch.empty_like(x), torch.empty(2 * cfg.T, dtype=torch.int32, device="cuda"),
            torch.empty(2 * cfg.T, device="cuda"),
            torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda"),
            torch.empty(1, device="cuda")]
    sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, *outs, ws)
    _ok(sm, ws)
    return [t.cpu() for t in outs]


def test_backward_top2_saved_state_and_determinism(sm):
    """SWITCH_FLAG_TRAINING with top-2: the forward keeps its state, the
    backward reads it; outputs and gradients equal the plain forward's and
    the recomputing backward's bit for bit, and repeat on a second call."""
    wl = SMALL2
    inp = make_inputs(wl)
    rng = np.random.default_rng(4)
    bias = (0.05 * rng.standard_normal(wl.n_experts)).astype(np.float32)
    dev = (dev_float(inp.x), dev_float(inp.w_r), dev_float(bias), dev_float(inp.w1),
           dev_float(inp.w2))
    g = dev_float(make_dout(wl))
    cfg0, cfg1 = _cfg(sm, wl), _cfg(sm, wl, sm.FLAG_TRAINING)
    ws0 = sm.backward_workspace(cfg0)
    f0 = _forward_all(sm, cfg0, dev, ws0)
    b0 = _all_grads(sm, cfg0, dev, g, ws0)
    b0r = _all_grads(sm, cfg0, dev, g, ws0)
    ws1 = sm.backward_workspace(cfg1)
    f1 = _forward_all(sm, cfg1, dev, ws1)
    b1 = _all_grads(sm, cfg1, dev, g, ws1)
    b2 = _all_grads(sm, cfg1, dev, g, ws1)
    for a, b in zip(f0, f1):
        assert torch.equal(a, b)
    for a, a2, b, c in zip(b0, b0r, b1, b2):
        assert torch.equal(a, a2) and torch.equal(a, b) and torch.equal(b, c)


def test_backward_top2_fullsize_base_sampled(sm):
    wl = WORKLOADS["base"]
    inp = make_inputs(wl)
    dout = make_dout(wl)
    idx2, dev = run_backward_top2(sm, wl, inp, dout, b_r=inp.b_r, to_host=False)
    T, N = wl.T, wl.n_experts
    r = orc.router_top2(inp.x, inp.w_r, inp.b_r)
    check_top2_routing(idx2, r)
    C = orc.capacity(2 * T, N, wl.capacity_factor)
    dsp = orc.dispatch_top2(idx2, N, C)
    p = r["probs"]
    gate2 = np.stack([p[np.arange(T), idx2[0]], p[np.arange(T), idx2[1]]])
    counts1 = np.bincount(idx2[0], minlength=N)
    f_scale = wl.alpha * N * counts1 / T / T
    drop2 = dsp["drop"]
    rng = np.random.default_rng(5)
    one = np.nonzero(drop2[1] & ~drop2[0])[0]
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 40, replace=False),
                                     rng.choice(one, min(8, one.size), replace=False)]))
    dg = np.zeros((2, toks.size))
    dxe = np.zeros((toks.size, wl.d_model))
    allow_dx = np.zeros((toks.size, wl.d_model))
    for rr in range(2):
        kept_j = np.nonzero(~drop2[rr, toks])[0]
        for e in np.unique(idx2[rr, toks[kept_j]]):
            js = kept_j[idx2[rr, toks[kept_j]] == e]
            ts = toks[js]
            dg_a, dxe_a, _, _ = orc.expert_backward(inp.x[ts], inp.w1[e], inp.w2[e],
                                                    gate2[rr, ts], dout[ts])
            dg[rr, js] = dg_a
            dxe[js] += dxe_a
            allow_dx[js] += relu_ambiguity(inp.x[ts], inp.w1[e], inp.w2[e], gate2[rr, ts],
                                           dout[ts])[1]
    w_r64 = inp.w_r.astype(np.float64)
    want_dx = np.zeros((toks.size, wl.d_model))
    for j, t in enumerate(toks):
        dp = f_scale.copy()
        for rr in range(2):
            if not drop2[rr, t]:
                dp[int(idx2[rr, t])] += dg[rr, j]
        dh = p[t] * (dp - np.sum(p[t] * dp))
        want_dx[j] = as_f64(dout[t]) + dxe[j] + dh @ w_r64
    tsel = torch.from_numpy(toks).cuda()
    grad_ok(host_f64(dev["dx"][tsel]), want_dx, "dx (sampled)", allow_dx)
    got_dg = host_f64(dev["dgate"].reshape(2, -1)[:, tsel])
    grad_ok(got_dg, dg, "dgate (sampled)")
    for e in (0, N // 2, N - 1):
        n = min(int(dsp["counts"][e]), C)
        g1, g2 = host_f64(dev["dw1"][e]), host_f64(dev["dw2"][e])
        if n == 0:
            assert np.all(g1 == 0) and np.all(g2 == 0)
            continue
        rows = dsp["slot_token"][e * C: e * C + n]
        route = np.where(idx2[0, rows] == e, 0, 1)
        g = gate2[route, rows]
        _, _, dw1_e, dw2_e = orc.expert_backward(inp.x[rows], inp.w1[e], inp.w2[e], g,
                                                 dout[rows])
        allow_w1 = relu_ambiguity(inp.x[rows], inp.w1[e], inp.w2[e], g, dout[rows])[0]
        grad_ok(g1, dw1_e, f"dw1[{e}]", allow_w1)
        grad_ok(g2, dw2_e, f"dw2[{e}]")
    dw_r = host_f64(dev["dw_r"])
    assert np.abs(dw_r.sum(axis=0)).max() <= 1e-3 * np.abs(dw_r).max()
    for k in ("dx", "dw1", "dw2"):
        assert bool(torch.isfinite(dev[k]).all()), k
