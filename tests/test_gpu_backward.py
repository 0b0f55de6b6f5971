"""Parity of switch_layer_backward against the oracle's backward pass.

The oracle is re-based on the GPU's top-1 choices (read from a forward call
on the same inputs; the backward recomputes the same routing), then every
gradient is compared element by element: bf16 dx, dw1, dw2 and the fp32
router gradients dw_r, db_r and the gate gradient, each with two bounds
relative to RMS(oracle):  max |GPU - oracle| <= 4e-2 and RMS(GPU - oracle)
<= 5e-3.  Derivation: a gradient element passes through up to three bf16
roundings (gate * dout, dA, and the bf16 output itself; H adds a fourth on
the dW2 / gate-gradient path), each a relative error of at most 2^-9, while
the fp32 accumulations add < 1e-5.  A sum of n independently rounded terms
then has an error of standard deviation about 3 * 2^-9 / sqrt(3) = 3.4e-3 of
its RMS; over 10^6 elements the largest is about 6 standard deviations
(0.02), plus the output's own rounding of at most 2^-9 x the largest value
(about 5 RMS, 0.01): 0.03, bounded by 4e-2.  The RMS bound (1.5 x the
standard deviation) is what catches a wrong index or a missing term: those
give errors of the order of the RMS itself.  The router's fp32 gradients
inherit bf16-level error through the gate gradient.  Routing flips (oracle
margin < 1e-6) are counted as in the forward tests.

At full size (Base, the Zipf-skewed workload with 60% drops, Large and XXL)
the oracle computes sampled tokens' dx and gate gradients, and sampled
experts' weight gradients, one by one; dw_r and db_r
are checked there through the softmax shift invariance (their sums over
experts vanish), which holds at any size.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import Workload, WORKLOADS, make_inputs, make_dout, as_f64
from gpu_util import dev_float, host_f64, check_routing

pytestmark = pytest.mark.gpu

GRAD_MAX_TOL = 4e-2
GRAD_RMS_TOL = 5e-3


# ReLU decisions near the kink: the GPU takes relu'(A) from its fp32
# accumulation of A, the oracle from float64; where |A| is below the fp32
# accumulation error both choices are correct.  A hidden unit counts as
# ambiguous when |A| < RELU_TAU * sum_k |x_k w_k| (about 17 units in the last
# place of the sum's L1 mass, an order of magnitude above the expected
# accumulation error); its whole contribution dH * x (to dW1) or dH * W1 (to
# dx) is allowed on top of the tolerance.  The RMS bound is not relaxed.
RELU_TAU = 1e-6


def relu_ambiguity(x_rows, w1_e, w2_e, g_rows, dout_rows):
    """Per-element allowances for dW1_e [F, d] and for the rows' dx [n, d]."""
    X, W1, W2 = as_f64(x_rows), as_f64(w1_e), as_f64(w2_e)
    A = X @ W1.T
    amb = np.abs(A) < RELU_TAU * (np.abs(X) @ np.abs(W1).T)
    dH = np.asarray(g_rows, np.float64)[:, None] * (as_f64(dout_rows) @ W2)
    contrib = np.abs(dH) * amb
    return contrib.T @ np.abs(X), contrib @ np.abs(W1), int(amb.sum())


def grad_ok(got, want, name, allow=None):
    want = np.asarray(want, np.float64)
    err = np.asarray(got, np.float64) - want
    rms = max(float(np.sqrt(np.mean(want * want))), 1e-30)
    excess = np.abs(err) if allow is None else np.maximum(np.abs(err) - allow, 0.0)
    mx = float(np.max(excess)) / rms
    rm = float(np.sqrt(np.mean(err * err))) / rms
    assert mx <= GRAD_MAX_TOL and rm <= GRAD_RMS_TOL, \
        f"{name}: max err / rms = {mx:.3g}, rms err / rms = {rm:.3g}"
    return mx, rm


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _forward_idx(sm, cfg, x, w_r, b_r, w1, w2, ws):
    out = torch.empty_like(x)
    idx = torch.empty(cfg.T, dtype=torch.int32, device="cuda")
    sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx, None, None, None, ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"
    return idx.cpu().numpy().astype(np.int64)


def run_backward(sm, wl, inp, dout, dloss=1.0, flags=0, b_r_override=None, reuse_ws=None,
                 to_host=True):
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                    dtype=wl.dtype, alpha=wl.alpha, flags=flags)
    ws = sm.backward_workspace(cfg) if reuse_ws is None else reuse_ws
    b_np = inp.b_r if b_r_override is None else b_r_override
    x, w_r, w1, w2 = dev_float(inp.x), dev_float(inp.w_r), dev_float(inp.w1), dev_float(inp.w2)
    b_r = None if b_np is None else dev_float(b_np)
    g = dev_float(dout)
    idx = _forward_idx(sm, cfg, x, w_r, b_r, w1, w2, ws)
    dx = torch.full_like(x, float("nan"))
    dw_r = torch.full_like(w_r, float("nan"))
    db_r = torch.full((wl.n_experts,), float("nan"), device="cuda")
    dw1 = torch.full_like(w1, float("nan"))
    dw2 = torch.full_like(w2, float("nan"))
    dgate = torch.full((wl.T,), float("nan"), device="cuda")
    sm.switch_layer_backward(cfg, x, w_r, b_r, w1, w2, g, dloss, dx, dw_r, db_r, dw1, dw2,
                             dgate, ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"
    res = {"dx": dx, "dw_r": dw_r, "db_r": db_r, "dw1": dw1, "dw2": dw2, "dgate": dgate}
    if to_host:
        res = {k: host_f64(v) for k, v in res.items()}
    return idx, res


def check_backward(sm, wl, dloss=1.0, flags=0, b_r_override=None):
    inp = make_inputs(wl)
    dout = make_dout(wl)
    idx, got = run_backward(sm, wl, inp, dout, dloss, flags, b_r_override)
    b_np = inp.b_r if b_r_override is None else b_r_override
    r = orc.router(inp.x, inp.w_r, b_np)
    flips = check_routing(idx, r)
    residual = not (flags & sm.FLAG_NO_RESIDUAL)
    want = orc.layer_backward(inp.x, inp.w_r, b_np, inp.w1, inp.w2, wl.capacity_factor, dout,
                              dloss=dloss, alpha=wl.alpha, residual=residual, idx=idx)
    for name in ("dx", "dw1", "dw2", "dw_r", "dgate"):
        assert np.isfinite(got[name]).all(), name
        print(wl.name, name, "max/rms err ratios %.3g %.3g" % grad_ok(got[name], want[name], name))
    if b_np is not None:
        grad_ok(got["db_r"], want["db_r"], "db_r")
    return got, want, flips


SMALL = Workload("bwd_small", T=3000, d_model=320, d_ff=576, n_experts=8, capacity_factor=1.0,
                 dtype="bf16", seed=91)


def test_backward_small(sm):
    got, want, _ = check_backward(sm, SMALL)
    d = want["drop"]
    assert d.any() and (~d).any()
    assert np.all(got["dgate"][d] == 0)


@pytest.mark.parametrize("flags", [0, 1, 16, 64], ids=["default", "simt_router", "no_residual",
                                                      "gemm1_pairs"])
def test_backward_flags(sm, flags):
    check_backward(sm, SMALL, dloss=0.5, flags=flags)


def test_backward_bias_and_loss_only(sm):
    """Router bias present; dloss = 3 weights the loss's gradient up."""
    rng = np.random.default_rng(5)
    bias = (0.05 * rng.standard_normal(SMALL.n_experts)).astype(np.float32)
    check_backward(sm, SMALL, dloss=3.0, b_r_override=bias)


def test_backward_empty_expert_and_heavy_drop(sm):
    """An expert no token picks has exactly zero weight gradients; with a
    capacity factor of 0.25 most tokens are dropped."""
    wl = Workload("bwd_drop", T=2048, d_model=256, d_ff=512, n_experts=8,
                  capacity_factor=0.25, dtype="bf16", seed=17)
    bias = np.zeros(wl.n_experts, dtype=np.float32)
    bias[3] = -60.0
    got, want, _ = check_backward(sm, wl, b_r_override=bias)
    assert np.all(got["dw1"][3] == 0) and np.all(got["dw2"][3] == 0)
    assert want["drop"].mean() > 0.5


def test_backward_no_drops_ragged(sm):
    """Every token kept (capacity factor N); sizes whose tiles are ragged in
    every dimension (C, d_model and d_ff not multiples of the tile)."""
    wl = Workload("bwd_ragged", T=1000, d_model=192, d_ff=320, n_experts=6,
                  capacity_factor=6.0, dtype="bf16", seed=23)
    got, want, _ = check_backward(sm, wl)
    assert not want["drop"].any()


def test_backward_single_expert_and_tiny_batch(sm):
    """N = 1 (p = 1: the router's gradients vanish, the layer is a dense
    residual FFN) and a batch smaller than one tile."""
    for wl in (Workload("bwd_dense", T=700, d_model=192, d_ff=320, n_experts=1,
                        capacity_factor=1.0, dtype="bf16", seed=31),
               Workload("bwd_tiny", T=37, d_model=64, d_ff=128, n_experts=4,
                        capacity_factor=1.0, dtype="bf16", seed=37)):
        got, want, _ = check_backward(sm, wl)
        if wl.n_experts == 1:
            assert np.all(got["dw_r"] == 0) and not want["drop"].any()


def test_backward_many_experts(sm):
    """N = 100: the router's bf16 planes are padded to 128 columns."""
    wl = Workload("bwd_n100", T=2500, d_model=128, d_ff=192, n_experts=100,
                  capacity_factor=1.0, dtype="bf16", seed=29)
    check_backward(sm, wl, dloss=2.0)


def test_backward_wide_router(sm):
    """N = 300: the tensor-core router with several weight tiles, planes padded
    to 320 columns, five extra K blocks per term in the dX GEMM.  About 40
    kept tokens per expert, so that a weight gradient is a sum of as many
    terms as the tolerance's derivation assumes (with ~10 its error tail is
    heavier)."""
    wl = Workload("bwd_n300", T=12000, d_model=128, d_ff=128, n_experts=300,
                  capacity_factor=1.5, dtype="bf16", seed=33)
    check_backward(sm, wl, dloss=1.5)


def _forward_all(sm, cfg, dev, ws):
    x, w_r, b_r, w1, w2 = dev
    out = torch.empty_like(x)
    idx = torch.empty(cfg.T, dtype=torch.int32, device="cuda")
    gate = torch.empty(cfg.T, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx, gate, counts, loss, ws)
    return [t.cpu() for t in (out, idx, gate, counts, loss)]


def _backward_all(sm, cfg, dev, g, ws):
    x, w_r, b_r, w1, w2 = dev
    outs = [torch.empty_like(x), torch.empty_like(w_r),
            torch.empty(cfg.n_experts, device="cuda"), torch.empty_like(w1),
            torch.empty_like(w2), torch.empty(cfg.T, device="cuda")]
    dx, dw_r, db_r, dw1, dw2, dgate = outs
    sm.switch_layer_backward(cfg, x, w_r, b_r, w1, w2, g, 1.0, dx, dw_r, db_r, dw1, dw2, dgate,
                             ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"
    return [t.cpu() for t in outs]


@pytest.mark.parametrize("flags", [0, 8, 1], ids=["default", "gather_in_gemm", "simt_router"])
def test_backward_saved_forward_state(sm, flags):
    """SWITCH_FLAG_TRAINING: the forward keeps probabilities, routing, x_disp
    and H; the backward reads them instead of recomputing.  The forward's
    outputs and every gradient equal, bit for bit, those of the plain forward
    and the recomputing backward, and a second backward call repeats them."""
    wl = SMALL
    inp = make_inputs(wl)
    rng = np.random.default_rng(2)
    bias = (0.05 * rng.standard_normal(wl.n_experts)).astype(np.float32)
    dev = (dev_float(inp.x), dev_float(inp.w_r), dev_float(bias), dev_float(inp.w1),
           dev_float(inp.w2))
    g = dev_float(make_dout(wl))
    mk = lambda f: sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts,  # noqa: E731
                             wl.capacity_factor, alpha=wl.alpha, flags=f)
    cfg0, cfg1 = mk(flags), mk(flags | sm.FLAG_TRAINING)
    ws0 = sm.backward_workspace(cfg0)
    f0 = _forward_all(sm, cfg0, dev, ws0)
    b0 = _backward_all(sm, cfg0, dev, g, ws0)
    ws1 = sm.backward_workspace(cfg1)
    f1 = _forward_all(sm, cfg1, dev, ws1)
    b1 = _backward_all(sm, cfg1, dev, g, ws1)
    b2 = _backward_all(sm, cfg1, dev, g, ws1)
    for a, b in zip(f0, f1):
        assert torch.equal(a, b)
    for a, b, c in zip(b0, b1, b2):
        assert torch.equal(a, b) and torch.equal(b, c)
    # the forward's state needs the backward's workspace size
    small = sm.workspace(cfg1)
    with pytest.raises(sm.SwitchError) as ei:
        _forward_all(sm, cfg1, dev, small)
    assert ei.value.status == 3


def test_backward_deterministic(sm):
    inp = make_inputs(SMALL)
    dout = make_dout(SMALL)
    _, a = run_backward(sm, SMALL, inp, dout)
    _, b = run_backward(sm, SMALL, inp, dout)
    for k in a:
        assert np.array_equal(a[k], b[k], equal_nan=True), k


def test_backward_rejects_misaligned_arguments(sm):
    """A pointer that is not 16-byte aligned is refused before any launch
    (both dtypes); nothing is written."""
    wl = SMALL
    for dtype in ("bf16", "f32"):
        cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                        dtype=dtype, alpha=wl.alpha)
        ws = sm.backward_workspace(cfg)
        t = torch.zeros(64, device="cuda")
        with pytest.raises(sm.SwitchError) as ei:
            sm.switch_layer_backward(cfg, t[1:], t, None, t, t, t, 1.0, t, t, None, t, t, None,
                                     ws)
        assert ei.value.status == 1


def test_backward_workspace_too_small(sm):
    wl = SMALL
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor, alpha=wl.alpha)
    ws = sm.workspace(cfg)                      # the forward's size only
    assert sm.switch_backward_workspace_size(cfg) > ws.numel()
    x = torch.zeros(wl.T, wl.d_model, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_layer_backward(cfg, x, x, None, x, x, x, 1.0, x, x, None, x, x, None, ws)
    assert ei.value.status == 3


# ----------------------------------------------------------- full size

@pytest.mark.parametrize("name", ["base", "zipf_cf1.0", "large", "xxl"])
def test_backward_fullsize_sampled(sm, name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    dout = make_dout(wl)
    idx, dev = run_backward(sm, wl, inp, dout, to_host=False)    # weights' gradients stay on the GPU
    T, N = wl.T, wl.n_experts
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    check_routing(idx, r)
    C = orc.capacity(T, N, wl.capacity_factor)
    dsp = orc.dispatch(idx, N, C)
    gate = r["probs"][np.arange(T), idx]
    f_scale = wl.alpha * N * dsp["counts"] / T / T
    rng = np.random.default_rng(3)
    dropped = np.nonzero(dsp["drop"])[0]
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 48, replace=False),
                                     rng.choice(dropped, min(8, dropped.size), replace=False)]))
    want_dx = np.zeros((toks.size, wl.d_model))
    want_dg = np.zeros(toks.size)
    dxe = np.zeros((toks.size, wl.d_model))
    allow_dx = np.zeros((toks.size, wl.d_model))
    kept_j = np.nonzero(~dsp["drop"][toks])[0]
    for e in np.unique(idx[toks[kept_j]]):          # one oracle call per expert
        js = kept_j[idx[toks[kept_j]] == e]
        ts = toks[js]
        dg_a, dxe_a, _, _ = orc.expert_backward(inp.x[ts], inp.w1[e], inp.w2[e], gate[ts],
                                                dout[ts])
        want_dg[js] = dg_a
        dxe[js] = dxe_a
        allow_dx[js] = relu_ambiguity(inp.x[ts], inp.w1[e], inp.w2[e], gate[ts], dout[ts])[1]
    w_r64 = inp.w_r.astype(np.float64)
    for j, t in enumerate(toks):
        p = r["probs"][t]
        dp = f_scale.copy()
        if not dsp["drop"][t]:
            dp[int(idx[t])] += want_dg[j]
        dh = p * (dp - np.sum(p * dp))
        want_dx[j] = as_f64(dout[t]) + dxe[j] + dh @ w_r64
    tsel = torch.from_numpy(toks).cuda()
    grad_ok(host_f64(dev["dx"][tsel]), want_dx, "dx (sampled)", allow_dx)
    grad_ok(host_f64(dev["dgate"][tsel]), want_dg, "dgate (sampled)")
    for e in (0, N // 2, N - 1):
        n = min(int(dsp["counts"][e]), C)
        g1, g2 = host_f64(dev["dw1"][e]), host_f64(dev["dw2"][e])
        if n == 0:
            assert np.all(g1 == 0) and np.all(g2 == 0)
            continue
        rows = dsp["slot_token"][e * C: e * C + n]
        _, _, dw1_e, dw2_e = orc.expert_backward(inp.x[rows], inp.w1[e], inp.w2[e], gate[rows],
                                                 dout[rows])
        allow_w1, _, n_amb = relu_ambiguity(inp.x[rows], inp.w1[e], inp.w2[e], gate[rows],
                                            dout[rows])
        print(name, f"expert {e}: {n_amb} hidden units within the ReLU decision margin")
        grad_ok(g1, dw1_e, f"dw1[{e}]", allow_w1)
        grad_ok(g2, dw2_e, f"dw2[{e}]")
    # softmax shift invariance: sum over experts of dW_r rows and of db_r vanish
    dw_r = host_f64(dev["dw_r"])
    scale = np.abs(dw_r).max()
    assert np.abs(dw_r.sum(axis=0)).max() <= 1e-3 * scale
    for k in ("dx", "dw1", "dw2"):
        assert bool(torch.isfinite(dev[k]).all()), k
