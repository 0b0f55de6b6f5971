"""Pins for the oracle's backward pass (``layer_backward`` and its two steps).

Each check ties the gradient to something other than its own formulas:

* central finite differences of the forward oracle's objective
  J = sum(dout * out) + dloss * loss, in float64, on tiny inputs whose routing
  margins and ReLU pre-activations keep every decision away from its switching
  point (so J is smooth there);
* the shift invariance of the softmax gate ("Switch Transformers: scaling to
  trillion-parameter models", section "Switch Routing: From Top-k to k = 1",
  gate equation): adding one vector to every row of W_r changes no
  probability, so the rows of dW_r sum to zero and so does db_r;
* a dropped token with no loss gradient: its block output is x alone
  (section "Expert Capacity and the Capacity Factor"), so dx = dout exactly;
* one expert with room for every token: p = 1, the layer is x + FFN(x), and
  the weight gradients equal torch autograd's for a dense ReLU MLP;
* top-2 (section "Switch Routing: From Top-k to k = 1", the top-k set and its
  gates): finite differences of the top-2 forward oracle, and with two
  experts and no drops the gates sum to 1, so the logits' gradients are
  opposite for every token.

The last test plants plausible mistakes in the backward (on the CPU) and
checks that some pin catches each one.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc

ALPHA = 0.01


def _case(seed, T=10, d=4, F=6, N=3, cf=1.0, bias=True):
    """Random float64 inputs whose decisions sit far from their kinks."""
    for s in range(seed, seed + 500):
        rng = np.random.default_rng(s)
        x = rng.standard_normal((T, d))
        w_r = rng.standard_normal((N, d))
        b_r = 0.3 * rng.standard_normal(N) if bias else None
        w1 = rng.standard_normal((N, F, d)) / np.sqrt(d)
        w2 = rng.standard_normal((N, d, F)) / np.sqrt(F)
        dout = rng.standard_normal((T, d))
        h = x @ w_r.T + (0 if b_r is None else b_r)
        hs = np.sort(h, axis=1)
        if N > 1 and np.min(hs[:, -1] - hs[:, -2]) < 1e-2:
            continue
        if np.min(np.abs(np.einsum("td,nfd->tnf", x, w1))) < 1e-3:
            continue
        C = orc.capacity(T, N, cf)
        if N > 1 and np.bincount(np.argmax(h, axis=1), minlength=N).max() <= C:
            continue                       # want some dropped tokens
        return x, w_r, b_r, w1, w2, dout
    raise RuntimeError("no smooth case found")


def _objective(O, x, w_r, b_r, w1, w2, cf, dout, dloss, residual):
    f = O.layer_forward(x, w_r, b_r, w1, w2, cf, alpha=ALPHA, residual=residual)
    return float(np.sum(dout * f["out"]) + dloss * f["loss"])


def _fd_grad(fun, a, eps=1e-6):
    g = np.zeros_like(a)
    it = np.nditer(a, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = a[i]
        a[i] = old + eps
        jp = fun()
        a[i] = old - eps
        jm = fun()
        a[i] = old
        g[i] = (jp - jm) / (2 * eps)
    return g


def _check_fd(O, seed, cf, dloss, residual, N=3):
    x, w_r, b_r, w1, w2, dout = _case(seed, N=N, cf=cf)
    got = O.layer_backward(x, w_r, b_r, w1, w2, cf, dout, dloss=dloss, alpha=ALPHA,
                           residual=residual)
    fun = lambda: _objective(O, x, w_r, b_r, w1, w2, cf, dout, dloss, residual)  # noqa: E731
    for name, arr in (("dx", x), ("dw_r", w_r), ("db_r", b_r), ("dw1", w1), ("dw2", w2)):
        want = _fd_grad(fun, arr)
        np.testing.assert_allclose(got[name], want, rtol=1e-6, atol=1e-8, err_msg=name)
    return got


# ------------------------------------------------------------------- pins

def pin_bwd_finite_differences(O):
    got = _check_fd(O, 11, cf=1.0, dloss=1.0, residual=True)
    assert got["drop"].any() and (~got["drop"]).any()     # both kinds of token covered


def pin_bwd_finite_differences_no_residual(O):
    _check_fd(O, 23, cf=0.75, dloss=3.0, residual=False)


def pin_bwd_loss_only(O):
    """dout = 0: the gradient is the loss's alone (P_i through the softmax)."""
    x, w_r, b_r, w1, w2, _ = _case(5)
    dout = np.zeros_like(x)
    got = O.layer_backward(x, w_r, b_r, w1, w2, 1.0, dout, dloss=2.0, alpha=ALPHA)
    fun = lambda: _objective(O, x, w_r, b_r, w1, w2, 1.0, dout, 2.0, True)  # noqa: E731
    np.testing.assert_allclose(got["dw_r"], _fd_grad(fun, w_r), rtol=1e-6, atol=1e-9)
    assert np.all(got["dw1"] == 0) and np.all(got["dw2"] == 0)


def pin_bwd_softmax_shift(O):
    x, w_r, b_r, w1, w2, dout = _case(31, T=40, N=5)
    got = O.layer_backward(x, w_r, b_r, w1, w2, 1.25, dout, dloss=1.0, alpha=ALPHA)
    scale = np.abs(got["dw_r"]).max()
    assert np.abs(got["dw_r"].sum(axis=0)).max() <= 1e-12 * max(scale, 1.0)
    assert abs(got["db_r"].sum()) <= 1e-12 * max(np.abs(got["db_r"]).max(), 1.0)
    assert np.abs(got["dh"].sum(axis=1)).max() <= 1e-12


def pin_bwd_dropped_passthrough(O):
    x, w_r, b_r, w1, w2, dout = _case(41, T=30, N=3)
    got = O.layer_backward(x, w_r, b_r, w1, w2, 0.5, dout, dloss=0.0, alpha=ALPHA)
    d = got["drop"]
    assert d.any()
    np.testing.assert_array_equal(got["dx"][d], dout[d])
    assert np.all(got["dgate"][d] == 0)


def pin_bwd_single_expert_dense(O):
    """N = 1, capacity for all: p = 1 (no router gradient), out = x + FFN(x)."""
    x, w_r, b_r, w1, w2, dout = _case(53, T=16, d=6, F=10, N=1)
    got = O.layer_backward(x, w_r, b_r, w1, w2, 1.0, dout, dloss=1.0, alpha=ALPHA)
    assert not got["drop"].any()
    assert np.all(got["dw_r"] == 0) and np.all(got["db_r"] == 0)
    X = torch.tensor(x, requires_grad=True)
    W1 = torch.tensor(w1[0], requires_grad=True)
    W2 = torch.tensor(w2[0], requires_grad=True)
    out = X + torch.nn.functional.linear(torch.relu(torch.nn.functional.linear(X, W1)), W2)
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(got["dw1"][0], W1.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dw2"][0], W2.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dx"], X.grad.numpy(), rtol=1e-12, atol=1e-12)


def _case_top2(seed, T=12, d=4, F=6, N=4, cf=0.5):
    """Like _case for top-2: first/second and second/third logit margins and
    ReLU pre-activations away from their switching points, drops present."""
    for s_ in range(seed, seed + 2000):
        rng = np.random.default_rng(s_)
        x = rng.standard_normal((T, d))
        w_r = rng.standard_normal((N, d))
        b_r = 0.3 * rng.standard_normal(N)
        w1 = rng.standard_normal((N, F, d)) / np.sqrt(d)
        w2 = rng.standard_normal((N, d, F)) / np.sqrt(F)
        dout = rng.standard_normal((T, d))
        hs = np.sort(x @ w_r.T + b_r, axis=1)
        if np.min(hs[:, -1] - hs[:, -2]) < 1e-2 or np.min(hs[:, -2] - hs[:, -3]) < 1e-2:
            continue
        if np.min(np.abs(np.einsum("td,nfd->tnf", x, w1))) < 1e-3:
            continue
        r = orc.router_top2(x, w_r, b_r)
        dsp = orc.dispatch_top2(r["idx2"], N, orc.capacity(2 * T, N, cf))
        if not dsp["drop"][0].any() and not dsp["drop"][1].any():
            continue
        return x, w_r, b_r, w1, w2, dout
    raise RuntimeError("no smooth top-2 case found")


def pin_bwd_top2_finite_differences(O):
    x, w_r, b_r, w1, w2, dout = _case_top2(7)
    cf = 0.5
    got = O.layer_backward_top2(x, w_r, b_r, w1, w2, cf, dout, dloss=2.0, alpha=ALPHA)

    def fun():
        f = O.layer_forward_top2(x, w_r, b_r, w1, w2, cf, alpha=ALPHA)
        return float(np.sum(dout * f["out"]) + 2.0 * f["loss"])

    for name, arr in (("dx", x), ("dw_r", w_r), ("db_r", b_r), ("dw1", w1), ("dw2", w2)):
        np.testing.assert_allclose(got[name], _fd_grad(fun, arr), rtol=1e-6, atol=1e-8,
                                   err_msg=name)
    assert got["drop2"][1].any()           # some second routes dropped


def pin_bwd_top2_two_experts_gates_sum(O):
    """N = 2, room for every assignment: both experts take every token and the
    two gates sum to 1, so the gate gradients enter only through their
    difference (dh_0 = -dh_1 for every token)."""
    x, w_r, b_r, w1, w2, dout = _case(61, T=8, N=2)
    got = O.layer_backward_top2(x, w_r, b_r, w1, w2, 4.0, dout, dloss=0.0, alpha=ALPHA)
    assert not got["drop2"].any()
    np.testing.assert_allclose(got["dh"][:, 0], -got["dh"][:, 1], rtol=0, atol=1e-14)


PINS = [pin_bwd_finite_differences, pin_bwd_finite_differences_no_residual,
        pin_bwd_loss_only, pin_bwd_softmax_shift, pin_bwd_dropped_passthrough,
        pin_bwd_single_expert_dense, pin_bwd_top2_finite_differences,
        pin_bwd_top2_two_experts_gates_sum]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(orc)


# ------------------------------------------------- planted mistakes (CPU)

def _mut_no_relu_mask(real):
    def f(x_rows, w1_e, w2_e, g_rows, dout_rows):
        from switch_inputs import as_f64
        X, W1, W2, G = as_f64(x_rows), as_f64(w1_e), as_f64(w2_e), as_f64(dout_rows)
        g = np.asarray(g_rows, np.float64)
        A = X @ W1.T
        H = np.maximum(A, 0.0)
        dY = g[:, None] * G
        dA = dY @ W2                                   # mask forgotten
        return np.sum(G * (H @ W2.T), axis=1), dA @ W1, dA.T @ X, dY.T @ H
    return f


def _mut_no_gate_scale(real):
    def f(x_rows, w1_e, w2_e, g_rows, dout_rows):
        return real(x_rows, w1_e, w2_e, np.ones_like(np.asarray(g_rows, np.float64)), dout_rows)
    return f


def _mut_dgate_of_hidden(real):
    def f(x_rows, w1_e, w2_e, g_rows, dout_rows):
        dg, dx, dw1, dw2 = real(x_rows, w1_e, w2_e, g_rows, dout_rows)
        return 0.5 * dg, dx, dw1, dw2
    return f


def _mut_softmax_no_centering(real):
    def f(x, w_r, probs, idx, drop, dgate, counts, alpha, dloss):
        from switch_inputs import as_f64
        p = np.asarray(probs, np.float64)
        T, N = p.shape
        dp = np.tile(dloss * alpha * N * np.asarray(counts, np.float64) / T / T, (T, 1))
        rows = np.nonzero(~np.asarray(drop, bool))[0]
        dp[rows, np.asarray(idx)[rows]] += np.asarray(dgate)[rows]
        dh = p * dp                                    # - sum_j p_j dp_j forgotten
        Wr = np.asarray(w_r, np.float64)
        return dh @ Wr, dh.T @ as_f64(x), dh.sum(axis=0), dh
    return f


def _mut_no_loss_term(real):
    def f(x, w_r, probs, idx, drop, dgate, counts, alpha, dloss):
        return real(x, w_r, probs, idx, drop, dgate, counts, alpha, 0.0)
    return f


def _mut_loss_without_N(real):
    def f(x, w_r, probs, idx, drop, dgate, counts, alpha, dloss):
        N = np.shape(probs)[1]
        return real(x, w_r, probs, idx, drop, dgate, counts, alpha / N, dloss)
    return f


def _mut_dropped_get_gate_grad(real):
    def f(x, w_r, probs, idx, drop, dgate, counts, alpha, dloss):
        T = np.shape(probs)[0]
        fake = np.asarray(dgate, np.float64) + 0.25 * np.asarray(drop, bool)
        return real(x, w_r, probs, idx, np.zeros(T, bool), fake, counts, alpha, dloss)
    return f


def _mut_top2_first_route_only(real):
    def f(x, w_r, probs, idx2, drop2, dgate2, counts1, alpha, dloss):
        d2 = np.asarray(dgate2, np.float64).copy()
        d2[1] = 0.0                                    # second gate's gradient lost
        return real(x, w_r, probs, idx2, drop2, d2, counts1, alpha, dloss)
    return f


def _mut_top2_f_over_both_routes(real):
    def f(x, w_r, probs, idx2, drop2, dgate2, counts1, alpha, dloss):
        N = np.shape(probs)[1]
        both = np.bincount(np.asarray(idx2).reshape(-1), minlength=N)
        return real(x, w_r, probs, idx2, drop2, dgate2, both, alpha, dloss)
    return f


MUTANTS = {
    "top2_second_gate_gradient_lost": ("router_backward_top2", _mut_top2_first_route_only),
    "top2_loss_f_over_both_routes": ("router_backward_top2", _mut_top2_f_over_both_routes),
    "relu_mask_forgotten": ("expert_backward", _mut_no_relu_mask),
    "gate_not_scaling_dY": ("expert_backward", _mut_no_gate_scale),
    "dgate_halved": ("expert_backward", _mut_dgate_of_hidden),
    "softmax_jacobian_uncentered": ("router_backward", _mut_softmax_no_centering),
    "loss_gradient_missing": ("router_backward", _mut_no_loss_term),
    "loss_gradient_without_N": ("router_backward", _mut_loss_without_N),
    "dropped_token_gate_gradient": ("router_backward", _mut_dropped_get_gate_grad),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, make = MUTANTS[name]
    monkeypatch.setattr(orc, attr, make(getattr(orc, attr)))
    caught = []
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, IndexError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
