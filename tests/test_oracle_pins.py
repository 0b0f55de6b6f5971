"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- hand-worked values from the pages' equations (tests/golden/), the
invariants the pages state, closed forms, and brute force on tiny inputs.

Pages cited: "Switch Transformers: scaling to trillion-parameter models"
(sections "Switch Routing: From Top-k to k = 1", "Expert Capacity and the
Capacity Factor", "The Load-Balancing Loss", "The Core Idea"); the top-2
pins follow the top-k set and combine of "Switch Routing".

The last test plants plausible mistakes in the oracle (on the CPU) and checks
that at least one pin catches each of them.
"""
import itertools
import math

import numpy as np
import pytest

import oracle.switch_oracle as orc
import golden_io

ALPHA = 0.01


# ---------------------------------------------------------------- helpers

def _logit_router_inputs(rows):
    """x = 0 and a per-token bias is impossible, so use x one-hot per distinct
    logit row: d = number of distinct rows, W_r[:, j] = ln(a) of row j."""
    distinct = []
    for r in rows:
        if r not in distinct:
            distinct.append(r)
    N = len(rows[0])
    d = len(distinct)
    w_r = np.zeros((N, d), dtype=np.float32)
    for j, r in enumerate(distinct):
        w_r[:, j] = np.log(np.asarray(r, dtype=np.float64)).astype(np.float32)
    x = np.zeros((len(rows), d), dtype=np.float32)
    for t, r in enumerate(rows):
        x[t, distinct.index(r)] = 1.0
    return x, w_r


def _assignment_inputs(idx, N):
    """x / W_r such that token t routes to idx[t]: one-hot x, W_r = 4 I."""
    T = len(idx)
    x = np.zeros((T, N), dtype=np.float32)
    x[np.arange(T), idx] = 1.0
    w_r = (4.0 * np.eye(N)).astype(np.float32)
    return x, w_r


# ------------------------------------------------------------------- pins

def pin_capacity(O):
    for T, N, cf, C in golden_io.capacity_cases():
        assert O.capacity(T, N, cf) == C, (T, N, cf, C)


def pin_softmax_hand(O):
    for a, p_frac, top in golden_io.softmax_cases():
        x, w_r = _logit_router_inputs([a, a])
        r = O.router(x, w_r)
        want = np.array([float(f) for f in p_frac])
        for t in range(2):
            np.testing.assert_allclose(r["probs"][t], want, rtol=3e-7, atol=0)
            assert r["idx"][t] == top
            assert abs(r["gate"][t] - want[top]) <= 3e-7 * want[top]
        # the same logits through the bias path (x = 0)
        xb = np.zeros((3, 5), dtype=np.float32)
        wb = np.ones((len(a), 5), dtype=np.float32)
        bb = np.log(np.asarray(a, dtype=np.float64)).astype(np.float32)
        rb = O.router(xb, wb, bb)
        np.testing.assert_allclose(rb["probs"], np.tile(want, (3, 1)),
                                   rtol=3e-7, atol=0)
        assert (rb["idx"] == top).all()


def pin_router_invariants(O):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 16)).astype(np.float32)
    w = rng.standard_normal((5, 16)).astype(np.float32)
    r = O.router(x, w)
    np.testing.assert_allclose(r["probs"].sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert (r["probs"] > 0).all()
    # argmax of p equals argmax of h (exp is increasing); gate = max p
    assert (r["idx"] == np.argmax(r["probs"], axis=1)).all()
    np.testing.assert_array_equal(r["gate"], r["probs"].max(axis=1))
    # N = 1: p == 1 exactly
    r1 = O.router(x, w[:1])
    assert (r1["probs"] == 1.0).all() and (r1["idx"] == 0).all()
    # W_r = 0: every logit ties, p = 1/N exactly, lowest index wins
    for N in (2, 4, 8):
        r0 = O.router(x, np.zeros((N, 16), np.float32))
        assert (r0["probs"] == 1.0 / N).all()
        assert (r0["idx"] == 0).all()


def pin_dispatch_hand(O):
    g = golden_io.dispatch_case()
    d = O.dispatch(np.array(g["idx"]), g["N"][0], g["C"][0])
    assert d["rank"].tolist() == g["rank"]
    assert d["drop"].astype(int).tolist() == g["drop"]
    assert d["counts"].tolist() == g["counts"]
    assert d["slot_token"].tolist() == g["slot_token"]


def _dispatch_by_groups(idx, N, C):
    """Independent characterisation: group tokens by expert with sorted(),
    keep the C earliest of each group."""
    T = len(idx)
    groups = {e: sorted(t for t in range(T) if idx[t] == e) for e in range(N)}
    rank = [groups[idx[t]].index(t) for t in range(T)]
    slots = []
    for e in range(N):
        kept = groups[e][:C]
        slots += kept + [-1] * (C - len(kept))
    return rank, [len(groups[e]) for e in range(N)], slots


def pin_dispatch_bruteforce(O):
    for N in (1, 2, 3):
        for T in range(0, 7 if N < 3 else 6):
            for C in (1, 2, 3):
                for idx in itertools.product(range(N), repeat=T):
                    d = O.dispatch(np.array(idx, dtype=np.int64), N, C)
                    rank, counts, slots = _dispatch_by_groups(idx, N, C)
                    assert d["rank"].tolist() == rank
                    assert d["drop"].tolist() == [r >= C for r in rank]
                    assert d["counts"].tolist() == counts
                    assert d["slot_token"].tolist() == slots


def pin_dispatch_via_router(O):
    """Assignments built through the router (one-hot x, W_r = 4 I)."""
    N, C = 3, 2
    for idx in itertools.product(range(N), repeat=5):
        x, w_r = _assignment_inputs(list(idx), N)
        r = O.router(x, w_r)
        assert r["idx"].tolist() == list(idx)
        d = O.dispatch(r["idx"], N, C)
        rank, counts, slots = _dispatch_by_groups(list(idx), N, C)
        assert d["slot_token"].tolist() == slots and d["counts"].tolist() == counts


def pin_aux_hand(O):
    for name, toks, f_want, P_want, loss_want in golden_io.aux_loss_cases():
        x, w_r = _logit_router_inputs(toks)
        r = O.router(x, w_r)
        N = w_r.shape[0]
        C = O.capacity(len(toks), N, 1.0)
        d = O.dispatch(r["idx"], N, C)
        loss, f, P = O.aux_loss(d["counts"], r["probs"], ALPHA)
        np.testing.assert_allclose(f, [float(v) for v in f_want], rtol=0, atol=0)
        np.testing.assert_allclose(P, [float(v) for v in P_want], rtol=3e-7)
        assert abs(loss - loss_want) <= 3e-7 * loss_want, (name, loss)


def pin_aux_uniform(O):
    """W_r = 0: f = (1, 0, ..., 0), P = 1/N, so loss = alpha exactly; the
    page's reason for the factor N (uniform routing gives sum f P = 1/N)."""
    rng = np.random.default_rng(3)
    for N in (2, 4, 16):
        x = rng.standard_normal((40, 8)).astype(np.float32)
        r = O.router(x, np.zeros((N, 8), np.float32))
        C = O.capacity(40, N, 1.0)
        d = O.dispatch(r["idx"], N, C)
        assert d["counts"][0] == 40 and d["counts"][1:].sum() == 0
        assert (~d["drop"]).sum() == C and d["drop"].sum() == 40 - C
        loss, f, P = O.aux_loss(d["counts"], r["probs"], ALPHA)
        assert loss == ALPHA
    # balanced hard routing (round robin): f = 1/N, loss = alpha * sum P = alpha
    N = 4
    idx = [t % N for t in range(32)]
    x, w_r = _assignment_inputs(idx, N)
    r = O.router(x, w_r)
    d = O.dispatch(r["idx"], N, O.capacity(32, N, 1.0))
    loss, f, P = O.aux_loss(d["counts"], r["probs"], ALPHA)
    np.testing.assert_allclose(f, 1.0 / N, rtol=0, atol=0)
    assert abs(loss - ALPHA) <= 1e-15


def _brute_dense(x, w1, w2):
    T, dm = x.shape
    F = w1.shape[0]
    out = [[float(x[t, c]) for c in range(dm)] for t in range(T)]
    for t in range(T):
        hid = []
        for j in range(F):
            a = 0.0
            for k in range(dm):
                a += float(x[t, k]) * float(w1[j, k])
            hid.append(a if a > 0.0 else 0.0)
        for c in range(dm):
            s = 0.0
            for j in range(F):
                s += hid[j] * float(w2[c, j])
            out[t][c] += s
    return np.array(out)


def pin_dense_reduction(O):
    """N = 1 and capacity factor >= 1: no drops, p = 1, the layer is the dense
    residual FFN out = x + relu(x W1^T) W2^T, checked against explicit loops."""
    rng = np.random.default_rng(11)
    T, dm, F = 6, 4, 5
    x = rng.standard_normal((T, dm)).astype(np.float32)
    w_r = rng.standard_normal((1, dm)).astype(np.float32)
    w1 = rng.standard_normal((1, F, dm)).astype(np.float32)
    w2 = rng.standard_normal((1, dm, F)).astype(np.float32)
    for cf in (1.0, 1.25, 2.0):
        res = O.layer_forward(x, w_r, None, w1, w2, cf, ALPHA)
        assert not res["drop"].any() and (res["gate"] == 1.0).all()
        np.testing.assert_allclose(res["out"], _brute_dense(x, w1[0], w2[0]),
                                   rtol=1e-12, atol=1e-12)
        assert res["loss"] == ALPHA


def pin_single_expert_signature(O):
    """k = 1: out - x = p_idx * E_idx(x) and no other expert contributes.
    Expert e maps every token to the signature 100 * (e + 1) * unit(e)."""
    rng = np.random.default_rng(5)
    N, dm, T = 3, 4, 30
    x = rng.standard_normal((T, dm)).astype(np.float32)
    x[:, 3] = 1.0
    w_r = rng.standard_normal((N, dm)).astype(np.float32)
    w1 = np.zeros((N, N, dm), np.float32)
    w2 = np.zeros((N, dm, N), np.float32)
    for e in range(N):
        w1[e, e, 3] = 1.0                 # hidden = unit(e)
        w2[e, e, e] = 100.0 * (e + 1)     # output = 100 (e+1) unit(e)
    res = O.layer_forward(x, w_r, None, w1, w2, 4.0, ALPHA)
    assert not res["drop"].any()
    delta = res["out"] - x.astype(np.float64)
    for t in range(T):
        e = res["idx"][t]
        want = np.zeros(dm)
        want[e] = res["gate"][t] * 100.0 * (e + 1)
        np.testing.assert_allclose(delta[t], want, rtol=1e-12, atol=1e-12)
        assert 0.0 < res["gate"][t] < 1.0


def pin_dropped_residual(O):
    """Dropped tokens: block output equals x bit for bit; kept ones differ."""
    rng = np.random.default_rng(9)
    T, dm, F, N = 40, 8, 16, 4
    x = rng.standard_normal((T, dm)).astype(np.float32)
    w_r = np.zeros((N, dm), np.float32)      # every token -> expert 0
    w1 = rng.standard_normal((N, F, dm)).astype(np.float32)
    w2 = rng.standard_normal((N, dm, F)).astype(np.float32)
    res = O.layer_forward(x, w_r, None, w1, w2, 0.5, ALPHA)   # C = 5
    assert res["C"] == 5 and res["drop"].sum() == T - 5
    assert res["slot_token"][:5].tolist() == [0, 1, 2, 3, 4]
    d = res["drop"]
    assert (res["out"][d] == x[d].astype(np.float64)).all()
    assert (res["out"][~d] != x[~d].astype(np.float64)).any(axis=1).all()
    # without the residual a dropped token gives 0
    res0 = O.layer_forward(x, w_r, None, w1, w2, 0.5, ALPHA, residual=False)
    assert (res0["out"][d] == 0.0).all()


def pin_relu_active(O):
    """Hidden pre-activations of both signs: the expert zeroes the negative
    ones (relu), checked on a one-token hand case: x = (1, -1),
    W1 = [[1, 0], [0, 1], [1, 1]] -> pre (1, -1, 0) -> hid (1, 0, 0);
    W2 = [[2, 3, 5], [7, 11, 13]] -> E(x) = (2, 7)."""
    x = np.array([[1.0, -1.0]], np.float32)
    w1 = np.array([[1, 0], [0, 1], [1, 1]], np.float32)
    w2 = np.array([[2, 3, 5], [7, 11, 13]], np.float32)
    np.testing.assert_array_equal(O.expert(x, w1, w2), [[2.0, 7.0]])


# ---------------------------------------------------------- top-2 pins

def pin_top2_router_hand(O):
    """Hand-worked top-2 sets and gates (tests/golden/top2_hand.txt)."""
    for a, gates, top in golden_io.top2_router_cases():
        x, w_r = _logit_router_inputs([a])
        r = O.router_top2(x, w_r)
        assert r["idx2"][:, 0].tolist() == top, (a, r["idx2"][:, 0])
        np.testing.assert_allclose(r["gate2"][:, 0], [float(g) for g in gates],
                                   rtol=1e-6, atol=0)


def pin_top2_router_invariants(O):
    """W_r = 0: all logits tie, every token takes experts (0, 1) with gates
    1/N each; on random inputs the two choices differ, the first gate is the
    k = 1 gate and the second is no larger than the first."""
    rng = np.random.default_rng(21)
    x = rng.standard_normal((50, 8)).astype(np.float32)
    for N in (2, 4, 8):
        r = O.router_top2(x, np.zeros((N, 8), np.float32))
        assert (r["idx2"][0] == 0).all() and (r["idx2"][1] == 1).all()
        np.testing.assert_allclose(r["gate2"], 1.0 / N, rtol=1e-12)
        w_r = rng.standard_normal((N, 8)).astype(np.float32)
        r = O.router_top2(x, w_r)
        r1 = O.router(x, w_r)
        assert (r["idx2"][0] != r["idx2"][1]).all()
        assert (r["idx2"][0] == r1["idx"]).all()
        assert (r["gate2"][1] <= r["gate2"][0]).all()
        # the second choice is the argmax of p with the first removed
        p = r1["probs"].copy()
        p[np.arange(50), r1["idx"]] = -1.0
        assert (np.argmax(p, axis=1) == r["idx2"][1]).all()


def pin_top2_dispatch_hand(O):
    g = golden_io.top2_dispatch_case()
    d = O.dispatch_top2(np.array([g["idx1"], g["idx2"]]), g["N"][0], g["C"][0])
    assert d["rank"].tolist() == [g["rank1"], g["rank2"]]
    assert d["drop"].astype(int).tolist() == [g["drop1"], g["drop2"]]
    assert d["counts"].tolist() == g["counts"]
    assert d["slot_token"].tolist() == g["slot_token"]


def pin_top2_dispatch_bruteforce(O):
    """Every (first, second) assignment of 3 tokens over 3 experts, C = 1..4:
    rank of assignment (r, t) = #{earlier assignments, first choices before
    second choices, each in batch order, with the same expert}."""
    N = 3
    pairs = [(a, b) for a in range(N) for b in range(N) if a != b]
    for choice in itertools.product(pairs, repeat=3):
        idx2 = np.array([[c[0] for c in choice], [c[1] for c in choice]])
        order = [(r, t) for r in range(2) for t in range(3)]
        for C in (1, 2, 3, 4):
            d = O.dispatch_top2(idx2, N, C)
            for i, (r, t) in enumerate(order):
                e = idx2[r, t]
                want = sum(1 for (r2, t2) in order[:i] if idx2[r2, t2] == e)
                assert d["rank"][r, t] == want and d["drop"][r, t] == (want >= C)
            assert d["counts"].tolist() == np.bincount(idx2.reshape(-1), minlength=N).tolist()


def pin_top2_dense_reduction(O):
    """N = 2 with two identical experts and capacity factor >= 1: both routes
    of every token are kept (C = T), the gates sum to 1, so the layer is the
    dense residual FFN out = x + relu(x W1^T) W2^T (explicit loops)."""
    rng = np.random.default_rng(31)
    T, dm, F = 5, 4, 3
    x = rng.standard_normal((T, dm)).astype(np.float32)
    w_r = rng.standard_normal((2, dm)).astype(np.float32)
    w1 = np.repeat(rng.standard_normal((1, F, dm)).astype(np.float32), 2, axis=0)
    w2 = np.repeat(rng.standard_normal((1, dm, F)).astype(np.float32), 2, axis=0)
    res = O.layer_forward_top2(x, w_r, None, w1, w2, 1.0, ALPHA)
    assert res["C"] == T and not res["drop2"].any()
    np.testing.assert_allclose(res["gate2"].sum(axis=0), 1.0, rtol=1e-12)
    np.testing.assert_allclose(res["out"], _brute_dense(x, w1[0], w2[0]), rtol=1e-10,
                               atol=1e-10)


def pin_top2_signature(O):
    """Each expert writes its own signature 100 (e + 1) unit(e): out - x holds
    exactly the two chosen experts' signatures scaled by their gates, and a
    dropped second route contributes nothing."""
    rng = np.random.default_rng(41)
    N, dm, T = 3, 4, 24
    x = rng.standard_normal((T, dm)).astype(np.float32)
    x[:, 3] = 1.0
    w_r = rng.standard_normal((N, dm)).astype(np.float32)
    w1 = np.zeros((N, N, dm), np.float32)
    w2 = np.zeros((N, dm, N), np.float32)
    for e in range(N):
        w1[e, e, 3] = 1.0
        w2[e, e, e] = 100.0 * (e + 1)
    for cf in (4.0, 0.5):
        res = O.layer_forward_top2(x, w_r, None, w1, w2, cf, ALPHA)
        delta = res["out"] - x.astype(np.float64)
        for t in range(T):
            want = np.zeros(dm)
            for r in range(2):
                if not res["drop2"][r, t]:
                    e = res["idx2"][r, t]
                    want[e] += res["gate2"][r, t] * 100.0 * (e + 1)
            np.testing.assert_allclose(delta[t], want, rtol=1e-12, atol=1e-12)
        if cf == 0.5:
            assert res["drop2"].any()
    assert res["loss"] == pytest.approx(
        ALPHA * N * np.sum(np.bincount(res["idx2"][0], minlength=N) / T * res["probs"].mean(0)))


def pin_token_outputs_signature(O):
    """The per-token checker used at full size: token t's block row is
    x_t + p_idx E_idx(x_t) when kept and x_t when dropped (and the same
    without x when the residual is off), with experts that each write the
    signature 100 (e + 1) unit(e) through a hidden unit that equals one, so
    the expected rows are closed forms.  Capacity 0.5 drops tokens."""
    rng = np.random.default_rng(17)
    N, dm, T = 3, 4, 30
    x = rng.standard_normal((T, dm)).astype(np.float32)
    x[:, 3] = 1.0
    w_r = rng.standard_normal((N, dm)).astype(np.float32)
    w1 = np.zeros((N, N, dm), np.float32)
    w2 = np.zeros((N, dm, N), np.float32)
    for e in range(N):
        w1[e, e, 3] = 1.0
        w2[e, e, e] = 100.0 * (e + 1)
    r = O.router(x, w_r)
    C = O.capacity(T, N, 0.5)
    dsp = O.dispatch(r["idx"], N, C)
    assert dsp["drop"].any() and not dsp["drop"].all()
    toks = np.arange(T)[::-1]               # any order of the requested tokens
    for residual in (True, False):
        rows = O.token_outputs(x, toks, r["idx"], dsp["drop"], r["gate"], w1, w2,
                               residual=residual)
        for j, t in enumerate(toks):
            want = x[t].astype(np.float64).copy() if residual else np.zeros(dm)
            if not dsp["drop"][t]:
                e = r["idx"][t]
                want[e] += r["gate"][t] * 100.0 * (e + 1)
            np.testing.assert_allclose(rows[j], want, rtol=1e-12, atol=1e-12)


def pin_token_outputs_match_layer(O):
    """token_outputs on every token equals the whole layer's output (the fp32
    Tiny workload and a small bf16 one with a Zipf bias and drops), with and
    without the residual."""
    from switch_inputs import Workload, make_inputs
    for wl in (Workload("t32", T=96, d_model=16, d_ff=32, n_experts=4, capacity_factor=0.75,
                        dtype="f32", seed=21),
               Workload("tbf", T=80, d_model=64, d_ff=64, n_experts=5, capacity_factor=1.0,
                        dtype="bf16", zipf_s=1.1, seed=22)):
        inp = make_inputs(wl)
        for residual in (True, False):
            res = O.layer_forward(inp.x, inp.w_r, inp.b_r, inp.w1, inp.w2,
                                  wl.capacity_factor, ALPHA, residual=residual)
            assert res["drop"].any()
            rows = O.token_outputs(inp.x, np.arange(wl.T), res["idx"], res["drop"],
                                   res["gate"], inp.w1, inp.w2, residual=residual)
            np.testing.assert_allclose(rows, res["out"], rtol=1e-12, atol=1e-15)


PINS = [pin_capacity, pin_softmax_hand, pin_router_invariants, pin_dispatch_hand,
        pin_dispatch_bruteforce, pin_dispatch_via_router, pin_aux_hand,
        pin_aux_uniform, pin_dense_reduction, pin_single_expert_signature,
        pin_dropped_residual, pin_relu_active, pin_top2_router_hand,
        pin_top2_router_invariants, pin_top2_dispatch_hand, pin_top2_dispatch_bruteforce,
        pin_top2_dense_reduction, pin_top2_signature, pin_token_outputs_signature,
        pin_token_outputs_match_layer]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(orc)


# ------------------------------------------------- planted mistakes (CPU)

def _mut_capacity_floor(T, N, cf):
    from fractions import Fraction
    return math.floor(Fraction(T) * Fraction(cf) / N)


def _mut_router_last_tie(real):
    def f(x, w_r, b_r=None):
        r = real(x, w_r, b_r)
        h32 = r["logits"].astype(np.float32)
        N = h32.shape[1]
        r["idx"] = (N - 1 - np.argmax(h32[:, ::-1], axis=1)).astype(np.int64)
        r["gate"] = r["probs"][np.arange(len(r["idx"])), r["idx"]]
        return r
    return f


def _mut_router_no_bias(real):
    return lambda x, w_r, b_r=None: real(x, w_r, None)


def _mut_dispatch_drop_gt(real):
    def f(idx, N, C):
        d = real(idx, N, C)
        d["drop"] = d["rank"] > C          # lets one token too many through
        return d
    return f


def _mut_dispatch_counts_kept(real):
    def f(idx, N, C):
        d = real(idx, N, C)
        d["counts"] = np.minimum(d["counts"], C)
        return d
    return f


def _mut_dispatch_from_one(real):
    def f(idx, N, C):
        d = real(idx, N, C)
        d["rank"] = d["rank"] + 1
        return d
    return f


def _mut_expert_no_relu(x_rows, w1_e, w2_e):
    from switch_inputs import as_f64
    return (as_f64(x_rows) @ as_f64(w1_e).T) @ as_f64(w2_e).T


def _mut_combine_no_gate(real):
    def f(x, idx, rank, drop, gate, Y, residual=True):
        return real(x, idx, rank, drop, np.ones_like(np.asarray(gate)), Y, residual)
    return f


def _mut_combine_drop_zero(real):
    def f(x, idx, rank, drop, gate, Y, residual=True):
        out = real(x, idx, rank, drop, gate, Y, residual)
        out[np.asarray(drop, bool)] = 0.0
        return out
    return f


def _mut_aux_P_from_f(real):
    def f(counts, probs, alpha):
        T = probs.shape[0]
        fake = np.zeros_like(np.asarray(probs, np.float64))
        idx = np.argmax(probs, axis=1)
        fake[np.arange(T), idx] = 1.0
        return real(counts, fake, alpha)
    return f


def _mut_aux_no_N(real):
    def f(counts, probs, alpha):
        loss, f_, P = real(counts, probs, alpha)
        return loss / len(counts), f_, P
    return f


def _mut_top2_second_highest_index(real):
    def f(x, w_r, b_r=None):
        r = real(x, w_r, b_r)
        h32 = r["logits"].astype(np.float32)
        T, N = h32.shape
        rest = h32.copy()
        rest[np.arange(T), r["idx2"][0]] = -np.inf
        r["idx2"][1] = (N - 1 - np.argmax(rest[:, ::-1], axis=1)).astype(np.int64)
        r["gate2"][1] = r["probs"][np.arange(T), r["idx2"][1]]
        return r
    return f


def _mut_top2_renormalised(real):
    def f(x, w_r, b_r=None):
        r = real(x, w_r, b_r)
        r["gate2"] = r["gate2"] / r["gate2"].sum(axis=0, keepdims=True)
        return r
    return f


def _mut_top2_token_major(real):
    def f(idx2, N, C):
        idx2 = np.asarray(idx2)
        T = idx2.shape[1]
        d = orc.dispatch(idx2.T.reshape(-1), N, C)      # (t, r) order instead
        rank = d["rank"].reshape(T, 2).T
        st = np.where(d["slot_token"] >= 0, d["slot_token"] // 2, -1)
        return {"rank": rank, "drop": rank >= C, "counts": d["counts"], "slot_token": st}
    return f


def _mut_token_outputs_next_expert(real):
    def f(x, tokens, idx, drop, gate, w1, w2, residual=True):
        N = np.shape(w1)[0]
        return real(x, tokens, (np.asarray(idx) + 1) % N, drop, gate, w1, w2, residual)
    return f


def _mut_token_outputs_first_gate(real):
    def f(x, tokens, idx, drop, gate, w1, w2, residual=True):
        g = np.full(len(gate), np.asarray(gate)[0])     # one token's gate for all
        return real(x, tokens, idx, drop, g, w1, w2, residual)
    return f


def _mut_token_outputs_keeps_dropped(real):
    def f(x, tokens, idx, drop, gate, w1, w2, residual=True):
        return real(x, tokens, idx, np.zeros(len(drop), bool), gate, w1, w2, residual)
    return f


def _mut_token_outputs_always_residual(real):
    def f(x, tokens, idx, drop, gate, w1, w2, residual=True):
        return real(x, tokens, idx, drop, gate, w1, w2, True)
    return f


MUTANTS = {
    "top2_second_on_last_tie": ("router_top2", _mut_top2_second_highest_index),
    "top2_gates_renormalised": ("router_top2", _mut_top2_renormalised),
    "top2_token_major_slots": ("dispatch_top2", _mut_top2_token_major),
    "capacity_floor": ("capacity", lambda real: _mut_capacity_floor),
    "argmax_last_on_tie": ("router", _mut_router_last_tie),
    "router_ignores_bias": ("router", _mut_router_no_bias),
    "drop_uses_gt": ("dispatch", _mut_dispatch_drop_gt),
    "counts_after_drop": ("dispatch", _mut_dispatch_counts_kept),
    "rank_from_one": ("dispatch", _mut_dispatch_from_one),
    "expert_no_relu": ("expert", lambda real: _mut_expert_no_relu),
    "combine_no_gate": ("combine", _mut_combine_no_gate),
    "dropped_not_residual": ("combine", _mut_combine_drop_zero),
    "P_from_hard_counts": ("aux_loss", _mut_aux_P_from_f),
    "loss_without_N": ("aux_loss", _mut_aux_no_N),
    "token_outputs_next_expert": ("token_outputs", _mut_token_outputs_next_expert),
    "token_outputs_first_gate": ("token_outputs", _mut_token_outputs_first_gate),
    "token_outputs_keeps_dropped": ("token_outputs", _mut_token_outputs_keeps_dropped),
    "token_outputs_always_residual": ("token_outputs", _mut_token_outputs_always_residual),
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
