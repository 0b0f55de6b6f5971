"""CPU oracle for the Switch-FFN layer: forward pass and its gradient.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plainly written
definition that the CUDA library is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the library never calls it and it never calls the library.  It
shares no code with the CUDA path: the one thing both sides use is the
seeded input generator in ``switch_inputs`` (which draws and encodes inputs
and computes no stage of the layer).

Every stage follows the page "Switch Transformers: scaling to
trillion-parameter models" (cited below as [P1 §section]):

* router logits ``h(x) = W_r . x`` and the softmax gate
  [P1 §"Switch Routing: From Top-k to k = 1", gate equation];
* the routing math in float32 [P1 §"Making Sparse Training Stable",
  selective precision] -- the oracle computes logits and probabilities in
  float64 and takes the top-1 decision on the float32-rounded logits;
* top-1 choice, k = 1 [P1 §"Switch Routing", and the dispatch figure
  "argmax p_i, k=1" in §"Expert Capacity and the Capacity Factor"];
* expert capacity = tokens / experts x capacity factor, rounded up
  [P1 §"Expert Capacity and the Capacity Factor", capacity equation];
* overflow tokens dropped to the residual, unused slots are padding
  [same section, the two trade-off bullets and the figure];
* N independent FFN experts [P1 §"The Core Idea"], ReLU, no biases;
* the gate-scaled combine ``y = p_i(x) E_i(x)`` over the single selected
  expert [P1 §"Switch Routing", combine equation with |T| = 1];
* the load-balancing loss ``alpha . N . sum_i f_i P_i`` with ``f_i`` the
  fraction of tokens whose argmax is ``i`` and ``P_i`` the mean router
  probability [P1 §"The Load-Balancing Loss", loss and f/P equations];
* the top-k variant with k = 2 that the pages contrast with k = 1
  [P1 §"Switch Routing: From Top-k to k = 1"]: the two largest gates, the
  output summed over both, each expert's capacity doubled.

Readings taken where the pages leave a step open: capacity rounds up; the
whole batch is one routing group and tokens take slots in batch order;
ties go to the lowest expert index; ``f_i`` counts routed tokens including
dropped ones (the page defines it through the argmax, before capacity);
the combine adds the residual ``x`` when asked (block output of a dropped
token is ``x``); no dropout (forward pass).  Top-2: the second choice is
the largest of the other logits (lowest index on ties); the gates are the
softmax over all experts, not renormalised; the 2T assignments take slots
first choices first, each route in batch order; ``f_i`` still counts first
choices.

The backward pass (``layer_backward``, ``layer_backward_top2``) is the chain
rule through those stages for J = sum(dout * out) + dloss * loss, routing
decisions held fixed (they are piecewise constant).

Arithmetic is float64 throughout (expert matmuls included); floating-point
inputs are the exact values of the bf16 / fp32 bit patterns the GPU reads.
Parity pins: every function here is pinned by a ``-m "not gpu"`` test
(``tests/test_oracle_pins.py``) against closed forms, hand-worked golden
values, invariants the pages state, and brute force; none is unpinned.
"""
from fractions import Fraction
import math

import numpy as np

from switch_inputs import as_f64


# ------------------------------------------------------------------ capacity

def capacity(T: int, n_experts: int, capacity_factor: float) -> int:
    """Expert capacity C = ceil(T / N x capacity_factor), exactly.

    [P1 §"Expert Capacity and the Capacity Factor", capacity equation]; the
    page prints no rounding, rounding up is the reading taken.  The float
    ``capacity_factor`` is taken at its exact binary value.
    """
    if T < 0 or n_experts <= 0 or not capacity_factor > 0:
        raise ValueError("need T >= 0, N > 0, capacity_factor > 0")
    return math.ceil(Fraction(T) * Fraction(capacity_factor) / n_experts)


# -------------------------------------------------------------------- router

def router(x, w_r, b_r=None):
    """Logits, softmax gate, top-1 expert, gate value and top-1/top-2 margin.

    ``x [T, d]`` (fp32 values or bf16 bits), ``w_r [N, d]`` fp32,
    ``b_r [N]`` or None.  Returns a dict:

    * ``logits`` float64 ``h = x . W_r^T (+ b)``
      [P1 §"Switch Routing", router logits];
    * ``probs`` float64 ``p_i = exp(h_i) / sum_j exp(h_j)`` [gate equation],
      evaluated with the row maximum subtracted (same value, no overflow);
    * ``idx`` int64: the expert of largest float32-rounded logit, lowest
      index on ties [k = 1; routing math in float32, §"Making Sparse
      Training Stable"];
    * ``gate`` float64 ``p_idx``;
    * ``margin`` float64: largest minus second largest probability
      (``inf`` when N = 1).
    """
    h = as_f64(x) @ np.asarray(w_r, dtype=np.float64).T
    if b_r is not None:
        h = h + np.asarray(b_r, dtype=np.float64)[None, :]
    T, N = h.shape
    if T == 0:
        z = np.zeros(0)
        return {"logits": h, "probs": h.copy(), "idx": np.zeros(0, np.int64),
                "gate": z, "margin": z}
    shifted = h - h.max(axis=1, keepdims=True)
    e = np.exp(shifted)
    p = e / e.sum(axis=1, keepdims=True)
    idx = np.argmax(h.astype(np.float32), axis=1).astype(np.int64)
    gate = p[np.arange(T), idx]
    if N == 1:
        margin = np.full(T, np.inf)
    else:
        top2 = np.sort(p, axis=1)[:, -2:]
        margin = top2[:, 1] - top2[:, 0]
    return {"logits": h, "probs": p, "idx": idx, "gate": gate,
            "margin": margin}


# ------------------------------------------------------------------ dispatch

def dispatch(idx, n_experts: int, C: int):
    """Capacity-bounded dispatch, one pass over the batch in token order.

    Each token takes the next free slot of its expert; once an expert holds
    C tokens, later tokens routed to it are dropped
    [P1 §"Expert Capacity and the Capacity Factor": overflow dropped,
    unused slots are padding].  Returns ``rank [T]`` (slot number within
    the expert, also for dropped tokens), ``drop [T]`` bool (rank >= C),
    ``counts [N]`` (tokens routed, before the capacity cut) and
    ``slot_token [N*C]`` (token in each slot, -1 for padding).
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    cnt = [0] * n_experts
    rank = np.empty(T, dtype=np.int64)
    drop = np.empty(T, dtype=bool)
    slot_token = np.full(n_experts * C, -1, dtype=np.int64)
    for t in range(T):
        e = int(idx[t])
        r = cnt[e]
        cnt[e] = r + 1
        rank[t] = r
        drop[t] = r >= C
        if r < C:
            slot_token[e * C + r] = t
    return {"rank": rank, "drop": drop,
            "counts": np.asarray(cnt, dtype=np.int64),
            "slot_token": slot_token}


# ---------------------------------------------------------------- experts

def expert(x_rows, w1_e, w2_e):
    """One expert FFN on rows of x: relu(x . W1_e^T) . W2_e^T, float64.

    ``w1_e [F, d]``, ``w2_e [d, F]`` (output-major) [P1 §"The Core Idea":
    each expert is an independent FFN; ReLU and no biases are the reading].
    """
    hid = as_f64(x_rows) @ as_f64(w1_e).T
    hid = np.maximum(hid, 0.0)
    return hid @ as_f64(w2_e).T


def expert_ffn(x, w1, w2, slot_token, counts, C, experts=None):
    """Every expert over its capacity buffer: ``Y [N, C, d]`` float64.

    Row r of expert e holds E_e(x[slot_token[e*C + r]]) for the
    n_e = min(counts[e], C) kept tokens; padding rows stay zero.
    ``experts`` restricts the work to a subset (others stay zero).
    """
    N = len(counts)
    d = x.shape[1]
    Y = np.zeros((N, C, d))
    for e in (range(N) if experts is None else experts):
        n = min(int(counts[e]), C)
        if n == 0:
            continue
        rows = slot_token[e * C: e * C + n]
        Y[e, :n] = expert(x[rows], w1[e], w2[e])
    return Y


# ------------------------------------------------------------------ combine

def combine(x, idx, rank, drop, gate, Y, residual=True):
    """Block output: x + p_idx(x) . E_idx(x) for kept tokens, x for dropped.

    [P1 §"Switch Routing", combine equation with one selected expert;
    §"Expert Capacity ...", a dropped token passes through the residual.]
    With ``residual=False`` the residual term is left out (dropped tokens
    give 0).
    """
    T, d = x.shape
    out = as_f64(x) if residual else np.zeros((T, d))
    kept = ~np.asarray(drop, dtype=bool)
    out[kept] += np.asarray(gate)[kept, None] * Y[np.asarray(idx)[kept],
                                                  np.asarray(rank)[kept]]
    return out


# ----------------------------------------------------------------- aux loss

def aux_loss(counts, probs, alpha: float):
    """loss = alpha . N . sum_i f_i P_i.

    f_i = counts_i / T (tokens whose argmax is i, dropped ones included),
    P_i = mean over tokens of p_i(x)
    [P1 §"The Load-Balancing Loss", loss equation and f/P equations].
    Returns (loss, f, P) in float64; an empty batch gives loss 0.
    """
    counts = np.asarray(counts, dtype=np.float64)
    N = counts.shape[0]
    T = probs.shape[0]
    if T == 0:
        return 0.0, np.zeros(N), np.zeros(N)
    f = counts / T
    P = np.asarray(probs, dtype=np.float64).sum(axis=0) / T
    return float(alpha * N * np.sum(f * P)), f, P


# ------------------------------------------------------------- whole layer

def layer_forward(x, w_r, b_r, w1, w2, capacity_factor, alpha=0.01,
                  residual=True, experts=None):
    """All stages in order; returns every intermediate in a dict."""
    T = x.shape[0]
    N = w_r.shape[0]
    C = capacity(T, N, capacity_factor)
    r = router(x, w_r, b_r)
    dsp = dispatch(r["idx"], N, C)
    Y = expert_ffn(x, w1, w2, dsp["slot_token"], dsp["counts"], C, experts)
    out = combine(x, r["idx"], dsp["rank"], dsp["drop"], r["gate"], Y,
                  residual)
    loss, f, P = aux_loss(dsp["counts"], r["probs"], alpha)
    return {"C": C, **r, **dsp, "Y": Y, "out": out, "loss": loss,
            "f": f, "P": P}


# ------------------------------------------------------- top-2 routing

def router_top2(x, w_r, b_r=None):
    """Top-k routing with k = 2 [P1 §"Switch Routing: From Top-k to k = 1":
    the top-k set T, output sum_{i in T} p_i(x) E_i(x), p the softmax over all
    N experts (not renormalised over T)].

    Returns the single-route dict of ``router`` plus:

    * ``idx2`` int64 ``[2, T]``: row 0 the top-1 expert (as ``idx``), row 1
      the expert of largest float32-rounded logit among the others, lowest
      index on ties;
    * ``gate2`` float64 ``[2, T]``: ``p`` at those experts;
    * ``margin2`` float64 ``[2, T]``: row 0 ``p(1st) - p(2nd)``, row 1
      ``p(2nd) - p(3rd)`` (``inf`` when there is no next expert).
    """
    r = router(x, w_r, b_r)
    h32 = r["logits"].astype(np.float32)
    p = r["probs"]
    T, N = p.shape
    if N < 2:
        raise ValueError("top-2 routing needs at least two experts")
    first = r["idx"]
    rest = h32.copy()
    rest[np.arange(T), first] = -np.inf
    second = np.argmax(rest, axis=1).astype(np.int64)
    idx2 = np.stack([first, second])
    gate2 = np.stack([p[np.arange(T), first], p[np.arange(T), second]])
    ps = -np.sort(-p, axis=1)
    third = ps[:, 2] if N > 2 else np.full(T, -np.inf)
    margin2 = np.stack([ps[:, 0] - ps[:, 1], ps[:, 1] - third])
    return {**r, "idx2": idx2, "gate2": gate2, "margin2": margin2}


def dispatch_top2(idx2, n_experts: int, C: int):
    """Capacity-bounded dispatch of both routes, first choices first.

    The 2T (token, expert) assignments take slots in route-major order:
    every token's first choice in batch order, then every token's second
    choice in batch order, sharing each expert's C slots (the reading for
    k = 2: the pages give the capacity per expert, not the priority between
    routes; first choices first keeps k = 1's behaviour for route 1).
    Assignment a = r * T + t.  Returns ``rank [2, T]``, ``drop [2, T]``,
    ``counts [N]`` (assignments routed to each expert, both routes, before
    the capacity cut) and ``slot_token [N*C]`` (the token of each slot, -1
    for padding).
    """
    idx2 = np.asarray(idx2)
    T = idx2.shape[1]
    d = dispatch(idx2.reshape(-1), n_experts, C)
    st = d["slot_token"]
    st = np.where(st >= 0, st % max(T, 1), -1)
    return {"rank": d["rank"].reshape(2, T), "drop": d["drop"].reshape(2, T),
            "counts": d["counts"], "slot_token": st}


def combine_top2(x, idx2, rank2, drop2, gate2, Y, residual=True):
    """x + sum over the two routes of p_i(x) . E_i(x), dropped routes give 0
    [P1 §"Switch Routing", combine equation with |T| = 2; a dropped
    assignment passes nothing, as in §"Expert Capacity ..."]."""
    T, d = x.shape
    out = as_f64(x) if residual else np.zeros((T, d))
    for r in range(2):
        kept = ~np.asarray(drop2[r], dtype=bool)
        out[kept] += np.asarray(gate2[r])[kept, None] * \
            Y[np.asarray(idx2[r])[kept], np.asarray(rank2[r])[kept]]
    return out


def layer_forward_top2(x, w_r, b_r, w1, w2, capacity_factor, alpha=0.01,
                       residual=True, experts=None):
    """Top-2 layer: capacity ceil(2T / N x capacity_factor) (each expert
    receives tokens from two routes [P1 §"Switch Routing", the k = 1 win
    "half the expert capacity"]); the load-balancing loss keeps its
    definition through the argmax, i.e. the first choices
    [P1 §"The Load-Balancing Loss", f_i]."""
    T = x.shape[0]
    N = w_r.shape[0]
    C = capacity(2 * T, N, capacity_factor)
    r = router_top2(x, w_r, b_r)
    dsp = dispatch_top2(r["idx2"], N, C)
    Y = expert_ffn(x, w1, w2, dsp["slot_token"], dsp["counts"], C, experts)
    out = combine_top2(x, r["idx2"], dsp["rank"], dsp["drop"], r["gate2"], Y,
                       residual)
    counts1 = np.bincount(r["idx2"][0], minlength=N)
    loss, f, P = aux_loss(counts1, r["probs"], alpha)
    return {"C": C, **r, "rank2": dsp["rank"], "drop2": dsp["drop"],
            "counts": dsp["counts"], "slot_token": dsp["slot_token"],
            "counts1": counts1, "Y": Y, "out": out, "loss": loss, "f": f, "P": P}


def token_outputs(x, tokens, idx, drop, gate, w1, w2, residual=True):
    """Block output rows for selected tokens only (for full-size sampling).

    Row j is x[t] + gate[t] . E_idx[t](x[t]) for t = tokens[j] when the token
    is kept, x[t] when it is dropped (without the x term when ``residual`` is
    False) [P1 §"Switch Routing", combine equation with one selected expert;
    §"Expert Capacity and the Capacity Factor", dropped tokens pass through
    the residual]: the same rows as ``layer_forward``'s output, one token at
    a time."""
    tokens = np.asarray(tokens)
    rows = as_f64(x[tokens]) if residual else np.zeros((len(tokens), x.shape[1]))
    for j, t in enumerate(tokens):
        if not drop[t]:
            e = int(idx[t])
            rows[j] += gate[t] * expert(x[t:t + 1], w1[e], w2[e])[0]
    return rows


# ------------------------------------------------------------ backward pass
#
# The gradient of  J = sum(dout * out) + dloss * loss  with respect to x, W_r,
# b_r, W1 and W2, at the forward pass above.  Routing decisions (the argmax,
# the capacity cut) and f_i are piecewise constant in the inputs, so no
# gradient flows through them; the gradient reaches the router through the
# gate value p_idx(x) that scales the expert output [P1 §"Switch Routing:
# From Top-k to k = 1": the gate value makes the router differentiable] and
# through P_i of the load-balancing loss [P1 §"The Load-Balancing Loss":
# P_i is the differentiable factor, f_i is not].  Each step below is the
# chain rule through one forward stage, in float64.


def expert_backward(x_rows, w1_e, w2_e, g_rows, dout_rows):
    """Backward of out_t = x_t + g_t . E_e(x_t) over one expert's kept rows.

    E_e(x) = relu(x W1_e^T) W2_e^T [P1 §"The Core Idea"].  Returns
    ``(dgate [n], dx [n, d], dW1_e [F, d], dW2_e [d, F])``: dgate_t is
    dout_t . E_e(x_t); the expert's input gradient excludes the residual.
    """
    X = as_f64(x_rows)
    W1 = as_f64(w1_e)
    W2 = as_f64(w2_e)
    G = as_f64(dout_rows)
    g = np.asarray(g_rows, dtype=np.float64)
    A = X @ W1.T                       # pre-activation
    H = np.maximum(A, 0.0)
    Y = H @ W2.T                       # expert output
    dgate = np.sum(G * Y, axis=1)
    dY = g[:, None] * G                # gradient at the expert output
    dW2 = dY.T @ H
    dA = (dY @ W2) * (A > 0.0)         # through the ReLU
    dW1 = dA.T @ X
    dX = dA @ W1
    return dgate, dX, dW1, dW2


def router_backward(x, w_r, probs, idx, drop, dgate, counts, alpha, dloss):
    """Backward of the router for top-1 routing.

    dJ/dp_{t,i} = dgate_t [i = idx_t, token kept]
                  + dloss . alpha . N . f_i / T     (loss = alpha N sum f_i P_i,
                                                     P_i = mean_t p_{t,i});
    the softmax Jacobian gives dh_{t,i} = p_{t,i} (dp_{t,i} - sum_j p_{t,j} dp_{t,j});
    h = x W_r^T + b gives dx = dh W_r, dW_r = dh^T x, db = sum_t dh.
    Returns ``(dx_router [T, d], dW_r [N, d], db [N], dh [T, N])``.
    """
    X = as_f64(x)
    Wr = np.asarray(w_r, dtype=np.float64)
    p = np.asarray(probs, dtype=np.float64)
    T, N = p.shape
    f = np.asarray(counts, dtype=np.float64) / T
    dp = np.tile(dloss * alpha * N * f / T, (T, 1))
    kept = ~np.asarray(drop, dtype=bool)
    rows = np.nonzero(kept)[0]
    dp[rows, np.asarray(idx)[rows]] += np.asarray(dgate, dtype=np.float64)[rows]
    dh = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    return dh @ Wr, dh.T @ X, dh.sum(axis=0), dh


def layer_backward(x, w_r, b_r, w1, w2, capacity_factor, dout, dloss=1.0,
                   alpha=0.01, residual=True, idx=None):
    """Gradients of J = sum(dout * out) + dloss * loss for the top-1 layer.

    ``idx`` (optional) imposes the top-1 choices (e.g. those of another
    implementation, to compare on identical routing); by default the
    router's own.  Returns a dict with ``dx [T, d]``, ``dw_r [N, d]``,
    ``db_r [N]``, ``dw1 [N, F, d]``, ``dw2 [N, d, F]`` (float64) and the
    intermediates ``dgate [T]``, ``dh [T, N]``, ``idx``, ``gate``, ``drop``,
    ``counts``, ``slot_token``, ``C``.
    """
    T, d = x.shape
    N = w_r.shape[0]
    C = capacity(T, N, capacity_factor)
    r = router(x, w_r, b_r)
    idx = r["idx"] if idx is None else np.asarray(idx, dtype=np.int64)
    gate = r["probs"][np.arange(T), idx]
    dsp = dispatch(idx, N, C)
    G = as_f64(dout)
    dx = G.copy() if residual else np.zeros((T, d))
    dgate = np.zeros(T)
    dw1 = np.zeros(np.shape(w1))
    dw2 = np.zeros(np.shape(w2))
    for e in range(N):
        n = min(int(dsp["counts"][e]), C)
        if n == 0:
            continue
        rows = dsp["slot_token"][e * C: e * C + n]
        dg, dxe, dw1[e], dw2[e] = expert_backward(x[rows], w1[e], w2[e], gate[rows], dout[rows])
        dgate[rows] = dg
        dx[rows] += dxe
    dxr, dw_r, db_r, dh = router_backward(x, w_r, r["probs"], idx, dsp["drop"], dgate,
                                          dsp["counts"], alpha, dloss)
    dx += dxr
    return {"dx": dx, "dw_r": dw_r, "db_r": db_r, "dw1": dw1, "dw2": dw2,
            "dgate": dgate, "dh": dh, "idx": idx, "gate": gate, "drop": dsp["drop"],
            "counts": dsp["counts"], "slot_token": dsp["slot_token"], "C": C,
            "probs": r["probs"]}


def layer_backward_top2(x, w_r, b_r, w1, w2, capacity_factor, dout, dloss=1.0,
                        alpha=0.01, residual=True, idx2=None):
    """Gradients of J = sum(dout * out) + dloss * loss for the top-2 layer.

    Same chain rule as ``layer_backward``, with both kept routes of a token:
    out = x + sum_r p_{idx_r} E_{idx_r}(x) [P1 §"Switch Routing": the gates
    are the full-softmax probabilities, not renormalised], so each kept route
    contributes its own expert gradients and a gate gradient
    dgate_r = dout . E_{idx_r}(x) at p_{idx_r}; the loss's f_i counts first
    choices and is held fixed, P_i is differentiated through every p_i.
    ``idx2`` ([2, T], optional) imposes the choices.  Returns the dict of
    ``layer_backward`` with ``dgate`` of shape [2, T] and ``drop2``.
    """
    T, d = x.shape
    N = w_r.shape[0]
    C = capacity(2 * T, N, capacity_factor)
    r = router_top2(x, w_r, b_r)
    idx2 = r["idx2"] if idx2 is None else np.asarray(idx2, dtype=np.int64)
    p = r["probs"]
    gate2 = np.stack([p[np.arange(T), idx2[0]], p[np.arange(T), idx2[1]]])
    dsp = dispatch_top2(idx2, N, C)
    G = as_f64(dout)
    dx = G.copy() if residual else np.zeros((T, d))
    dgate = np.zeros((2, T))
    dw1 = np.zeros(np.shape(w1))
    dw2 = np.zeros(np.shape(w2))
    for e in range(N):
        n = min(int(dsp["counts"][e]), C)
        if n == 0:
            continue
        tok = dsp["slot_token"][e * C: e * C + n]
        # the route of each slot: the token's first choice if it is e, else its second
        route = np.where(idx2[0, tok] == e, 0, 1)
        g = gate2[route, tok]
        dg, dxe, dw1[e], dw2[e] = expert_backward(x[tok], w1[e], w2[e], g, dout[tok])
        dgate[route, tok] = dg
        np.add.at(dx, tok, dxe)
    counts1 = np.bincount(idx2[0], minlength=N)
    dxr, dw_r, db_r, dh = router_backward_top2(x, w_r, p, idx2, dsp["drop"], dgate, counts1,
                                               alpha, dloss)
    dx += dxr
    return {"dx": dx, "dw_r": dw_r, "db_r": db_r, "dw1": dw1, "dw2": dw2, "dgate": dgate,
            "dh": dh, "idx2": idx2, "gate2": gate2, "drop2": dsp["drop"],
            "counts": dsp["counts"], "C": C}


def router_backward_top2(x, w_r, probs, idx2, drop2, dgate2, counts1, alpha, dloss):
    """Router backward for top-2 routing: as ``router_backward`` with
    dJ/dp_{t,i} = sum over the token's kept routes r with idx_r = i of
    dgate_r[t], plus dloss . alpha . N . f_i / T where f_i counts first
    choices (``counts1``) [P1 §"The Load-Balancing Loss", f through the
    argmax].  Returns ``(dx_router, dW_r, db, dh)``."""
    X = as_f64(x)
    p = np.asarray(probs, dtype=np.float64)
    T, N = p.shape
    f = np.asarray(counts1, dtype=np.float64) / T
    dp = np.tile(dloss * alpha * N * f / T, (T, 1))
    for rr in range(2):
        rows = np.nonzero(~np.asarray(drop2[rr], dtype=bool))[0]
        dp[rows, np.asarray(idx2)[rr, rows]] += np.asarray(dgate2)[rr, rows]
    dh = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    Wr = np.asarray(w_r, dtype=np.float64)
    return dh @ Wr, dh.T @ X, dh.sum(axis=0), dh
