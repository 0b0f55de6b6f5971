"""GPU parity of each stage, called through the C ABI, against the CPU oracle
on the same seeded inputs.  Sizes span several 128-row tiles, ragged tails
in every dimension the kernels tile (tokens, capacity rows, d_ff and
d_model column tiles) and the degenerate cases the layer has."""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import (Workload, make_inputs, make_router, make_x, f32_to_bf16_bits,
                           as_f64)
from gpu_util import (dev_float, host_f64, rms_ratio, check_routing, rel_err, PROB_RTOL,
                      BF16_RMS_TOL, F32_RMS_TOL, LOSS_RTOL)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _cfg(sm, wl, flags=0, **kw):
    return sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                     dtype=wl.dtype, alpha=wl.alpha, flags=flags, **kw)


def _ok(sm, ws):
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"


I32 = dict(dtype=torch.int32, device="cuda")
F32 = dict(dtype=torch.float32, device="cuda")

# ----------------------------------------------------------------- router

ROUTER_CASES = [
    Workload("r_small", T=3000, d_model=320, d_ff=64, n_experts=8, capacity_factor=1.25,
             dtype="bf16", seed=11),
    Workload("r_base", T=1000, d_model=768, d_ff=64, n_experts=128, capacity_factor=1.25,
             dtype="bf16", seed=12),
    Workload("r_zipf", T=777, d_model=256, d_ff=64, n_experts=64, capacity_factor=1.0,
             dtype="bf16", zipf_s=1.1, seed=13),
    Workload("r_odd", T=333, d_model=128, d_ff=64, n_experts=37, capacity_factor=1.0,
             dtype="bf16", seed=14),
    Workload("r_f32", T=515, d_model=64, d_ff=64, n_experts=4, capacity_factor=1.25,
             dtype="f32", seed=15),
    Workload("r_wide", T=300, d_model=64, d_ff=64, n_experts=1000, capacity_factor=1.0,
             dtype="bf16", seed=16),
]


@pytest.mark.parametrize("flags", [0, 1], ids=["default", "simt"])
@pytest.mark.parametrize("wl", ROUTER_CASES, ids=lambda w: w.name)
def test_router(sm, wl, flags):
    x = make_x(wl)
    w_r, b_r = make_router(wl)
    r = orc.router(x, w_r, b_r)
    cfg = _cfg(sm, wl, flags)
    ws = sm.workspace(cfg)
    idx = torch.empty(wl.T, **I32)
    gate = torch.empty(wl.T, **F32)
    probs = torch.empty(wl.T, wl.n_experts, **F32)
    sm.switch_router(cfg, dev_float(x), dev_float(w_r), None if b_r is None else dev_float(b_r),
                     idx, gate, probs, ws)
    _ok(sm, ws)
    p = probs.cpu().numpy()
    assert rel_err(p, r["probs"]).max() <= PROB_RTOL
    ig = idx.cpu().numpy()
    check_routing(ig, r)
    want_gate = r["probs"][np.arange(wl.T), ig]
    assert rel_err(gate.cpu().numpy(), want_gate).max() <= PROB_RTOL


def test_router_three_term_split(sm):
    """Three bf16 terms (their sum is W_r exactly): reported, and held to
    the same probability tolerance."""
    wl = ROUTER_CASES[1]
    x = make_x(wl)
    w_r, b_r = make_router(wl)
    r = orc.router(x, w_r, b_r)
    cfg = _cfg(sm, wl, sm.FLAG_ROUTER_3TERM)
    ws = sm.workspace(cfg)
    idx = torch.empty(wl.T, **I32)
    gate = torch.empty(wl.T, **F32)
    probs = torch.empty(wl.T, wl.n_experts, **F32)
    sm.switch_router(cfg, dev_float(x), dev_float(w_r), None, idx, gate, probs, ws)
    _ok(sm, ws)
    err = rel_err(probs.cpu().numpy(), r["probs"]).max()
    print(f"three-term router: max prob rel err {err:.3e}")
    assert err <= PROB_RTOL
    check_routing(idx.cpu().numpy(), r)


def test_router_uniform_ties(sm):
    """W_r = 0: every logit ties, p = 1/N, expert 0 (lowest index) wins."""
    wl = Workload("ties", T=300, d_model=128, d_ff=64, n_experts=16, capacity_factor=1.0,
                  dtype="bf16", seed=3)
    x = make_x(wl)
    for flags in (0, sm.FLAG_ROUTER_SIMT):
        cfg = _cfg(sm, wl, flags)
        ws = sm.workspace(cfg)
        idx = torch.full((wl.T,), -5, **I32)
        gate = torch.empty(wl.T, **F32)
        probs = torch.empty(wl.T, 16, **F32)
        sm.switch_router(cfg, dev_float(x), torch.zeros(16, 128, **F32), None, idx, gate,
                         probs, ws)
        _ok(sm, ws)
        assert (idx.cpu().numpy() == 0).all()
        assert (probs.cpu().numpy() == 1.0 / 16).all()
        assert (gate.cpu().numpy() == 1.0 / 16).all()


# --------------------------------------------------------------- dispatch

def _dispatch_gpu(sm, wl, idx=None, probs=None, x=None, want_xdisp=False):
    cfg = _cfg(sm, wl)
    C = sm.switch_capacity(wl.T, wl.n_experts, wl.capacity_factor)
    ws = sm.workspace(cfg)
    rank = torch.empty(wl.T, **I32)
    drop = torch.empty(wl.T, dtype=torch.uint8, device="cuda")
    counts = torch.empty(wl.n_experts, **I32)
    slot = torch.empty(max(wl.n_experts * C, 1), **I32)
    xd = None
    if want_xdisp:
        dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        xd = torch.full((wl.n_experts * C, wl.d_model), 7.0, dtype=dt, device="cuda")
    sm.switch_dispatch(cfg, None if idx is None else torch.from_numpy(idx.astype(np.int32)).cuda(),
                       None if probs is None else torch.from_numpy(probs).cuda(),
                       rank, drop, counts, slot, x, xd, ws)
    st = sm.switch_get_device_error(ws)
    return C, st, rank.cpu().numpy(), drop.cpu().numpy(), counts.cpu().numpy(), \
        slot.cpu().numpy()[: wl.n_experts * C], xd


DISPATCH_CASES = [(3000, 8, 1.25), (1000, 128, 1.25), (4099, 64, 0.3), (129, 3, 4.0),
                  (1, 4, 1.0), (5000, 1024, 1.0), (700, 1, 1.0), (2048, 16, 0.01)]


@pytest.mark.parametrize("T,N,cf", DISPATCH_CASES)
def test_dispatch_from_idx_bitexact(sm, T, N, cf):
    rng = np.random.default_rng(T * 7 + N)
    # skewed assignment so that some experts overflow and others stay empty
    w = rng.dirichlet(np.full(N, 0.3))
    idx = rng.choice(N, size=T, p=w).astype(np.int64)
    wl = Workload("d", T=T, d_model=64, d_ff=64, n_experts=N, capacity_factor=cf, dtype="bf16")
    C, st, rank, drop, counts, slot, _ = _dispatch_gpu(sm, wl, idx=idx)
    assert st[0] == 0
    want = orc.dispatch(idx, N, orc.capacity(T, N, cf))
    assert C == orc.capacity(T, N, cf)
    np.testing.assert_array_equal(rank, want["rank"])
    np.testing.assert_array_equal(drop.astype(bool), want["drop"])
    np.testing.assert_array_equal(counts, want["counts"])
    np.testing.assert_array_equal(slot, want["slot_token"])


def test_dispatch_from_router_probs_bitexact(sm):
    """Fed the oracle's fp32 probabilities: the top-1 is taken on those same
    fp32 values (lowest index on ties) on both sides."""
    wl = Workload("dp", T=2500, d_model=256, d_ff=64, n_experts=32, capacity_factor=1.0,
                  dtype="bf16", seed=21)
    x = make_x(wl)
    w_r, _ = make_router(wl)
    p32 = orc.router(x, w_r)["probs"].astype(np.float32)
    idx32 = np.argmax(p32, axis=1)
    C, st, rank, drop, counts, slot, xd = _dispatch_gpu(sm, wl, probs=p32, x=dev_float(x),
                                                          want_xdisp=True)
    assert st[0] == 0
    want = orc.dispatch(idx32, 32, C)
    np.testing.assert_array_equal(rank, want["rank"])
    np.testing.assert_array_equal(drop.astype(bool), want["drop"])
    np.testing.assert_array_equal(counts, want["counts"])
    np.testing.assert_array_equal(slot, want["slot_token"])
    # gathered rows: bit copies of x, zeros in padding slots
    xd_bits = xd.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(32 * C):
        t = want["slot_token"][s]
        if t >= 0:
            assert (xd_bits[s] == x[t]).all()
        else:
            assert (xd_bits[s] == 0).all()


def test_dispatch_rejects_bad_expert_ids(sm):
    wl = Workload("bad", T=200, d_model=64, d_ff=64, n_experts=4, capacity_factor=2.0,
                  dtype="bf16")
    idx = np.zeros(200, np.int64)
    idx[17] = 9
    idx[150] = -2
    C, st, rank, drop, counts, slot, _ = _dispatch_gpu(sm, wl, idx=idx)
    assert st[0] == 6      # SWITCH_ERR_DEVICE_BOUNDS
    assert drop[17] == 1 and drop[150] == 1 and rank[17] == -1
    assert counts.sum() == 198


# ------------------------------------------------------------- expert FFN

FFN_CASES = [
    Workload("f_ragged", T=3000, d_model=320, d_ff=576, n_experts=8, capacity_factor=1.25,
             dtype="bf16", seed=31),
    Workload("f_many", T=4096, d_model=256, d_ff=512, n_experts=32, capacity_factor=1.0,
             dtype="bf16", seed=32),
    Workload("f_tiny", T=512, d_model=64, d_ff=256, n_experts=4, capacity_factor=1.25,
             dtype="f32", seed=33),
]


@pytest.mark.parametrize("flags", [0, 8, 32, 40, 64, 72, 2048, 2048 | 8],
                         ids=["default", "gather_in_gemm", "one_sm", "one_sm_gather", "pairs",
                              "pairs_gather", "rows_pairs", "rows_pairs_gather"])
@pytest.mark.parametrize("wl", FFN_CASES, ids=lambda w: w.name)
def test_expert_ffn(sm, wl, flags):
    inp = make_inputs(wl)
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(r["idx"], wl.n_experts, C)
    Y = orc.expert_ffn(inp.x, inp.w1, inp.w2, dsp["slot_token"], dsp["counts"], C)
    cfg = _cfg(sm, wl, flags)
    ws = sm.workspace(cfg)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    y = torch.full((wl.n_experts * C, wl.d_model), float("nan"), dtype=dt, device="cuda")
    sm.switch_expert_ffn(cfg, dev_float(inp.x),
                         torch.from_numpy(dsp["slot_token"].astype(np.int32)).cuda(),
                         torch.from_numpy(dsp["counts"].astype(np.int32)).cuda(),
                         dev_float(inp.w1), dev_float(inp.w2), y, ws)
    _ok(sm, ws)
    yg = host_f64(y).reshape(wl.n_experts, C, wl.d_model)
    kept = np.zeros((wl.n_experts, C), bool)
    for e in range(wl.n_experts):
        kept[e, : min(int(dsp["counts"][e]), C)] = True
    tol = BF16_RMS_TOL if wl.dtype == "bf16" else F32_RMS_TOL
    assert rms_ratio(yg[kept], Y[kept]) <= tol
    assert np.isnan(yg[~kept]).all()     # padding rows untouched


@pytest.mark.parametrize("flags", [128, 128 | 32, 128 | 64, 128 | 2048],
                         ids=["default", "one_sm", "pairs", "rows_pairs"])
@pytest.mark.parametrize("wl", FFN_CASES, ids=lambda w: w.name)
def test_expert_ffn_rows_dispatched(sm, wl, flags):
    """x_disp from switch_dispatch fed to switch_expert_ffn (ROWS_DISPATCHED):
    same rows as the oracle's FFN, and bit-identical to the call that
    dispatches the rows itself."""
    inp = make_inputs(wl)
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(r["idx"], wl.n_experts, C)
    Y = orc.expert_ffn(inp.x, inp.w1, inp.w2, dsp["slot_token"], dsp["counts"], C)
    x = dev_float(inp.x)
    _, st, _, _, counts, slot, xd = _dispatch_gpu(sm, wl, idx=r["idx"], x=x, want_xdisp=True)
    assert st[0] == 0
    np.testing.assert_array_equal(counts, dsp["counts"])
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    counts_d = torch.from_numpy(counts.astype(np.int32)).cuda()
    w1, w2 = dev_float(inp.w1), dev_float(inp.w2)
    cfg = _cfg(sm, wl, flags)
    ws = sm.workspace(cfg)
    y = torch.full((wl.n_experts * C, wl.d_model), float("nan"), dtype=dt, device="cuda")
    sm.switch_expert_ffn(cfg, xd, None, counts_d, w1, w2, y, ws)
    _ok(sm, ws)
    y_ref = torch.full_like(y, float("nan"))
    cfg0 = _cfg(sm, wl, flags & ~128)
    sm.switch_expert_ffn(cfg0, x, torch.from_numpy(slot.astype(np.int32)).cuda(), counts_d,
                         w1, w2, y_ref, ws)
    _ok(sm, ws)
    kept = np.zeros((wl.n_experts, C), bool)
    for e in range(wl.n_experts):
        kept[e, : min(int(counts[e]), C)] = True
    yg = host_f64(y).reshape(wl.n_experts, C, wl.d_model)
    tol = BF16_RMS_TOL if wl.dtype == "bf16" else F32_RMS_TOL
    assert rms_ratio(yg[kept], Y[kept]) <= tol
    assert np.isnan(yg[~kept]).all()
    np.testing.assert_array_equal(yg[kept], host_f64(y_ref).reshape(wl.n_experts, C, -1)[kept])


def test_expert_ffn_dense_reduction(sm):
    """N = 1, capacity factor 1: one expert holds every token, the layer is a
    dense FFN (checked against the oracle's single-expert FFN)."""
    wl = Workload("dense", T=700, d_model=192, d_ff=320, n_experts=1, capacity_factor=1.0,
                  dtype="bf16", seed=41)
    inp = make_inputs(wl)
    cfg = _cfg(sm, wl)
    ws = sm.workspace(cfg)
    y = torch.empty(700, 192, dtype=torch.bfloat16, device="cuda")
    sm.switch_expert_ffn(cfg, dev_float(inp.x), torch.arange(700, **I32),
                         torch.tensor([700], **I32), dev_float(inp.w1), dev_float(inp.w2), y, ws)
    _ok(sm, ws)
    want = orc.expert(inp.x, inp.w1[0], inp.w2[0])
    assert rms_ratio(host_f64(y), want) <= BF16_RMS_TOL


# ---------------------------------------------------------------- combine

@pytest.mark.parametrize("residual", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_combine(sm, residual, dtype):
    wl = Workload("c", T=2000, d_model=256, d_ff=64, n_experts=16, capacity_factor=0.7,
                  dtype=dtype, seed=51)
    x = make_x(wl)
    w_r, _ = make_router(wl)
    r = orc.router(x, w_r)
    C = orc.capacity(wl.T, 16, 0.7)
    dsp = orc.dispatch(r["idx"], 16, C)
    assert dsp["drop"].any()
    rng = np.random.default_rng(5)
    Yv = rng.standard_normal((16, C, 256)).astype(np.float32)
    if dtype == "bf16":
        Ybits = f32_to_bf16_bits(Yv)
        Y64 = as_f64(Ybits)
        ydev = dev_float(Ybits)
    else:
        Y64 = Yv.astype(np.float64)
        ydev = dev_float(Yv)
    gate32 = r["gate"].astype(np.float32)
    want = orc.combine(x, r["idx"], dsp["rank"], dsp["drop"], gate32.astype(np.float64), Y64,
                       residual)
    cfg = _cfg(sm, wl)
    out = torch.empty(wl.T, 256, dtype=ydev.dtype, device="cuda")
    sm.switch_combine(cfg, dev_float(x) if residual else None,
                      torch.from_numpy(r["idx"].astype(np.int32)).cuda(),
                      torch.from_numpy(dsp["rank"].astype(np.int32)).cuda(),
                      torch.from_numpy(dsp["drop"].astype(np.uint8)).cuda(),
                      torch.from_numpy(gate32).cuda(), ydev.reshape(16 * C, 256), out)
    torch.cuda.synchronize()
    got = host_f64(out)
    tol = BF16_RMS_TOL if dtype == "bf16" else F32_RMS_TOL
    assert rms_ratio(got, want) <= tol
    d = dsp["drop"]
    assert (got[d] == want[d]).all()       # dropped: residual (or 0) bit for bit


# --------------------------------------------------------------- aux loss

# (T, N): float4 columns; one column per thread (N % 4 != 0); blocks left
# with no rows (T = 9473 over 148 blocks of 65 rows); N >= 512 (several
# passes over the experts in the final sum), also with scalar columns
AUX_CASES = [(3333, 24), (10000, 37), (9473, 128), (2000, 600), (777, 1001)]


@pytest.mark.parametrize("T,N", AUX_CASES, ids=lambda v: str(v))
def test_aux_loss(sm, T, N):
    wl = Workload("a", T=T, d_model=128, d_ff=64, n_experts=N, capacity_factor=1.0,
                  dtype="bf16", seed=61)
    x = make_x(wl)
    w_r, _ = make_router(wl)
    r = orc.router(x, w_r)
    C = orc.capacity(wl.T, N, 1.0)
    counts = orc.dispatch(r["idx"], N, C)["counts"]
    p32 = r["probs"].astype(np.float32)
    loss_w, f_w, P_w = orc.aux_loss(counts, p32.astype(np.float64), wl.alpha)
    cfg = _cfg(sm, wl)
    ws = sm.workspace(cfg)
    loss = torch.empty(1, **F32)
    f = torch.empty(N, **F32)
    P = torch.empty(N, **F32)
    cnt = torch.from_numpy(counts.astype(np.int32)).cuda()
    pd = torch.from_numpy(p32).cuda()
    sm.switch_aux_loss(cfg, cnt, pd, loss, f, P, ws)
    _ok(sm, ws)
    assert abs(loss.item() - loss_w) <= LOSS_RTOL * loss_w
    assert rel_err(P.cpu().numpy(), P_w).max() <= LOSS_RTOL
    np.testing.assert_allclose(f.cpu().numpy(), f_w, rtol=1e-7)
    # the same call again: bit for bit (fixed order of additions)
    loss2, P2 = torch.empty_like(loss), torch.empty_like(P)
    sm.switch_aux_loss(cfg, cnt, pd, loss2, None, P2, ws)
    _ok(sm, ws)
    assert torch.equal(loss, loss2) and torch.equal(P, P2)
    # uniform router: loss = alpha exactly in exact arithmetic
    pu = np.full((wl.T, N), 1.0 / N, np.float32)
    sm.switch_aux_loss(cfg, cnt, torch.from_numpy(pu).cuda(), loss, None, None, ws)
    _ok(sm, ws)
    assert abs(loss.item() - wl.alpha) <= LOSS_RTOL * wl.alpha


# ------------------------------------------------------------ edge cases

def test_empty_batch_is_noop(sm):
    wl = Workload("z", T=0, d_model=64, d_ff=64, n_experts=4, capacity_factor=1.0, dtype="bf16")
    cfg = _cfg(sm, wl)
    assert sm.switch_workspace_size(cfg) > 0
    ws = sm.workspace(cfg)
    out = torch.full((1, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    counts = torch.full((4,), -1, **I32)
    sm.switch_layer_forward(cfg, out, torch.zeros(4, 64, **F32), None,
                            torch.zeros(4, 64, 64, dtype=torch.bfloat16, device="cuda"),
                            torch.zeros(4, 64, 64, dtype=torch.bfloat16, device="cuda"),
                            out, None, None, counts, None, ws)
    _ok(sm, ws)
    assert (out.float().cpu() == 3.0).all() and (counts.cpu() == -1).all()


def test_host_argument_errors(sm):
    wl = Workload("e", T=64, d_model=64, d_ff=64, n_experts=4, capacity_factor=1.0, dtype="bf16")
    cfg = _cfg(sm, wl)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    idx = torch.empty(64, **I32)
    gate = torch.empty(64, **F32)
    x = torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_router(cfg, x, torch.zeros(4, 64, **F32), None, idx, gate, None, small)
    assert ei.value.status == 3
    ws = sm.workspace(cfg)
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_router(cfg, x, None, None, idx, gate, None, ws)
    assert ei.value.status == 1
    bad = _cfg(sm, wl.with_(d_model=96))
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_router(bad, x, torch.zeros(4, 96, **F32), None, idx, gate, None, ws)
    assert ei.value.status == 2
