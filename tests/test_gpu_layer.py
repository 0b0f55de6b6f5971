"""End-to-end parity of switch_layer_forward against the oracle.

Routing: the GPU's top-1 choice must equal the oracle's except on tokens
whose oracle top-1/top-2 margin is below 1e-6 (counted).  The oracle is then
re-based on the GPU's choices (dispatch, experts, combine, loss recomputed
from them) so that every other output is compared element by element.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import Workload, make_inputs, TINY, as_f64
from gpu_util import (dev_float, host_f64, rms_ratio, check_routing, rel_err, PROB_RTOL,
                      BF16_RMS_TOL, F32_RMS_TOL, LOSS_RTOL)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def run_layer(sm, wl, inp, flags=0):
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                    dtype=wl.dtype, alpha=wl.alpha, flags=flags)
    ws = sm.workspace(cfg)
    x = dev_float(inp.x)
    out = torch.full_like(x, float("nan"))
    idx = torch.empty(wl.T, dtype=torch.int32, device="cuda")
    gate = torch.empty(wl.T, dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.n_experts, dtype=torch.int32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    sm.switch_layer_forward(cfg, x, dev_float(inp.w_r),
                            None if inp.b_r is None else dev_float(inp.b_r),
                            dev_float(inp.w1), dev_float(inp.w2), out, idx, gate, counts, loss,
                            ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"
    return (host_f64(out), idx.cpu().numpy().astype(np.int64), gate.cpu().numpy(),
            counts.cpu().numpy(), float(loss.item()))


def check_layer(sm, wl, flags=0, residual=True):
    inp = make_inputs(wl)
    out, idx, gate, counts, loss = run_layer(sm, wl, inp, flags)
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    flips = check_routing(idx, r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(idx, wl.n_experts, C)                   # re-based on GPU routing
    np.testing.assert_array_equal(counts, dsp["counts"])
    g64 = r["probs"][np.arange(wl.T), idx]
    assert rel_err(gate, g64).max() <= PROB_RTOL
    Y = orc.expert_ffn(inp.x, inp.w1, inp.w2, dsp["slot_token"], dsp["counts"], C)
    want = orc.combine(inp.x, idx, dsp["rank"], dsp["drop"], g64, Y, residual)
    tol = BF16_RMS_TOL if wl.dtype == "bf16" else F32_RMS_TOL
    assert rms_ratio(out, want) <= tol
    d = dsp["drop"]
    if residual:
        assert (out[d] == as_f64(inp.x)[d]).all()
    else:
        assert (out[d] == 0.0).all()
    loss_w, _, _ = orc.aux_loss(dsp["counts"], r["probs"], wl.alpha)
    assert abs(loss - loss_w) <= LOSS_RTOL * loss_w
    return flips, d.mean()


E2E = Workload("e2e", T=3000, d_model=320, d_ff=576, n_experts=8, capacity_factor=1.0,
               dtype="bf16", seed=71)


@pytest.mark.parametrize("flags", [0, 1, 2, 4, 8, 1 | 4 | 8, 32, 32 | 8, 64, 64 | 8, 2048,
                                   2048 | 4, 2048 | 32],
                         ids=["fused", "simt_router", "three_term", "unfused", "gather_in_gemm",
                              "simt_unfused_gather", "gemm_1sm", "gemm_1sm_gather", "gemm_pairs",
                              "gemm_pairs_gather", "gemm1_rows_pairs", "gemm1_rows_pairs_unfused",
                              "gemm1_rows_pairs_1sm"])
def test_layer_bf16(sm, flags):
    flips, drop_rate = check_layer(sm, E2E, flags)
    assert drop_rate > 0     # cf = 1.0 with random routing overflows some experts


def test_layer_capacity_within_one_pair_tile(sm):
    """128 < C <= 256: the default GEMM1 runs on row-major CTA pairs."""
    wl = Workload("c160", T=2048, d_model=256, d_ff=512, n_experts=16, capacity_factor=1.25,
                  dtype="bf16", seed=74)
    assert 128 < sm.switch_capacity(wl.T, wl.n_experts, wl.capacity_factor) <= 256
    check_layer(sm, wl)
    check_layer(sm, wl, sm.FLAG_NO_RESIDUAL, residual=False)


def test_layer_no_residual(sm):
    check_layer(sm, E2E, sm.FLAG_NO_RESIDUAL, residual=False)


def test_layer_tiny_f32(sm):
    check_layer(sm, TINY)


def test_layer_bias_zipf_small(sm):
    wl = Workload("zs", T=4000, d_model=256, d_ff=512, n_experts=16, capacity_factor=1.25,
                  dtype="bf16", zipf_s=1.1, seed=72)
    flips, drop_rate = check_layer(sm, wl)
    assert drop_rate > 0.1


def test_layer_many_experts_simt_router(sm):
    wl = Workload("wide", T=2048, d_model=128, d_ff=128, n_experts=300, capacity_factor=2.0,
                  dtype="bf16", seed=73)
    check_layer(sm, wl)


def test_layer_all_to_one_expert(sm):
    """W_r = 0: every token ties, all go to expert 0; C of them are kept."""
    wl = Workload("one", T=1000, d_model=128, d_ff=256, n_experts=4, capacity_factor=1.0,
                  dtype="bf16", seed=74)
    inp = make_inputs(wl)
    inp.w_r[:] = 0
    out, idx, gate, counts, loss = run_layer(sm, wl, inp)
    assert (idx == 0).all() and counts.tolist() == [1000, 0, 0, 0]
    assert (gate == 0.25).all()
    assert abs(loss - wl.alpha) <= LOSS_RTOL * wl.alpha
    C = 250
    x64 = as_f64(inp.x)
    assert (out[C:] == x64[C:]).all()
    Y = orc.expert(inp.x[:C], inp.w1[0], inp.w2[0])
    assert rms_ratio(out[:C], x64[:C] + 0.25 * Y) <= BF16_RMS_TOL


def test_layer_single_token_and_capacity_one(sm):
    for T, cf in ((1, 1.0), (37, 0.05)):
        wl = Workload("t", T=T, d_model=64, d_ff=128, n_experts=4, capacity_factor=cf,
                      dtype="bf16", seed=75 + T)
        check_layer(sm, wl)


@pytest.mark.parametrize("T,N,d,F,flags", [(1, 4, 64, 128, 0), (37, 4, 64, 128, 0),
                                           (300, 37, 128, 192, 0), (300, 300, 64, 64, 0),
                                           (513, 16, 64, 128, 8), (129, 64, 128, 64, 4),
                                           (1, 2, 64, 128, 512), (300, 37, 128, 192, 512),
                                           (300, 300, 64, 64, 512), (513, 16, 64, 128, 512 | 8)])
def test_workspace_bounds_respected(sm, T, N, d, F, flags):
    """Canary bytes right after the workspace stay untouched, for small and
    odd shapes where padded per-expert scratch is easiest to mis-size."""
    wl = Workload("ws", T=T, d_model=d, d_ff=F, n_experts=N, capacity_factor=1.0,
                  dtype="bf16", seed=81)
    inp = make_inputs(wl)
    cfg = sm.config(T, d, F, N, 1.0, flags=flags)
    n = sm.switch_workspace_size(cfg)
    canary = 1 << 16
    buf = torch.full((n + canary,), 0xA5, dtype=torch.uint8, device="cuda")
    buf[:n].zero_()
    ws = buf[:n]
    x = dev_float(inp.x)
    out = torch.empty_like(x)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    sm.switch_layer_forward(cfg, x, dev_float(inp.w_r), None, dev_float(inp.w1),
                            dev_float(inp.w2), out, None, None, None, loss, ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0
    assert (buf[n:] == 0xA5).all(), "a kernel wrote past the end of the workspace"


@pytest.mark.parametrize("flags", [0, 512, 4, 64])
def test_layer_ignores_stale_workspace(sm, flags):
    """Scratch contents do not matter: a workspace full of 0xFF bytes (NaN in
    bf16 and fp32) past its zeroed error word gives the same output, bit for
    bit, as a zero-filled one (padding rows of the internal buffers are never
    stored from)."""
    wl = Workload("stale", T=2000, d_model=256, d_ff=512, n_experts=16, capacity_factor=1.0,
                  dtype="bf16", seed=83)
    inp = make_inputs(wl)
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, 1.0, flags=flags)
    n = sm.switch_workspace_size(cfg)
    x = dev_float(inp.x)
    w_r, w1, w2 = dev_float(inp.w_r), dev_float(inp.w1), dev_float(inp.w2)
    outs = []
    for fill in (0x00, 0xFF):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        ws[:256].zero_()
        out = torch.empty_like(x)
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        sm.switch_layer_forward(cfg, x, w_r, None, w1, w2, out, None, None, None, loss, ws)
        st, where, info = sm.switch_get_device_error(ws)
        assert st == 0, f"device error {st} at {where} ({info})"
        outs.append((out.clone(), loss.item()))
    assert torch.equal(outs[0][0], outs[1][0]) and outs[0][1] == outs[1][1]
    assert torch.isfinite(outs[1][0].float()).all()
