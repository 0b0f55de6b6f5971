"""Full-size parity: every named workload, in the launch configuration the
benchmark times (switch_layer_forward with default flags).

Checked in full: the top-1 choice (equal to the oracle's except on tokens
whose oracle top-1/top-2 probability margin is below 1e-6, counted), the
per-expert counts (bit-exact once the oracle is re-based on the GPU's
choices), every gate (1e-5 relative) and the load-balancing loss (1e-5
relative).  Checked on sampled tokens the oracle computes one by one: the
block output rows (bf16: max |err| <= 2e-2 x RMS of the sampled oracle
rows; fp32: 1e-5), including dropped tokens, which must equal x bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import WORKLOADS, make_inputs, as_f64
from gpu_util import (dev_float, host_f64, check_routing, rel_err, rms_ratio, PROB_RTOL,
                      BF16_RMS_TOL, F32_RMS_TOL, LOSS_RTOL)

pytestmark = pytest.mark.gpu

NAMES = ["tiny", "base", "zipf_cf1.0", "zipf_cf1.25", "zipf_cf2.0", "large", "xxl"]


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _sample_tokens(T, drop, rng, n=40):
    picks = {0, 1, T // 2, T - 2, T - 1}
    picks.update(int(t) for t in rng.choice(T, size=min(n, T), replace=False))
    dropped = np.nonzero(drop)[0]
    if dropped.size:
        picks.update(int(t) for t in rng.choice(dropped, size=min(8, dropped.size),
                                                 replace=False))
    return np.array(sorted(picks))


@pytest.mark.parametrize("name", NAMES)
def test_fullsize_layer(sm, name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    cfg = sm.config(wl.T, wl.d_model, wl.d_ff, wl.n_experts, wl.capacity_factor,
                    dtype=wl.dtype, alpha=wl.alpha)
    ws = sm.workspace(cfg)
    x = dev_float(inp.x)
    w1 = dev_float(inp.w1)
    w2 = dev_float(inp.w2)
    out = torch.empty_like(x)
    idx = torch.empty(wl.T, dtype=torch.int32, device="cuda")
    gate = torch.empty(wl.T, dtype=torch.float32, device="cuda")
    counts = torch.empty(wl.n_experts, dtype=torch.int32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    sm.switch_layer_forward(cfg, x, dev_float(inp.w_r),
                            None if inp.b_r is None else dev_float(inp.b_r), w1, w2, out, idx,
                            gate, counts, loss, ws)
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"
    del w1, w2
    ig = idx.cpu().numpy().astype(np.int64)

    r = orc.router(inp.x, inp.w_r, inp.b_r)
    flips = check_routing(ig, r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(ig, wl.n_experts, C)
    np.testing.assert_array_equal(counts.cpu().numpy(), dsp["counts"])
    g64 = r["probs"][np.arange(wl.T), ig]
    assert rel_err(gate.cpu().numpy(), g64).max() <= PROB_RTOL
    loss_w, _, _ = orc.aux_loss(dsp["counts"], r["probs"], wl.alpha)
    assert abs(loss.item() - loss_w) <= LOSS_RTOL * loss_w

    rng = np.random.default_rng(1234)
    toks = _sample_tokens(wl.T, dsp["drop"], rng)
    want = orc.token_outputs(inp.x, toks, ig, dsp["drop"], g64, inp.w1, inp.w2)
    got = host_f64(out[torch.from_numpy(toks).cuda()])
    tol = BF16_RMS_TOL if wl.dtype == "bf16" else F32_RMS_TOL
    assert rms_ratio(got, want) <= tol
    d = dsp["drop"][toks]
    assert (got[d] == as_f64(inp.x[toks])[d]).all()
    kept = int(np.minimum(dsp["counts"], C).sum())
    print(f"{name}: flips {flips}, drop rate {1 - kept / wl.T:.4f}, "
          f"padding {1 - kept / (wl.n_experts * C):.4f}, loss {loss.item():.6f}")
