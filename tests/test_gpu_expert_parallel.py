"""Expert parallelism on one GPU: G ranks simulated in one process.

Each simulated rank has its own workspace, exchange record, receive buffer
and output, and the ranks' calls run in the protocol's order on one stream
(route on every rank; the records laid end to end, standing in for the
all-gather; dispatch on every rank; experts on every rank).  No kernel waits
on another rank's kernel: the "peer" pointers are ordinary buffers on this
GPU, so the exchange is exercised without a second GPU.

The G ranks' batches form one routing group, so every result must equal
the one-GPU layer (switch_layer_forward) on the concatenated batch: outputs,
choices, gates and counts bit for bit, the loss bit for bit when every rank
holds a multiple of 128 tokens (else to fp32 summation order).  The counts
and the expert term are also checked against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc
from switch_inputs import Workload, WORKLOADS, make_inputs
from gpu_util import dev_float, host_f64, check_routing, bf16_rms_excess, BF16_RMS_TOL

pytestmark = pytest.mark.gpu

I32 = dict(dtype=torch.int32, device="cuda")


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _ok(sm, ws):
    st, where, info = sm.switch_get_device_error(ws)
    assert st == 0, f"device error {st} at {where} ({info})"


def run_ep_simulated(sm, wl, dev, G, flags=0):
    """The expert-parallel protocol for G ranks of T / G tokens each."""
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    Tr, E = T // G, N // G
    cfg = sm.config(Tr, d, F, N, wl.capacity_factor, alpha=wl.alpha, flags=flags)
    eps = [sm.ep(G, r) for r in range(G)]
    ws_b, rec_b, recv_b = sm.switch_ep_sizes(cfg, eps[0])
    ws = [torch.zeros(ws_b, dtype=torch.uint8, device="cuda") for _ in range(G)]
    rec = [torch.zeros(rec_b, dtype=torch.uint8, device="cuda") for _ in range(G)]
    recv = [torch.full((recv_b,), 0xFF, dtype=torch.uint8, device="cuda") for _ in range(G)]
    out = [torch.full((Tr, d), float("nan"), dtype=torch.bfloat16, device="cuda")
           for _ in range(G)]
    idx = [torch.empty(Tr, **I32) for _ in range(G)]
    gate = [torch.empty(Tr, dtype=torch.float32, device="cuda") for _ in range(G)]
    counts = [torch.empty(N, **I32) for _ in range(G)]
    loss = [torch.empty(1, dtype=torch.float32, device="cuda") for _ in range(G)]
    xs = [dev["x"][r * Tr:(r + 1) * Tr] for r in range(G)]
    for r in range(G):
        sm.switch_ep_route(cfg, eps[r], xs[r], dev["w_r"], dev["b_r"], idx[r], gate[r], rec[r],
                           ws[r])
    records = torch.cat(rec)                 # what the all-gather delivers
    for r in range(G):
        sm.switch_ep_dispatch(cfg, eps[r], xs[r], records, recv, out[r], counts[r], loss[r],
                              ws[r])
    for r in range(G):
        sm.switch_ep_experts(cfg, eps[r], dev["w1"][r * E:(r + 1) * E],
                             dev["w2"][r * E:(r + 1) * E], recv[r], out, ws[r])
    torch.cuda.synchronize()
    for r in range(G):
        _ok(sm, ws[r])
    for r in range(1, G):
        assert torch.equal(counts[r], counts[0]) and torch.equal(loss[r], loss[0])
    return torch.cat(out), torch.cat(idx), torch.cat(gate), counts[0], loss[0]


def run_one_gpu(sm, wl, dev, flags=0):
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    cfg = sm.config(T, d, F, N, wl.capacity_factor, alpha=wl.alpha, flags=flags)
    ws = sm.workspace(cfg)
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(T, **I32)
    gate = torch.empty(T, dtype=torch.float32, device="cuda")
    counts = torch.empty(N, **I32)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    sm.switch_layer_forward(cfg, dev["x"], dev["w_r"], dev["b_r"], dev["w1"], dev["w2"], out, idx,
                            gate, counts, loss, ws)
    _ok(sm, ws)
    return out, idx, gate, counts, loss


def _dev(inp):
    return {"x": dev_float(inp.x), "w_r": dev_float(inp.w_r),
            "b_r": None if inp.b_r is None else dev_float(inp.b_r),
            "w1": dev_float(inp.w1), "w2": dev_float(inp.w2)}


CASES = [
    (Workload("ep_g2", T=2048, d_model=256, d_ff=512, n_experts=8, capacity_factor=1.0,
              dtype="bf16", seed=81), 2, 0),
    (Workload("ep_g4_drops", T=4096, d_model=256, d_ff=512, n_experts=16,
              capacity_factor=0.5, dtype="bf16", seed=82), 4, 0),
    (Workload("ep_g4_zipf", T=4096, d_model=320, d_ff=576, n_experts=8, capacity_factor=1.25,
              dtype="bf16", zipf_s=1.1, seed=83), 4, 0),
    (Workload("ep_g2_nores", T=2048, d_model=256, d_ff=512, n_experts=8, capacity_factor=1.0,
              dtype="bf16", seed=84), 2, 16),          # SWITCH_FLAG_NO_RESIDUAL
    (Workload("ep_g2_pairs", T=2048, d_model=256, d_ff=512, n_experts=8, capacity_factor=1.0,
              dtype="bf16", seed=85), 2, 64),          # SWITCH_FLAG_GEMM_PAIRS
    (Workload("ep_g8_simt", T=2048, d_model=128, d_ff=256, n_experts=16, capacity_factor=1.0,
              dtype="bf16", seed=86), 8, 1),           # SWITCH_FLAG_ROUTER_SIMT
    (Workload("ep_g1", T=1024, d_model=128, d_ff=256, n_experts=4, capacity_factor=1.0,
              dtype="bf16", seed=87), 1, 0),
]


@pytest.mark.parametrize("wl,G,flags", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_ep_equals_one_gpu(sm, wl, G, flags):
    inp = make_inputs(wl)
    dev = _dev(inp)
    out, idx, gate, counts, loss = run_ep_simulated(sm, wl, dev, G, flags)
    out1, idx1, gate1, counts1, loss1 = run_one_gpu(sm, wl, dev, flags)
    assert torch.equal(idx, idx1) and torch.equal(gate, gate1)
    assert torch.equal(counts, counts1)
    assert torch.equal(out.view(torch.int16), out1.view(torch.int16)), "outputs differ"
    assert torch.equal(loss, loss1)
    # and the oracle: routing, counts of the whole batch
    ig = idx.cpu().numpy().astype(np.int64)
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    check_routing(ig, r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(ig, wl.n_experts, C)
    np.testing.assert_array_equal(counts.cpu().numpy(), dsp["counts"])


def test_ep_ragged_rank_tiles(sm):
    """T / G not a multiple of 128: outputs still equal the one-GPU layer bit
    for bit; the loss's per-part sums split differently (fp32 order only)."""
    wl = Workload("ep_ragged", T=2000, d_model=256, d_ff=512, n_experts=8,
                  capacity_factor=1.0, dtype="bf16", seed=88)
    dev = _dev(make_inputs(wl))
    out, idx, gate, counts, loss = run_ep_simulated(sm, wl, dev, 2)
    out1, idx1, gate1, counts1, loss1 = run_one_gpu(sm, wl, dev)
    assert torch.equal(idx, idx1) and torch.equal(counts, counts1)
    assert torch.equal(out.view(torch.int16), out1.view(torch.int16))
    assert abs(loss.item() - loss1.item()) <= 1e-6 * abs(loss1.item())


def test_ep_expert_term_against_oracle(sm):
    """The expert term alone (no residual) of the simulated ranks, on every
    kept token, against the oracle relative to its RMS."""
    wl = Workload("ep_term", T=4096, d_model=256, d_ff=512, n_experts=16,
                  capacity_factor=1.0, dtype="bf16", seed=89)
    inp = make_inputs(wl)
    out, idx, _, _, _ = run_ep_simulated(sm, wl, _dev(inp), 4, 16)
    ig = idx.cpu().numpy().astype(np.int64)
    r = orc.router(inp.x, inp.w_r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(ig, wl.n_experts, C)
    g = r["probs"][np.arange(wl.T), ig]
    Y = orc.expert_ffn(inp.x, inp.w1, inp.w2, dsp["slot_token"], dsp["counts"], C)
    want = orc.combine(inp.x, ig, dsp["rank"], dsp["drop"], g, Y, residual=False)
    got = host_f64(out)
    kept = ~dsp["drop"]
    assert bf16_rms_excess(got[kept], want[kept]) <= BF16_RMS_TOL
    assert (got[dsp["drop"]] == 0).all()


@pytest.mark.slow
def test_ep_base_eight_ranks(sm):
    """The Base workload split over 8 simulated ranks (16 experts and 8192
    tokens each) equals the one-GPU layer bit for bit."""
    wl = WORKLOADS["base"]
    dev = _dev(make_inputs(wl))
    out, idx, gate, counts, loss = run_ep_simulated(sm, wl, dev, 8)
    out1, idx1, gate1, counts1, loss1 = run_one_gpu(sm, wl, dev)
    assert torch.equal(idx, idx1) and torch.equal(counts, counts1)
    assert torch.equal(out.view(torch.int16), out1.view(torch.int16))
    assert torch.equal(loss, loss1)

