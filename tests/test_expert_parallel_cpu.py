"""Expert parallelism on the CPU: the host side of the protocol.

* The library's host-side checks of an expert-parallel group (sizes,
  rejected configurations) through the C ABI, no kernel launched.
* Two gloo ranks run ExpertParallelSwitch.forward -- the record all-gather in
  rank order and the barriers -- with the library's calls stood in for by
  the oracle on each rank's own tokens (the kernels need a GPU; they are
  checked on one by tests/test_gpu_expert_parallel.py).  Each rank turns the
  gathered per-expert counts into global batch-order ranks (earlier ranks'
  tokens first); the ranks' results, put together, must equal the oracle's
  dispatch of the concatenated batch bit for bit, and the loss formed from
  the gathered per-part probability sums must equal the oracle's loss on the
  whole batch.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.switch_oracle as orc
from switch_inputs import Workload, make_inputs


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import build
    build.build()
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def test_ep_sizes_and_rejections(sm):
    base = dict(T=256, d_model=128, d_ff=256, n_experts=8, capacity_factor=1.0)
    ok = sm.config(**base)
    ws, rec, recv = sm.switch_ep_sizes(ok, sm.ep(2, 1))
    # record: per-64-token parts of probability sums, then the counts
    assert rec == 16 * ((4 * 8 * 4 + 4 * 8 + 15) // 16)
    C = sm.switch_capacity(2 * 256, 8, 1.0)
    assert recv >= (8 // 2) * C * (128 * 2 + 8)
    assert ws > 0 and ws % 1024 == 0
    assert sm.switch_ep_sizes(sm.config(**{**base, "T": 0}), sm.ep(4, 3))[2] == 0
    for cfg, ep, status in [
        (ok, sm.ep(3, 0), 2),                                   # N % G != 0
        (ok, sm.ep(2, 2), 1),                                   # rank out of range
        (ok, sm.ep(0, 0), 1),
        (ok, sm.ep(32, 0), 1),                                  # more ranks than supported
        (sm.config(**base, flags=sm.FLAG_TOP2), sm.ep(2, 0), 2),
        (sm.config(**base, flags=sm.FLAG_GEMM_1SM), sm.ep(2, 0), 2),
        (sm.config(**base, dtype="f32"), sm.ep(2, 0), 2),
        (sm.config(**{**base, "d_model": 100}), sm.ep(2, 0), 2),
    ]:
        with pytest.raises(sm.SwitchError) as ei:
            sm.switch_ep_sizes(cfg, ep)
        assert ei.value.status == status


class OracleEpLib:
    """The library's expert-parallel calls computed by the oracle on the
    calling rank's tokens (CPU tensors), with the record laid out as the
    library lays it out: per-128-token sums of the probabilities, then the
    per-expert counts.  Row exchange and GEMMs are not stood in for."""

    def __init__(self, real, wl, x_local, rank):
        self.real, self.wl, self.x, self.rank = real, wl, x_local, rank
        self.config, self.ep = real.config, real.ep
        self.switch_ep_sizes = real.switch_ep_sizes

    def _offsets(self, cfg):
        N = cfg.n_experts
        parts_max = (cfg.T + 63) // 64
        return (4 * N * parts_max + 15) // 16 * 16

    def switch_ep_route(self, cfg, ep, x, w_r, b_r, idx, gate, record, ws):
        N, T = cfg.n_experts, cfg.T
        r = orc.router(self.x, w_r.numpy(), None if b_r is None else b_r.numpy())
        local = orc.dispatch(r["idx"], N, 10 ** 9)           # ranks within this rank
        parts = [r["probs"][i:i + 128].sum(axis=0) for i in range(0, T, 128)]
        rec = record.numpy()
        rec[:] = 0
        psum = np.asarray(parts, dtype=np.float32).reshape(-1)
        rec[:psum.nbytes] = psum.view(np.uint8)
        off = self._offsets(cfg)
        rec[off:off + 4 * N] = local["counts"].astype(np.int32).view(np.uint8)
        self.local = {"idx": r["idx"], "rank": local["rank"], "probs": r["probs"]}

    def switch_ep_dispatch(self, cfg, ep, x, records, recv_peers, out, counts, loss, ws):
        N, T, G = cfg.n_experts, cfg.T, ep.world_size
        recs = records.numpy().reshape(G, -1)
        off = self._offsets(cfg)
        table = np.stack([recs[q, off:off + 4 * N].view(np.int32) for q in range(G)])
        nparts = (T + 127) // 128
        psum = np.concatenate([recs[q, :4 * N * nparts].view(np.float32).reshape(nparts, N)
                               for q in range(G)])
        C = self.real.switch_capacity(G * T, N, cfg.capacity_factor)
        before = table[:ep.rank].sum(axis=0)
        e = self.local["idx"]
        grank = before[e] + self.local["rank"]
        total = table.sum(axis=0)
        counts.copy_(torch.from_numpy(total.astype(np.int32)))
        f = total / (G * T)
        P = psum.astype(np.float64).sum(axis=0) / (G * T)
        loss.fill_(float(cfg.alpha * N * np.sum(f * P)))
        self.meta = {"rank": grank, "drop": grank >= C, "idx": e, "C": C}

    def switch_ep_experts(self, *args):
        pass


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WL = Workload("ep_cpu", T=640, d_model=64, d_ff=64, n_experts=4, capacity_factor=0.75,
              dtype="bf16", zipf_s=1.1, seed=91)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_mixture_experts_switch_b200 import switch_moe
        from sparse_mixture_experts_switch_b200.expert_parallel import ExpertParallelSwitch
        inp = make_inputs(WL)
        Tr = WL.T // world
        x_local = inp.x[rank * Tr:(rank + 1) * Tr]
        lib = OracleEpLib(switch_moe, WL, x_local, rank)

        def peer_alloc(shape, dtype, device):
            return torch.zeros(shape, dtype=dtype), [0] * world

        layer = ExpertParallelSwitch(Tr, WL.d_model, WL.d_ff, WL.n_experts,
                                     WL.capacity_factor, alpha=WL.alpha, device="cpu",
                                     peer_alloc=peer_alloc, lib=lib)
        E = WL.n_experts // world
        assert list(layer.experts) == list(range(rank * E, (rank + 1) * E))
        _, loss, counts = layer.forward(None, torch.from_numpy(inp.w_r),
                                        torch.from_numpy(inp.b_r), None, None)
        m = lib.meta
        out[rank] = {"rank": m["rank"].tolist(), "drop": m["drop"].tolist(),
                     "idx": m["idx"].tolist(), "C": m["C"], "loss": float(loss.item()),
                     "counts": counts.tolist()}
    finally:
        dist.destroy_process_group()


def test_ep_protocol_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    inp = make_inputs(WL)
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    C = orc.capacity(WL.T, WL.n_experts, WL.capacity_factor)
    want = orc.dispatch(r["idx"], WL.n_experts, C)
    got_rank = np.concatenate([out[q]["rank"] for q in range(world)])
    got_drop = np.concatenate([out[q]["drop"] for q in range(world)])
    got_idx = np.concatenate([out[q]["idx"] for q in range(world)])
    np.testing.assert_array_equal(got_idx, r["idx"])
    np.testing.assert_array_equal(got_rank, want["rank"])
    np.testing.assert_array_equal(got_drop, want["drop"])
    assert want["drop"].any() and not want["drop"].all()
    loss_want, _, _ = orc.aux_loss(want["counts"], r["probs"], WL.alpha)
    for q in range(world):
        assert out[q]["C"] == C
        assert out[q]["counts"] == want["counts"].tolist()
        assert out[q]["loss"] == pytest.approx(loss_want, rel=1e-6)


def _rank_leaves_main(rank, world, port, out):
    """Both ranks run one step; rank 1 then leaves (between steps, nothing in
    flight); rank 0's next step must end with an error from its first
    collective (the peer's connection closes, or the short process-group
    timeout runs out) instead of waiting for ever."""
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    from sparse_mixture_experts_switch_b200 import switch_moe
    from sparse_mixture_experts_switch_b200.expert_parallel import ExpertParallelSwitch
    inp = make_inputs(WL)
    Tr = WL.T // world
    lib = OracleEpLib(switch_moe, WL, inp.x[rank * Tr:(rank + 1) * Tr], rank)

    def peer_alloc(shape, dtype, device):
        return torch.zeros(shape, dtype=dtype), [0] * world

    layer = ExpertParallelSwitch(Tr, WL.d_model, WL.d_ff, WL.n_experts, WL.capacity_factor,
                                 alpha=WL.alpha, device="cpu", peer_alloc=peer_alloc, lib=lib)
    w_r, b_r = torch.from_numpy(inp.w_r), torch.from_numpy(inp.b_r)
    layer.forward(None, w_r, b_r, None, None)
    if rank == 1:
        out[1] = "left"
        os._exit(0)                      # gone without a goodbye
    import time
    t0 = time.monotonic()
    try:
        layer.forward(None, w_r, b_r, None, None)
        out[0] = "completed"
    except Exception as e:               # noqa: BLE001 -- any collective error counts
        out[0] = f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"
    os._exit(0)


def test_ep_rank_leaving_ends_the_next_step_with_an_error():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.start_processes(_rank_leaves_main, args=(world, port, out), nprocs=world,
                             join=False, start_method="spawn")
    assert ctx.join(timeout=120) or ctx.join(timeout=60), "ranks did not finish"
    assert out[1] == "left"
    assert out[0].startswith("error after"), out[0]
    assert float(out[0].split()[2]) < 60.0
    print(out[0])
