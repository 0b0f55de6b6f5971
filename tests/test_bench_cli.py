"""bench.py's command line and its profiling workload, on the CPU."""
import sys

import pytest

from switch_inputs import WORKLOADS, PROFILE_WORKLOADS
import oracle.switch_oracle as orc


def _args(monkeypatch, *argv):
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", *argv])
    return bench.parse_args()


def test_stage_choices_cover_every_staged_call(monkeypatch):
    import bench
    for stage in bench.STAGES:
        a = _args(monkeypatch, "--stage", stage, "--workload", "base_e64")
        assert a.stage == stage and a.workload == "base_e64"
    with pytest.raises(SystemExit):
        _args(monkeypatch, "--stage", "no_such_stage")


def test_profile_workload_keeps_base_per_expert_shape():
    """base_e64 halves the tokens and the experts of Base: the capacity, the
    tokens per expert and the GEMM shapes are Base's, so its counters stand
    for Base's kernels."""
    base, small = WORKLOADS["base"], PROFILE_WORKLOADS["base_e64"]
    assert (small.d_model, small.d_ff, small.capacity_factor, small.dtype) == \
        (base.d_model, base.d_ff, base.capacity_factor, base.dtype)
    assert small.T * base.n_experts == base.T * small.n_experts
    assert orc.capacity(small.T, small.n_experts, small.capacity_factor) == \
        orc.capacity(base.T, base.n_experts, base.capacity_factor)
    # not one of the benchmark's workloads (the bench's 'all' list)
    assert "base_e64" not in WORKLOADS


def test_launch_count_matches_the_forward(monkeypatch):
    import bench
    # bf16: weight split, router, scan (+ loss), slots + row copy, GEMM1, GEMM2
    assert bench.launches_per_step(None, WORKLOADS["base"]) == 6
    assert bench.launches_per_step(None, WORKLOADS["tiny"]) == 7


def test_layer_roofline_arithmetic():
    """The bench's layer roofline for Base, by hand: useful FLOPs
    2·T·d·N (router) + 4·T_kept·d·F (the two expert GEMMs) at the bf16 peak,
    against x read three times, every expert weight once and out written
    once at the HBM peak."""
    import bench
    wl = WORKLOADS["base"]
    pk = {"bf16_tflops": 1646.3, "hbm_gbs": 6433.9, "bf16_tflops_sustained": 1394.0}
    T_kept = 65484
    b = bench.layer_bounds(wl, T_kept, pk)
    flops = 2 * 65536 * 768 * 128 + 4 * T_kept * 768 * 3072
    nbytes = 4 * 65536 * 768 * 2 + 2 * 128 * 768 * 3072 * 2
    assert b["useful_flops"] == pytest.approx(flops, rel=1e-12)
    assert b["min_bytes"] == nbytes
    assert b["t_compute_us"] == pytest.approx(flops / 1646.3e12 * 1e6, rel=1e-12)
    assert b["t_mem_us"] == pytest.approx(nbytes / 6433.9e9 * 1e6, rel=1e-12)
    assert b["bound"] == "tensor" and 380 < b["t_compute_us"] < 386 and 248 < b["t_mem_us"] < 252
    row = bench.workload_row(wl, 640, 0.661, 571e-6, T_kept, pk)
    assert row["tokens_per_s"] == pytest.approx(65536 / 0.661e-3)
    assert row["expert_ffn_frac_burst"] == pytest.approx(4 * T_kept * 768 * 3072 / 571e-6
                                                         / 1e12 / 1646.3)
    assert row["padding"] == pytest.approx(1 - T_kept / (128 * 640))
