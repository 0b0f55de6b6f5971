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
