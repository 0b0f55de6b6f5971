"""Helpers for the GPU parity tests: device copies of the seeded inputs and
the tolerances the comparisons use.

Tolerances (stated once):
* integer outputs (expert index, rank, drop, counts, slots): bit-exact;
  end to end, a top-1 choice may differ from the oracle's only on a token
  whose oracle top-1/top-2 probability margin is below 1e-6, and each such
  flip is counted;
* fp32 router probabilities and gates: max relative error 1e-5;
* bf16 expert / combined outputs: max |GPU - oracle| / RMS(oracle) <= 2e-2;
  where the output compared is the expert term alone (no residual, whose
  values spread far beyond their RMS because the gates vary from token to
  token), each element is first allowed the half ulp of bf16 that rounding
  the exact value to the output dtype costs (`bf16_rms_excess`): a
  correctly rounded element 8 RMS from zero is already up to 0.03 RMS off;
* fp32 expert / combined outputs (fp32 FMA, no TF32): the same ratio <= 1e-5;
* load-balancing loss: relative error 1e-5.
"""
import numpy as np
import torch

from switch_inputs import as_f64

PROB_RTOL = 1e-5
MARGIN_FLIP = 1e-6
BF16_RMS_TOL = 2e-2
F32_RMS_TOL = 1e-5
LOSS_RTOL = 1e-5


def dev_float(a, dtype_bits=None):
    """numpy fp32 array, or uint16 bf16 bit patterns, to a CUDA tensor."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_f64(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def rms_ratio(got, want):
    want = np.asarray(want, dtype=np.float64)
    rms = np.sqrt(np.mean(want * want))
    return float(np.max(np.abs(np.asarray(got, np.float64) - want)) / max(rms, 1e-30))


def bf16_half_ulp(want):
    """Half a unit in the last place of bf16 (8 significant bits) at each
    value: the most that rounding the exact value to bf16 moves it."""
    want = np.abs(np.asarray(want, dtype=np.float64))
    _, ex = np.frexp(want)                 # want = m 2^ex, 0.5 <= m < 1
    return np.where(want > 0, np.ldexp(1.0, ex - 9), 0.0)


def bf16_rms_excess(got, want):
    """max over elements of (|got - want| - half bf16 ulp of want), over the
    RMS of want: the error beyond the output's own rounding to bf16."""
    want = np.asarray(want, dtype=np.float64)
    rms = np.sqrt(np.mean(want * want))
    err = np.abs(np.asarray(got, np.float64) - want) - bf16_half_ulp(want)
    return float(max(np.max(err), 0.0) / max(rms, 1e-30))


def check_routing(idx_gpu, r_oracle):
    """Top-1 choice: equal, or a counted flip on a margin < 1e-6 token."""
    idx_gpu = np.asarray(idx_gpu)
    diff = np.nonzero(idx_gpu != r_oracle["idx"])[0]
    bad = diff[r_oracle["margin"][diff] >= MARGIN_FLIP]
    assert bad.size == 0, f"routing differs on {bad.size} tokens with margin >= 1e-6: {bad[:10]}"
    return int(diff.size)


def rel_err(got, want):
    want = np.asarray(want, np.float64)
    return np.abs(np.asarray(got, np.float64) - want) / np.abs(want)


def as_f64_inputs(inp):
    return as_f64(inp.x)
