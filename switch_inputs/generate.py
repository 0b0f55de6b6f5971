"""Seeded synthetic inputs for the Switch-FFN layer.

This module is shared by the CPU oracle, the tests and the benchmark.  It
draws random numbers and encodes them (fp32 -> bf16 bit patterns); it holds no
stage of the layer itself (no logits, softmax, routing, capacity, FFN or loss).

Recipe (stated once, used everywhere):

* ``x ~ N(0, 1)``, shape ``[T, d_model]``; rounded once to bf16 (round to
  nearest even) for the bf16 workloads, kept fp32 for the fp32 workload.
* Weights are drawn from a normal of standard deviation ``sqrt(s / fan_in)``
  with ``s = 0.1`` (the 10x-reduced initialisation scale of "Switch
  Transformers: scaling to trillion-parameter models", section "Making Sparse
  Training Stable", smaller initialisation), truncated at two standard
  deviations by redrawing.  ``fan_in`` is ``d_model`` for the router and
  ``W1`` and ``d_ff`` for ``W2``.
* Layouts: ``w_r [N, d_model]`` fp32 (one row per expert); ``w1 [N, d_ff,
  d_model]`` and ``w2 [N, d_model, d_ff]``, each expert's matrix stored
  output-major like a linear layer's ``[out, in]`` weight, so that
  ``E_e(x) = relu(x @ w1[e].T) @ w2[e].T``.  bf16 workloads store ``w1``/``w2``
  as bf16 bit patterns (uint16); the router stays fp32.
* The backward pass's upstream gradient ``dout ~ N(0, 1)``, shape
  ``[T, d_model]``, encoded like x (``make_dout``).
* Workloads with ``zipf_s`` add a router bias ``b_e = beta * ln z_e`` where
  ``z_e`` is the Zipf(s) law over experts (expert 0 heaviest).  ``beta`` is
  fitted so that, with the router's logits modelled as independent Gaussians
  of standard deviation ``||w_r[e]||`` around the bias, expert 0 would win a
  share ``z_0`` of the tokens.  The realised routing is whatever the seeded
  draw gives; tests and the benchmark report it rather than assume it.

Every tensor gets its own ``SeedSequence`` (and every expert of ``w1``/``w2``
its own child), so one expert's weights can be regenerated alone.
"""
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Workload

_TENSOR_IDS = {"x": 1, "w_r": 2, "w1": 3, "w2": 4, "dout": 5}
INIT_SCALE = 0.1


# ----------------------------------------------------------------- encodings

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# ------------------------------------------------------------------ drawing

def _rng(wl: Workload, tensor: str, *sub: int) -> np.random.Generator:
    ss = np.random.SeedSequence([wl.seed, _TENSOR_IDS[tensor], *sub])
    return np.random.Generator(np.random.PCG64(ss))


def _trunc_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    v = rng.standard_normal(size=shape, dtype=np.float32)
    bad = np.abs(v) > 2.0
    while bad.any():
        v[bad] = rng.standard_normal(size=int(bad.sum()), dtype=np.float32)
        bad = np.abs(v) > 2.0
    v *= np.float32(std)
    return v


def make_x(wl: Workload) -> np.ndarray:
    """x as fp32 values (f32 workloads) or bf16 bit patterns (bf16)."""
    rng = _rng(wl, "x")
    x = rng.standard_normal(size=(wl.T, wl.d_model), dtype=np.float32)
    return x if wl.dtype == "f32" else f32_to_bf16_bits(x)


def make_dout(wl: Workload) -> np.ndarray:
    """Upstream gradient of the block output for the backward pass: ``N(0, 1)``
    of shape ``[T, d_model]``, encoded like x (bf16 bits or fp32)."""
    rng = _rng(wl, "dout")
    g = rng.standard_normal(size=(wl.T, wl.d_model), dtype=np.float32)
    return g if wl.dtype == "f32" else f32_to_bf16_bits(g)


def make_router(wl: Workload):
    """(w_r [N, d] fp32, b_r [N] fp32 or None)."""
    rng = _rng(wl, "w_r")
    w_r = _trunc_normal(rng, (wl.n_experts, wl.d_model),
                        np.sqrt(INIT_SCALE / wl.d_model))
    b_r = None if wl.zipf_s is None else zipf_bias(w_r, wl.zipf_s)
    return w_r, b_r


def make_expert_w1(wl: Workload, e: int) -> np.ndarray:
    w = _trunc_normal(_rng(wl, "w1", e), (wl.d_ff, wl.d_model),
                      np.sqrt(INIT_SCALE / wl.d_model))
    return w if wl.dtype == "f32" else f32_to_bf16_bits(w)


def make_expert_w2(wl: Workload, e: int) -> np.ndarray:
    w = _trunc_normal(_rng(wl, "w2", e), (wl.d_model, wl.d_ff),
                      np.sqrt(INIT_SCALE / wl.d_ff))
    return w if wl.dtype == "f32" else f32_to_bf16_bits(w)


def _fill_experts(out: np.ndarray, make_one, wl: Workload) -> np.ndarray:
    """Fill out[e] = make_one(wl, e) for every expert, on a thread pool (each
    expert has its own generator, so the result does not depend on the
    number of threads; numpy releases the GIL while drawing)."""
    from concurrent.futures import ThreadPoolExecutor

    def one(e):
        out[e] = make_one(wl, e)

    workers = max(1, min(wl.n_experts, os.cpu_count() or 1, 32))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(one, range(wl.n_experts)))
    return out


def make_w1(wl: Workload) -> np.ndarray:
    dt = np.float32 if wl.dtype == "f32" else np.uint16
    return _fill_experts(np.empty((wl.n_experts, wl.d_ff, wl.d_model), dtype=dt),
                         make_expert_w1, wl)


def make_w2(wl: Workload) -> np.ndarray:
    dt = np.float32 if wl.dtype == "f32" else np.uint16
    return _fill_experts(np.empty((wl.n_experts, wl.d_model, wl.d_ff), dtype=dt),
                         make_expert_w2, wl)


# ------------------------------------------------------------- zipf bias

def zipf_law(n: int, s: float) -> np.ndarray:
    z = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return z / z.sum()


def _gaussian_top_share(bias: np.ndarray, sd: np.ndarray) -> float:
    """P(expert 0 has the largest of independent N(bias_e, sd_e^2) draws)."""
    from scipy.special import ndtr
    u = np.linspace(-9.0, 9.0, 6001)
    phi = np.exp(-0.5 * u * u) / np.sqrt(2.0 * np.pi)
    arg = (bias[0] - bias[1:, None] + sd[0] * u[None, :]) / sd[1:, None]
    integrand = phi * np.prod(ndtr(arg), axis=0)
    return float(np.trapezoid(integrand, u))


def zipf_bias(w_r: np.ndarray, s: float) -> np.ndarray:
    """Router bias b_e = beta * ln z_e with beta fitted by bisection."""
    n = w_r.shape[0]
    z = zipf_law(n, s)
    lnz = np.log(z)
    sd = np.sqrt(np.sum(w_r.astype(np.float64) ** 2, axis=1))
    lo, hi = 0.0, 1.0
    while _gaussian_top_share(hi * lnz, sd) < z[0]:
        hi *= 2.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if _gaussian_top_share(mid * lnz, sd) < z[0]:
            lo = mid
        else:
            hi = mid
    return (0.5 * (lo + hi) * lnz).astype(np.float32)


# ---------------------------------------------------------------- bundle

@dataclass
class Inputs:
    wl: Workload
    x: np.ndarray                 # [T, d]  f32 or bf16 bits
    w_r: np.ndarray               # [N, d]  f32
    b_r: Optional[np.ndarray]     # [N]     f32 or None
    w1: np.ndarray                # [N, F, d]
    w2: np.ndarray                # [N, d, F]


def make_inputs(wl: Workload) -> Inputs:
    w_r, b_r = make_router(wl)
    return Inputs(wl, make_x(wl), w_r, b_r, make_w1(wl), make_w2(wl))


def as_f64(a: np.ndarray) -> np.ndarray:
    """Values of an input tensor in float64 (decodes bf16 bit patterns)."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)
