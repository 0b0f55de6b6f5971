"""The seeded input generator: encodings, determinism and the stated recipe."""
import numpy as np
import torch

from switch_inputs import (TINY, BASE, WORKLOADS, f32_to_bf16_bits, bf16_bits_to_f32,
                           make_x, make_router, make_expert_w1, make_expert_w2,
                           zipf_law)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0, -2.5, 1 + 2**-8, 1 + 3 * 2**-9, 3.0e38,
                                  1e-40, 0.0, -0.0], np.float32)])
    ours = f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_deterministic_and_per_expert():
    wl = TINY.with_(T=64)
    np.testing.assert_array_equal(make_x(wl), make_x(wl))
    np.testing.assert_array_equal(make_expert_w1(wl, 2), make_expert_w1(wl, 2))
    assert not np.array_equal(make_expert_w1(wl, 1), make_expert_w1(wl, 2))
    assert not np.array_equal(make_x(wl), make_x(wl.with_(seed=wl.seed + 1)))


def test_truncated_normal_scale():
    wl = BASE.with_(n_experts=4)
    w_r, b_r = make_router(wl)
    assert b_r is None and w_r.dtype == np.float32
    sd = np.sqrt(0.1 / wl.d_model)
    assert np.abs(w_r).max() <= 2 * sd * (1 + 1e-6)
    # std of a normal truncated at 2 sigma is 0.8796 sigma
    assert abs(w_r.std() / sd - 0.8796) < 0.02
    w2 = bf16_bits_to_f32(make_expert_w2(wl, 0))
    sd2 = np.sqrt(0.1 / wl.d_ff)
    assert w2.shape == (wl.d_model, wl.d_ff)
    assert np.abs(w2).max() <= 2 * sd2 * (1 + 2**-8)


def test_zipf_bias_orders_experts():
    wl = WORKLOADS["zipf_cf1.0"]
    w_r, b_r = make_router(wl)
    assert b_r is not None and b_r.shape == (wl.n_experts,)
    assert (np.diff(b_r) < 0).all()          # expert 0 has the largest bias
    z = zipf_law(wl.n_experts, 1.1)
    assert abs(z[0] - 0.2505) < 5e-4
