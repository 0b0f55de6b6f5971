"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark."""
from .configs import (Workload, WORKLOADS, PROFILE_WORKLOADS, TINY, BASE, ZIPF_100,  # noqa: F401
                      ZIPF_125, ZIPF_200, LARGE, XXL)
from .generate import (Inputs, make_inputs, make_x, make_dout, make_router, make_w1, make_w2,  # noqa: F401
                       make_expert_w1, make_expert_w2, f32_to_bf16_bits,
                       bf16_bits_to_f32, as_f64, zipf_law, zipf_bias)
