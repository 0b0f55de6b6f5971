"""Named workloads: the shapes of the synthetic Switch-FFN layers.

Shapes only; nothing here computes any stage of the layer.  The shapes stand
in for the Switch-Base / Switch-Large / Switch-XXL style layers of
"Switch Transformers: scaling to trillion-parameter models" (sections "The
Architecture in Place" and "Scaling to a Trillion Parameters", model table);
no dataset is involved.
"""
from dataclasses import dataclass, replace
from typing import Optional


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # tokens in the batch (one routing group)
    d_model: int
    d_ff: int
    n_experts: int
    capacity_factor: float
    dtype: str             # "bf16" (x, W1, W2, out) or "f32"
    alpha: float = 0.01
    zipf_s: Optional[float] = None   # per-expert router bias following Zipf(s)
    seed: int = 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny", T=512, d_model=64, d_ff=256, n_experts=4,
                capacity_factor=1.25, dtype="f32", seed=1000)
BASE = Workload("base", T=65536, d_model=768, d_ff=3072, n_experts=128,
                capacity_factor=1.25, dtype="bf16", seed=1001)
ZIPF_100 = Workload("zipf_cf1.0", T=32768, d_model=768, d_ff=3072, n_experts=64,
                    capacity_factor=1.0, dtype="bf16", zipf_s=1.1, seed=1002)
ZIPF_125 = ZIPF_100.with_(name="zipf_cf1.25", capacity_factor=1.25)
ZIPF_200 = ZIPF_100.with_(name="zipf_cf2.0", capacity_factor=2.0)
LARGE = Workload("large", T=32768, d_model=1024, d_ff=4096, n_experts=128,
                 capacity_factor=1.0, dtype="bf16", seed=1003)
XXL = Workload("xxl", T=16384, d_model=4096, d_ff=10240, n_experts=64,
               capacity_factor=1.25, dtype="bf16", seed=1004)

WORKLOADS = {w.name: w for w in
             (TINY, BASE, ZIPF_100, ZIPF_125, ZIPF_200, LARGE, XXL)}

# A smaller case with Base's per-expert shape (half the tokens and half the
# experts: the same capacity and tile shapes), for counter captures that
# replay a kernel many times; not one of the benchmark's workloads.
BASE_E64 = BASE.with_(name="base_e64", T=32768, n_experts=64, seed=1005)
PROFILE_WORKLOADS = {w.name: w for w in (BASE_E64,)}
