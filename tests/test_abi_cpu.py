"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and its host-side logic (exact capacity, argument validation,
workspace sizing) answers correctly.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import golden_io

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "switch_moe.h")


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import build
    build.build()
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(switch_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(sm):
    names = _declared()
    assert "switch_layer_forward" in names and len(names) >= 10
    lib = ctypes.CDLL(sm.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"libswitchmoe.so does not export {n}"


def test_capacity_matches_golden(sm):
    for T, N, cf, C in golden_io.capacity_cases():
        assert sm.switch_capacity(T, N, cf) == C, (T, N, cf)


def test_capacity_rejects_bad_input(sm):
    assert sm.switch_capacity(-1, 4, 1.0) == -1
    assert sm.switch_capacity(10, 0, 1.0) == -1
    assert sm.switch_capacity(10, 4, 0.0) == -1
    assert sm.switch_capacity(10, 4, float("nan")) == -1
    assert sm.switch_capacity(10, 4, float("inf")) == -1
    assert sm.switch_capacity(10, 4, 1e-300) == 1


def test_capacity_matches_oracle_on_a_sweep(sm):
    from oracle.switch_oracle import capacity
    for T in (1, 2, 3, 7, 100, 511, 512, 513, 65536, 123457):
        for N in (1, 2, 3, 7, 64, 128, 1000):
            for cf in (0.01, 0.3, 0.5, 1.0, 1.1, 1.25, 1.3, 2.0, 3.7, 64.0):
                assert sm.switch_capacity(T, N, cf) == capacity(T, N, cf), (T, N, cf)


def test_workspace_validation(sm):
    good = sm.config(65536, 768, 3072, 128, 1.25)
    n = sm.switch_workspace_size(good)
    assert n > 128 * 640 * 3072 * 2       # holds the hidden activations
    for bad, status in ((sm.config(1024, 100, 3072, 128, 1.25), 2),          # d % 64
                        (sm.config(1024, 768, 3000, 128, 1.25), 2),          # F % 64
                        (sm.config(1024, 768, 3072, 0, 1.25), 1),            # N < 1
                        (sm.config(1024, 768, 3072, 2000, 1.25), 1),         # N > 1024
                        (sm.config(1024, 768, 3072, 128, -1.0), 1),          # cf <= 0
                        (sm.config(-5, 768, 3072, 128, 1.0), 1),             # T < 0
                        (sm.config(1024, 66, 3072, 128, 1.0, dtype="f32"), 2)):
        with pytest.raises(sm.SwitchError) as ei:
            sm.switch_workspace_size(bad)
        assert ei.value.status == status
    assert sm.switch_workspace_size(sm.config(512, 64, 256, 4, 1.25, dtype="f32")) > 0


def test_backward_workspace_extends_the_forward(sm):
    """The backward's workspace holds the forward's regions and its own
    after them: at least the forward size plus dA [N*C, d_ff] bf16, dh [T, N]
    fp32 and the kept probabilities [T, N] fp32; invalid configs are refused
    the same way."""
    for T, d, F, N, cf in ((65536, 768, 3072, 128, 1.25), (1000, 192, 320, 6, 6.0),
                           (2500, 128, 192, 100, 1.0), (1, 64, 64, 1, 1.0),
                           (16384, 4096, 10240, 64, 1.25)):
        cfg = sm.config(T, d, F, N, cf)
        fwd = sm.switch_workspace_size(cfg)
        bwd = sm.switch_backward_workspace_size(cfg)
        C = sm.switch_capacity(T, N, cf)
        assert bwd >= fwd + N * C * F * 2 + 2 * T * N * 4, (T, d, F, N)
        top2 = sm.config(T, d, F, max(N, 2), cf, flags=sm.FLAG_TOP2)
        assert sm.switch_backward_workspace_size(top2) >= sm.switch_workspace_size(top2)
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_backward_workspace_size(sm.config(1024, 100, 3072, 128, 1.25))
    assert ei.value.status == 2


def test_status_strings(sm):
    for s in range(7):
        assert sm.switch_status_string(s)


def test_binding_flags_match_the_header(sm):
    """Every SWITCH_FLAG_* of the header has the same value in the binding,
    and the binding defines no flag the header does not."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    header = {m.group(1): int(m.group(2))
              for m in re.finditer(r"\bSWITCH_FLAG_([A-Z0-9_]+)\s*=\s*(\d+)", src)}
    binding = {k[len("FLAG_"):]: v for k, v in vars(sm).items()
               if k.startswith("FLAG_") and isinstance(v, int)}
    assert header and header == binding
    assert len(set(header.values())) == len(header)          # distinct bits
    assert all(v & (v - 1) == 0 for v in header.values())    # one bit each
