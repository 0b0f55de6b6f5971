"""switch_dispatch_noalloc: dispatch for callers that cannot allocate device
memory (an engine plugin handed only its tensors and a stream, or a serving
loop that must not call cudaMalloc after start-up).  Its scratch is a fixed
array inside the library, so its results must match switch_dispatch, which
uses a caller workspace, bit for bit -- on two calls in a row, since the
array keeps the previous call's contents.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle.switch_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    from sparse_mixture_experts_switch_b200 import switch_moe
    return switch_moe


def _outputs(T, N, C, dev="cuda"):
    return (torch.full((T,), -7, dtype=torch.int32, device=dev),
            torch.full((T,), 9, dtype=torch.uint8, device=dev),
            torch.full((N,), -7, dtype=torch.int32, device=dev),
            torch.full((max(N * C, 1),), -7, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("source", ["idx", "probs"])
def test_noalloc_dispatch_matches_workspace_dispatch(sm, source):
    cases = [(65536, 128, 1.25, 1), (3001, 16, 0.4, 2)]     # two calls in a row
    for T, N, cf, seed in cases:
        rng = np.random.default_rng(seed)
        probs = rng.dirichlet(np.full(N, 0.5), size=T).astype(np.float32)
        idx = np.argmax(probs, axis=1).astype(np.int32)
        cfg = sm.config(T, 64, 64, N, cf)
        C = sm.switch_capacity(T, N, cf)
        i_dev = torch.from_numpy(idx).cuda() if source == "idx" else None
        p_dev = torch.from_numpy(probs).cuda() if source == "probs" else None
        ws = sm.workspace(cfg)
        want = _outputs(T, N, C)
        sm.switch_dispatch(cfg, i_dev, p_dev, *want, None, None, ws)
        got = _outputs(T, N, C)
        sm.switch_dispatch_noalloc(cfg, i_dev, p_dev, *got)
        torch.cuda.synchronize()
        st, _, _ = sm.switch_get_device_error(ws)
        assert st == 0
        for w, g in zip(want, got):
            assert torch.equal(w, g)
        assert int(got[2].sum()) == T
        # and the oracle's dispatch of the same choices, bit for bit
        ref = orc.dispatch(idx, N, C)
        np.testing.assert_array_equal(got[0].cpu().numpy(), ref["rank"])
        np.testing.assert_array_equal(got[1].cpu().numpy().astype(bool), ref["drop"])
        np.testing.assert_array_equal(got[2].cpu().numpy(), ref["counts"])
        np.testing.assert_array_equal(got[3].cpu().numpy(), ref["slot_token"])


def test_noalloc_rejects_sizes_beyond_its_array(sm):
    T, N = 131072 + 128, 4
    cfg = sm.config(T, 64, 64, N, 1.0)
    C = sm.switch_capacity(T, N, 1.0)
    out = _outputs(T, N, C)
    idx = torch.zeros(T, dtype=torch.int32, device="cuda")
    with pytest.raises(sm.SwitchError) as ei:
        sm.switch_dispatch_noalloc(cfg, idx, None, *out)
    assert ei.value.status == 2          # SWITCH_ERR_UNSUPPORTED, nothing launched
    assert (out[0] == -7).all()
