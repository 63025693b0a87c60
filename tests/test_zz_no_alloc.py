"""moe_capacity_noalloc: the capacity stage for callers that cannot allocate
device memory, with its scratch in a static device array inside the library.

Its results must equal moe_capacity's (the workspace version) exactly, on two
calls in a row: the second call runs on the array the first one left behind.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_54_b200 as moe


def _topk(T, E, k, seed):
    rng = np.random.default_rng(seed)
    w = 1.0 / np.arange(1, E + 1) ** 1.1
    return np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum())
                     for _ in range(T)]).astype(np.int32)


def _same(a, b):
    for name in ("counts", "pos", "keep", "kept", "offsets", "dropped", "n_dropped"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


@pytest.mark.parametrize("priority", [0, 1])
def test_noalloc_capacity_matches_the_workspace_version_on_two_calls(priority):
    calls = [(4096, 64, 6, 1.25, 1), (1000, 8, 2, 1.0, 2)]   # second call is smaller
    for T, E, k, cf, seed in calls:
        cfg = moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=cf, priority=priority)
        topk = torch.tensor(_topk(T, E, k, seed + priority), device="cuda")
        ref = moe.moe_capacity(cfg, topk)
        got = moe.moe_capacity_noalloc(cfg, topk)
        torch.cuda.synchronize()
        _same(got, ref)
        assert int(got.n_dropped.item()) > 0


def test_noalloc_capacity_rejects_shapes_beyond_its_static_scratch():
    # ceil(T/256) * k * E > 65536 entries of the histogram table
    cfg = moe.moe_config(T=256 * 40, d=64, E=256, k=8, d_ff=64, dtype=1, cf=1.0)
    topk = torch.zeros((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_capacity_noalloc(cfg, topk)
    assert ei.value.status == 5   # MOE_ERR_WORKSPACE
