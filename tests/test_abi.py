"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe_b200.h declares, and rejects bad arguments
before launching anything."""
import ctypes
import math
import os
import re

import pytest

import mixture_experts_layer_54_b200 as moe
from mixture_experts_layer_54_b200 import _abi
from moe_inputs import CONFIGS

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moe_b200.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_entry_point():
    names = declared_functions()
    assert "moe_forward" in names and "moe_route" in names and len(names) >= 16
    lib = ctypes.CDLL(_abi.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(_abi.SIGNATURES), set(names) - set(_abi.SIGNATURES)


def test_capacity_factor_below_one_is_rejected():
    cfg = moe.moe_config(CONFIGS["mixtral"], cf=0.99)
    with pytest.raises(moe.CapacityFactorError):
        moe.moe_validate(cfg)
    with pytest.raises(ValueError):
        moe.moe_capacity_value(moe.moe_config(CONFIGS["switch"], cf=float("nan")))


def test_capacity_value_worked_example():
    # "Lab 18 - Mixture of experts", section 3: T=4096, E=8, k=2, cf=1.25 -> 1280
    cfg = moe.moe_config(T=4096, d=1024, E=8, k=2, d_ff=4096, dtype=1, cf=1.25)
    assert moe.moe_capacity_value(cfg) == 1280
    assert moe.moe_capacity_value(moe.moe_config(CONFIGS["deepseek_v3"])) == 4096
    assert moe.moe_capacity_value(moe.moe_config(CONFIGS["deepseekmoe"])) == 2304


def test_capacity_value_is_held_at_T_for_huge_factors():
    # an expert receives at most T assignments; a huge finite factor must not
    # overflow the integer conversion (it keeps everything, like +infinity)
    cfg = moe.moe_config(T=4096, d=1024, E=8, k=2, d_ff=4096, dtype=1, cf=1e20)
    assert moe.moe_capacity_value(cfg) == 4096
    assert moe.moe_capacity_value(moe.moe_config(cfg, cf=1.25, T=10, E=2)) == 10
    assert moe.moe_perm_rows(cfg) == moe.moe_perm_rows(moe.moe_config(cfg, cf=math.inf))


@pytest.mark.parametrize("kw", [dict(k=9, E=8), dict(k=3, E=2), dict(E=300, k=2),
                                dict(d=100), dict(d_ff=100), dict(T=-1)])
def test_bad_shapes_are_rejected(kw):
    base = dict(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0)
    base.update(kw)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_validate(moe.moe_config(**base))
    assert ei.value.status == _abi.MOE_ERR_SHAPE


def test_bad_codes_are_rejected():
    for kw in (dict(act=2), dict(score=5), dict(dtype=3), dict(priority=3), dict(renorm=4)):
        base = dict(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0)
        base.update(kw)
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_validate(moe.moe_config(**base))
        assert ei.value.status == _abi.MOE_ERR_DTYPE


def test_score_priority_is_only_taken_by_the_scored_capacity_call():
    L = moe.lib()
    scored = moe.moe_config(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0, priority=2)
    token = moe.moe_config(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0, priority=0)
    nul = [None] * 8
    assert L.moe_capacity(ctypes.byref(scored), *nul, None, 0, None) == _abi.MOE_ERR_DTYPE
    assert L.moe_capacity_noalloc(ctypes.byref(scored), *nul, None) == _abi.MOE_ERR_DTYPE
    assert L.moe_capacity_scored(ctypes.byref(token), *nul, None, None, 0,
                                 None) == _abi.MOE_ERR_DTYPE
    assert L.moe_capacity_scored(ctypes.byref(scored), *nul, None, None, 0,
                                 None) == _abi.MOE_ERR_NULL
    # the score order needs room for its sort keys
    assert moe.moe_stage_workspace_size(scored) >= moe.moe_stage_workspace_size(token)


def test_seq_loss_and_bias_step_check_their_arguments_before_any_launch():
    L = moe.lib()
    cfg = moe.moe_config(T=256, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0)
    for seq_len in (0, 16, 48, 96, 512):   # not a multiple of 32, or not dividing T
        assert L.moe_seq_balance_loss(ctypes.byref(cfg), seq_len, None, None, None, None,
                                      None) == _abi.MOE_ERR_SHAPE
    assert L.moe_seq_balance_loss(ctypes.byref(cfg), 64, None, None, None, None,
                                  None) == _abi.MOE_ERR_NULL
    assert L.moe_bias_update(ctypes.byref(cfg), None, ctypes.c_float(float("nan")), None,
                             None) == _abi.MOE_ERR_SHAPE
    assert L.moe_bias_update(ctypes.byref(cfg), None, ctypes.c_float(1e-3), None,
                             None) == _abi.MOE_ERR_NULL


def test_sharded_capacity_checks_its_arguments_before_any_launch():
    L = moe.lib()
    tok = moe.moe_config(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0)
    rank = moe.moe_config(T=64, d=128, E=8, k=2, d_ff=128, dtype=1, cf=1.0, priority=1)
    nul = [None] * 8
    args = lambda cfg, C, n, i: (ctypes.byref(cfg), C, None, n, i, *nul, None, 0, None)
    assert L.moe_capacity_sharded(*args(rank, 10, 2, 0)) == _abi.MOE_ERR_DTYPE
    for C, n, i in ((-1, 2, 0), (10, 0, 0), (10, 2, 2), (10, 2, -1)):
        assert L.moe_capacity_sharded(*args(tok, C, n, i)) == _abi.MOE_ERR_SHAPE
    assert L.moe_capacity_sharded(*args(tok, 10, 2, 1)) == _abi.MOE_ERR_NULL


def test_null_pointers_are_rejected_before_any_launch():
    cfg = moe.moe_config(CONFIGS["tiny"])
    L = moe.lib()
    st = L.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None,
                     None, 0, None)
    assert st == _abi.MOE_ERR_NULL
    st = L.moe_forward(ctypes.byref(cfg), None, None, None, None, 0, None)
    assert st == _abi.MOE_ERR_NULL
    small = ctypes.c_void_p(4096)   # never dereferenced: the size check fails first
    ws_need = moe.moe_stage_workspace_size(cfg)
    st = L.moe_capacity(ctypes.byref(cfg), small, small, small, small, small, small, small,
                        small, small, ws_need - 1, None)
    assert st == _abi.MOE_ERR_WORKSPACE


def test_sizes_cover_every_config():
    for name, shape in CONFIGS.items():
        cfg = moe.moe_config(shape)
        R = moe.moe_perm_rows(cfg)
        C = moe.moe_capacity_value(cfg)
        assert R % _abi.MOE_ROW_ALIGN == 0
        assert R >= min(shape.T * shape.k, shape.E * C) + shape.E * (_abi.MOE_ROW_ALIGN - 1)
        assert moe.moe_workspace_size(cfg) > moe.moe_stage_workspace_size(cfg) > 0
        assert moe.moe_loss_partials_count(cfg) == math.ceil(shape.T / 32) * (shape.E + 1)


def test_binding_refuses_views_and_host_tensors_before_calling_the_library():
    """The library reads dense row-major device buffers: the binding refuses a
    strided view (whatever its device) and a host tensor."""
    import torch
    from mixture_experts_layer_54_b200 import ops
    cfg = moe.moe_config(CONFIGS["tiny"])
    W_r = torch.zeros((cfg.d, cfg.E))
    with pytest.raises(ValueError, match="contiguous"):
        moe.moe_route(cfg, torch.zeros((cfg.d, cfg.T)).t(), W_r, ws=torch.zeros(256))
    with pytest.raises(ValueError, match="CUDA"):
        ops._p(torch.zeros(4))
    assert ops._p(None) is None


def test_package_exports_every_binding():
    from mixture_experts_layer_54_b200 import ops
    missing = [n for n in ops.__all__ if not hasattr(moe, n)]
    assert not missing, missing
    assert set(ops.__all__) <= set(moe.__all__), set(ops.__all__) - set(moe.__all__)
