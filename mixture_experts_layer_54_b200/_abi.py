"""ctypes declarations of the C ABI in include/moe_b200.h (marshalling only).

Loading fails loudly when libmoe_b200.so is missing: there is no fallback
implementation anywhere in this package.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_NULL = 1
MOE_ERR_SHAPE = 2
MOE_ERR_CAPACITY_FACTOR = 3
MOE_ERR_ALIGN = 4
MOE_ERR_WORKSPACE = 5
MOE_ERR_DTYPE = 6
MOE_ERR_CUDA = 7
MOE_ERR_DEVICE_TIMEOUT = 8

MOE_ROW_ALIGN = 128


class MoeConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d", "E", "k", "d_ff", "n_shared", "d_ff_shared", "act", "score", "renorm",
                 "dtype", "priority")] + [("capacity_factor", ctypes.c_double)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("W_r", "logit_bias", "select_bias", "W1", "W3", "W2", "Ws1", "Ws3", "Ws2")]


class MoeOutputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("y", "topk_idx", "gates", "keep", "dropped", "counts", "n_dropped", "aux",
                 "zloss")]


# name -> (restype, argtypes)
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfig)
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_validate": (ctypes.c_int, [_CFG]),
    "moe_capacity_value": (ctypes.c_int, [_CFG, ctypes.POINTER(ctypes.c_int64)]),
    "moe_perm_rows": (ctypes.c_int64, [_CFG]),
    "moe_loss_partials_count": (ctypes.c_int64, [_CFG]),
    "moe_stage_workspace_size": (ctypes.c_size_t, [_CFG]),
    "moe_workspace_size": (ctypes.c_size_t, [_CFG]),
    "moe_route": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                 _P]),
    "moe_capacity": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                    _P]),
    "moe_capacity_noalloc": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_capacity_scored": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           ctypes.c_size_t, _P]),
    "moe_capacity_sharded": (ctypes.c_int, [_CFG, ctypes.c_int64, _P, ctypes.c_int32,
                                            ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P,
                                            _P, ctypes.c_size_t, _P]),
    "moe_seq_balance_loss": (ctypes.c_int, [_CFG, ctypes.c_int32, _P, _P, _P, _P, _P]),
    "moe_bias_update": (ctypes.c_int, [_CFG, _P, ctypes.c_float, _P, _P]),
    "moe_dispatch": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch_rows": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn_gather": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                             _P, ctypes.c_size_t, _P]),
    "moe_expert_ffn": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                      ctypes.c_size_t, _P]),
    "moe_expert_ffn_slots": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_combine_slots": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P]),
    "moe_losses": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_CFG, ctypes.POINTER(MoeWeights), _P,
                                   ctypes.POINTER(MoeOutputs), _P, ctypes.c_size_t, _P]),
    "moe_device_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
    "moe_clear_device_status": (ctypes.c_int, [_P, _P]),
    "moe_probe_wait_timeout": (ctypes.c_int, [_P, ctypes.c_uint64, _P]),
}

_lib = None


def lib():
    """The loaded library; raises ImportError if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m mixture_experts_layer_54_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        text = lib().moe_status_string(status).decode()
        super().__init__(f"{where}: {text} (status {status})")


class CapacityFactorError(MoEError, ValueError):
    """capacity_factor < 1.0: the layer would drop tokens under perfect balance."""


def check(status: int, where: str):
    if status == MOE_OK:
        return
    if status == MOE_ERR_CAPACITY_FACTOR:
        raise CapacityFactorError(status, where)
    raise MoEError(status, where)
