"""Plain CPU oracle for the token-choice MoE forward pass.

TEST INFRASTRUCTURE ONLY.  Tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package; the
product path (the CUDA library and its binding) never does, and this package
imports nothing from the product.

The arithmetic lives in ``moe_oracle.c`` (double precision, per token, in the
pages' order); this module only marshals numpy arrays into it, plus two host
helpers that are plain counting: ``capacity`` and ``moe_param_counts``.

Sources, by page title:
  "Lab 18 - Mixture of experts" (sections 1-4, "What to implement"),
  "Lab 01 - Router, Load Balancing, Capacity & the MoE Layer" ("The traps"),
  "Mixture of Experts - parameters without the FLOPs" (section 2).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

F32, BF16 = 0, 1
_ERRORS = {2: "bad shape", 3: "capacity factor must be >= 1.0"}


class OracleError(ValueError):
    """Raised where the pages say the operation must fail (e.g. cf < 1)."""


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (OpenMP over tokens in the FFN loop)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_route.argtypes = [I, I, I, I, I, I, P, I, P, P, P, P, P, P, P, P]
        lib.oracle_capacity_value.argtypes = [I, I, I, ctypes.c_double, P]
        lib.oracle_capacity.argtypes = [I, I, I, ctypes.c_double, I, P, P, P, P, P, P, P]
        lib.oracle_capacity_walk.argtypes = [I, I, I, ctypes.c_int64, I, P, P, P, P, P, P]
        lib.oracle_losses.argtypes = [I, I, I, I, P, P, P, P, P]
        lib.oracle_ffn_tokens.argtypes = [I, I, I, I, I, I, I, I, P, I, P, P, P,
                                          P, P, P, P, P, P, I, P, I, P]
        lib.oracle_num_threads.argtypes = []
        lib.oracle_capacity_walk_scored.argtypes = [I, I, I, ctypes.c_int64, P, P, P, P, P, P,
                                                    P]
        lib.oracle_seq_losses.argtypes = [I, I, I, I, I, P, P, P, P]
        lib.oracle_bias_update.argtypes = [I, I, I, P, ctypes.c_float, P, P]
        for f in (lib.oracle_route, lib.oracle_capacity_value, lib.oracle_capacity,
                  lib.oracle_capacity_walk, lib.oracle_capacity_walk_scored,
                  lib.oracle_seq_losses, lib.oracle_bias_update,
                  lib.oracle_losses, lib.oracle_ffn_tokens, lib.oracle_num_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _check(status: int):
    if status != 0:
        raise OracleError(_ERRORS.get(status, f"oracle status {status}"))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _storage(a):
    """Return (contiguous array, dtype code).  bf16 arrives as uint16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {a.dtype}")


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------- router

@dataclass
class Route:
    z: np.ndarray        # [T, E] float64 logits
    scores: np.ndarray   # [T, E] float64: softmax p, or sigmoid s
    topk: np.ndarray     # [T, k] int32, best first
    gates: np.ndarray    # [T, k] float64
    lse: np.ndarray      # [T] float64 log-sum-exp of the logits


def route(x, W_r, k: int, score: int = 0, renorm: int = -1, logit_bias=None,
          select_bias=None) -> Route:
    """Router of "Lab 18" section 1 (z = x W_r, softmax, top-k, gates).

    score 0 = softmax, 1 = sigmoid with optional selection-only bias (the
    DeepSeek-V3 note in section 1 and the auxiliary-loss-free paragraph of
    section 2).  renorm -1 renormalizes exactly when k > 1.
    """
    x, xdt = _storage(x)
    T, d = x.shape
    W_r = np.ascontiguousarray(W_r, dtype=np.float32)
    E = W_r.shape[1]
    assert W_r.shape[0] == d
    lb = None if logit_bias is None else np.ascontiguousarray(logit_bias, dtype=np.float32)
    sb = None if select_bias is None else np.ascontiguousarray(select_bias, dtype=np.float32)
    z = np.empty((T, E), np.float64)
    s = np.empty((T, E), np.float64)
    topk = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    lse = np.empty((T,), np.float64)
    _check(_load().oracle_route(T, d, E, k, score, renorm, _ptr(x), xdt, _ptr(W_r), _ptr(lb),
                                _ptr(sb), _ptr(z), _ptr(s), _ptr(topk), _ptr(gates), _ptr(lse)))
    return Route(z, s, topk, gates, lse)


# ------------------------------------------------------------------------- capacity

def capacity(T: int, E: int, k: int, cf: float) -> int:
    """C = ceil(cf * T * k / E) ("Lab 18" section 3); cf < 1 raises ("Lab 01" traps)."""
    C = ctypes.c_int64()
    _check(_load().oracle_capacity_value(T, E, k, float(cf), ctypes.byref(C)))
    return int(C.value)


@dataclass
class Capacity:
    C: int
    counts: np.ndarray   # [E] int32, before any drop
    pos: np.ndarray      # [T, k] int32 queue position in the expert
    keep: np.ndarray     # [T, k] uint8
    dropped: np.ndarray  # [T] uint8, every slot dropped
    n_dropped: int       # dropped assignments


def capacity_walk(topk, E: int, cf: float | None = None, priority: int = 0,
                  C: int | None = None, sel_scores=None) -> Capacity:
    """Priority-order walk with one counter per expert ("Lab 18" section 3).

    C comes from the capacity factor cf, or is given directly as the pages'
    capacity_mask takes it.
    priority 0 = token order, first come first served ("Lab 01" step 4);
    priority 1 = rank-major (GShard, "Lab 18" section 3);
    priority 2 = batch-prioritized (V-MoE, "Lab 18" section 3): highest router
                 score first, ties in token then slot order; sel_scores [T, k]
                 are the scores of the selected experts, taken as fp32.
    """
    topk = np.ascontiguousarray(topk, dtype=np.int32)
    T, k = topk.shape
    if C is None:
        C = capacity(T, E, k, cf)
    nd = ctypes.c_int64()
    counts = np.empty((E,), np.int32)
    pos = np.empty((T, k), np.int32)
    keep = np.empty((T, k), np.uint8)
    dropped = np.empty((T,), np.uint8)
    if priority == 2:
        sel = np.ascontiguousarray(sel_scores, dtype=np.float32)
        assert sel.shape == (T, k)
        _check(_load().oracle_capacity_walk_scored(T, E, k, int(C), _ptr(topk), _ptr(sel),
                                                   _ptr(counts), _ptr(pos), _ptr(keep),
                                                   _ptr(dropped), ctypes.byref(nd)))
    else:
        _check(_load().oracle_capacity_walk(T, E, k, int(C), priority, _ptr(topk),
                                            _ptr(counts), _ptr(pos), _ptr(keep), _ptr(dropped),
                                            ctypes.byref(nd)))
    return Capacity(int(C), counts, pos, keep, dropped, int(nd.value))


def selected_scores(scores, topk) -> np.ndarray:
    """The router score of each selected expert, [T, k], rounded to fp32 (the
    precision the batch-prioritized ranking is taken in)."""
    scores = np.asarray(scores)
    topk = np.asarray(topk)
    return np.take_along_axis(scores, topk.astype(np.int64), axis=1).astype(np.float32)


# --------------------------------------------------------------------------- losses

def losses(scores, counts, lse, k: int, score: int = 0):
    """(L_aux, L_z) of "Lab 18" section 2, without the alpha coefficients."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    T, E = scores.shape
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    lse = np.ascontiguousarray(lse, dtype=np.float64)
    aux = ctypes.c_double()
    zl = ctypes.c_double()
    _check(_load().oracle_losses(T, E, k, score, _ptr(scores), _ptr(counts), _ptr(lse),
                                 ctypes.byref(aux), ctypes.byref(zl)))
    return float(aux.value), float(zl.value)


def seq_losses(scores, topk, k: int, L: int, score: int = 0):
    """Sequence-wise balance loss: the Switch loss per sequence of L tokens,
    averaged over the T / L sequences (the balancing unit variant of the cs336
    lecture 4 field map, "Training a router you cannot differentiate").
    Returns (mean, per_sequence values)."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    T, E = scores.shape
    topk = np.ascontiguousarray(topk, dtype=np.int32)
    assert topk.shape == (T, k)
    if L < 1 or T % L:
        raise OracleError("bad shape")
    mean = ctypes.c_double()
    per = np.empty((T // L,), np.float64)
    _check(_load().oracle_seq_losses(T, E, k, score, L, _ptr(scores), _ptr(topk),
                                     ctypes.byref(mean), _ptr(per)))
    return float(mean.value), per


def bias_update(counts, T: int, k: int, gamma: float, bias) -> np.ndarray:
    """DeepSeek-V3 auxiliary-loss-free balancing step ("Lab 18" section 2):
    the selection bias of an overloaded expert moves down by gamma, of an
    underloaded one up by gamma, in fp32."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    E = counts.shape[0]
    bias = np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty((E,), np.float32)
    _check(_load().oracle_bias_update(T, E, k, _ptr(counts), ctypes.c_float(gamma), _ptr(bias),
                                      _ptr(out)))
    return out


# ------------------------------------------------------------------------------ FFN

def ffn_tokens(x, topk, gates, keep, W1, W3, W2, act: int, Ws1=None, Ws3=None, Ws2=None,
               tokens=None) -> np.ndarray:
    """y rows for the listed tokens ("Lab 18" section 1: sum of gated expert FFNs).

    x [T, d]; W1/W3 [E, F, d]; W2 [E, d, F]; Ws1/Ws3 [S, Fs, d]; Ws2 [S, d, Fs];
    all float32 or bf16-as-uint16 (weights share one storage type).
    act 0 = GELU two-matrix MLP, 1 = SwiGLU three-matrix FFN.
    """
    x, xdt = _storage(x)
    T, d = x.shape
    topk = np.ascontiguousarray(topk, dtype=np.int32)
    k = topk.shape[1]
    gates = np.ascontiguousarray(gates, dtype=np.float64)
    keep = None if keep is None else np.ascontiguousarray(keep, dtype=np.uint8)
    W1, wdt = _storage(W1)
    E, F, _ = W1.shape
    W2, wdt2 = _storage(W2)
    W3v = None
    if act == 1:
        W3v, wdt3 = _storage(W3)
        assert wdt3 == wdt
    assert wdt2 == wdt
    S = 0 if Ws1 is None else Ws1.shape[0]
    Fs = 0 if Ws1 is None else Ws1.shape[1]
    Ws1v = Ws3v = Ws2v = None
    if S:
        Ws1v, _ = _storage(Ws1)
        Ws2v, _ = _storage(Ws2)
        if act == 1:
            Ws3v, _ = _storage(Ws3)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    y = np.empty((len(tokens), d), np.float64)
    _check(_load().oracle_ffn_tokens(T, d, E, k, F, act, S, Fs, _ptr(x), xdt, _ptr(topk),
                                     _ptr(gates), _ptr(keep), _ptr(W1), _ptr(W3v), _ptr(W2),
                                     _ptr(Ws1v), _ptr(Ws3v), _ptr(Ws2v), wdt, _ptr(tokens),
                                     len(tokens), _ptr(y)))
    return y


# -------------------------------------------------------------------------- forward

@dataclass
class Forward:
    route: Route
    cap: Capacity
    aux: float
    zloss: float
    y: np.ndarray        # [n_tokens, d] float64 (rows of `tokens`, all tokens by default)
    tokens: np.ndarray


def forward(x, W_r, W1, W3, W2, *, k: int, act: int, cf: float, score: int = 0,
            renorm: int = -1, priority: int = 0, logit_bias=None, select_bias=None,
            Ws1=None, Ws3=None, Ws2=None, tokens=None, capacity_override=None) -> Forward:
    """MoE.forward of "Lab 18" ("What to implement" row 5), returning y (not x + y)."""
    r = route(x, W_r, k, score, renorm, logit_bias, select_bias)
    E = np.asarray(W_r).shape[1]
    sel = selected_scores(r.scores, r.topk) if priority == 2 else None
    cap = capacity_walk(r.topk, E, cf, priority, C=capacity_override, sel_scores=sel)
    aux, zl = losses(r.scores, cap.counts, r.lse, k, score)
    if tokens is None:
        tokens = np.arange(np.asarray(x).shape[0], dtype=np.int32)
    y = ffn_tokens(x, r.topk, r.gates, cap.keep, W1, W3, W2, act, Ws1, Ws3, Ws2, tokens)
    return Forward(r, cap, aux, zl, y, np.asarray(tokens))


# --------------------------------------------------------------- parameter counting

def moe_param_counts(d: int, d_ff: int, n_experts: int, k: int, n_shared: int = 0,
                     d_ff_shared: int | None = None, matrices: int = 2,
                     router: bool | None = None):
    """(total, active) parameters of one MoE layer ("Lab 18" section 1 table).

    Experts have `matrices` weight matrices of d x d_ff and no biases (2 = GELU
    MLP, 3 = SwiGLU).  The router (d x E) is counted in both totals for a layer
    with more than one expert; a single expert with k = 1 is the dense FFN.
    """
    if router is None:
        router = n_experts > 1
    d_ff_shared = d_ff if d_ff_shared is None else d_ff_shared
    per_expert = matrices * d * d_ff
    per_shared = matrices * d * d_ff_shared
    r = d * n_experts if router else 0
    total = n_experts * per_expert + n_shared * per_shared + r
    active = k * per_expert + n_shared * per_shared + r
    return total, active


def sparsity_ratio(d: int, d_ff: int, n_experts: int, k: int, matrices: int = 2) -> float:
    """Active over total routed-expert parameters: k/E, exactly 1.0 when k == E
    ("Lab 01" traps)."""
    _, active = moe_param_counts(d, d_ff, n_experts, k, 0, matrices=matrices, router=False)
    total, _ = moe_param_counts(d, d_ff, n_experts, k, 0, matrices=matrices, router=False)
    return active / total


__all__ = ["build", "route", "capacity", "capacity_walk", "losses", "ffn_tokens", "forward",
           "moe_param_counts", "sparsity_ratio", "OracleError", "num_threads"]
