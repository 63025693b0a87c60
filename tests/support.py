"""Shared test helpers: moving seeded inputs into the oracle, and the near-tie
filter that keeps routing decisions far from rounding boundaries.

The filter needs router logits, so it calls the oracle (never the CUDA path)
and redraws rejected rows through ``moe_inputs.resample_rows``.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_inputs import Inputs, resample_rows, SCORE_SIGMOID

# gap below which two neighbouring selection keys count as a near tie
TIE_GAP = 1e-4


def storage(t: torch.Tensor | None):
    """torch tensor -> numpy array the oracle takes (fp32, or bf16 bit patterns)."""
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def oracle_route(inp: Inputs, rows=None) -> oracle.Route:
    s = inp.shape
    x = inp.x if rows is None else inp.x[torch.as_tensor(rows, device=inp.x.device)]
    return oracle.route(storage(x), storage(inp.W_r), s.k, s.score, s.renorm,
                        storage(inp.logit_bias), storage(inp.select_bias))


def selection_keys(inp: Inputs, r: oracle.Route) -> np.ndarray:
    """The keys top-k ranks: router logits for softmax (same order as p), and
    sigmoid score + selection bias for sigmoid routing."""
    if inp.shape.score == SCORE_SIGMOID:
        b = 0.0 if inp.select_bias is None else f64(inp.select_bias)[None, :]
        return r.scores + b
    return r.z


def near_tie_rows(inp: Inputs, r: oracle.Route) -> np.ndarray:
    """Tokens where any two neighbours among the k+1 largest selection keys are
    closer than TIE_GAP (the k-th/(k+1)-th gap decides membership, the others
    the best-first order)."""
    k = inp.shape.k
    keys = selection_keys(inp, r)
    E = keys.shape[1]
    top = -np.sort(-keys, axis=1)[:, : min(k + 1, E)]
    gaps = top[:, :-1] - top[:, 1:]
    if gaps.shape[1] == 0:
        return np.zeros(0, dtype=np.int64)
    return np.nonzero(gaps.min(axis=1) < TIE_GAP)[0]


def remove_near_ties(inp: Inputs, max_rounds: int = 50) -> Inputs:
    """Redraw x rows until no token has a near tie (in place)."""
    for attempt in range(max_rounds):
        rows = near_tie_rows(inp, oracle_route(inp))
        if rows.size == 0:
            return inp
        resample_rows(inp, rows, attempt)
    raise RuntimeError("near ties persist after resampling")


def oracle_forward(inp: Inputs, tokens=None, capacity_override=None) -> oracle.Forward:
    s = inp.shape
    return oracle.forward(storage(inp.x), storage(inp.W_r), storage(inp.W1), storage(inp.W3),
                          storage(inp.W2), k=s.k, act=s.act, cf=s.cf, score=s.score,
                          renorm=s.renorm, priority=s.priority,
                          logit_bias=storage(inp.logit_bias),
                          select_bias=storage(inp.select_bias), Ws1=storage(inp.Ws1),
                          Ws3=storage(inp.Ws3), Ws2=storage(inp.Ws2), tokens=tokens,
                          capacity_override=capacity_override)
