"""A second, pure-Python per-token loop over tiny random layers, compared with
the C oracle.  It re-states the same method (so it is a cross-check of the C
code, not a pin of the reading; the pins are in test_oracle_pins.py)."""
import math

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import CONFIGS, generate
from support import oracle_forward, remove_near_ties, storage, near_tie_rows, oracle_route


def py_forward(x, W_r, W1, W3, W2, k, act, C, score=0, sbias=None, priority=0, Ws=None):
    T, d = x.shape
    E = W_r.shape[1]
    topk, gates, scores, lses = [], [], [], []
    for t in range(T):
        z = [sum(float(x[t, c]) * float(W_r[c, e]) for c in range(d)) for e in range(E)]
        m = max(z)
        S = sum(math.exp(v - m) for v in z)
        lses.append(m + math.log(S))
        v = [math.exp(u - m) / S for u in z] if score == 0 else [1 / (1 + math.exp(-u)) for u in z]
        key = [v[e] + (sbias[e] if (score == 1 and sbias is not None) else 0.0) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-key[e], e))[:k]
        tot = sum(v[e] for e in order)
        topk.append(order)
        gates.append([v[e] / tot if k > 1 else v[e] for e in order])
        scores.append(v)
    counter = [0] * E
    keep = [[0] * k for _ in range(T)]
    seq = [(t, j) for t in range(T) for j in range(k)] if priority == 0 else \
          [(t, j) for j in range(k) for t in range(T)]
    for t, j in seq:
        e = topk[t][j]
        keep[t][j] = int(counter[e] < C)
        counter[e] += 1

    def ffn(xt, A, B, Cm, F):
        h = []
        for f in range(F):
            a = sum(float(A[f, c]) * xt[c] for c in range(d))
            if act == 0:
                h.append(0.5 * a * (1 + math.erf(a / math.sqrt(2))))
            else:
                b = sum(float(B[f, c]) * xt[c] for c in range(d))
                h.append(a / (1 + math.exp(-a)) * b)
        return [sum(float(Cm[c, f]) * h[f] for f in range(F)) for c in range(d)]

    y = np.zeros((T, d))
    F = W1.shape[1]
    for t in range(T):
        xt = [float(v) for v in x[t]]
        for j in range(k):
            if keep[t][j]:
                e = topk[t][j]
                o = ffn(xt, W1[e], None if W3 is None else W3[e], W2[e], F)
                y[t] += gates[t][j] * np.array(o)
        if Ws is not None:
            for s in range(Ws[0].shape[0]):
                o = ffn(xt, Ws[0][s], None if Ws[1] is None else Ws[1][s], Ws[2][s], Ws[0].shape[1])
                y[t] += np.array(o)
    f = np.bincount(np.array(topk).reshape(-1), minlength=E) / (T * k)
    sc = np.array(scores)
    if score == 1:
        sc = sc / sc.sum(axis=1, keepdims=True)
    aux = E * float((f * sc.mean(axis=0)).sum())
    zl = float(np.mean(np.array(lses) ** 2))
    return np.array(topk), np.array(gates), np.array(keep), y, aux, zl


@pytest.mark.parametrize("act,score,priority,S", [(0, 0, 0, 0), (1, 0, 1, 0), (1, 1, 0, 1),
                                                   (0, 0, 1, 2)])
def test_c_oracle_agrees_with_python_loop(act, score, priority, S):
    rng = np.random.default_rng(100 + act * 10 + score + priority * 3 + S)
    T, d, E, F, k = 14, 5, 4, 6, 2
    x = rng.normal(size=(T, d)).astype(np.float32)
    W_r = rng.normal(size=(d, E)).astype(np.float32)
    W1 = rng.normal(size=(E, F, d)).astype(np.float32) * 0.4
    W3 = rng.normal(size=(E, F, d)).astype(np.float32) * 0.4 if act else None
    W2 = rng.normal(size=(E, d, F)).astype(np.float32) * 0.4
    Ws = None
    if S:
        Ws = (rng.normal(size=(S, 3, d)).astype(np.float32),
              rng.normal(size=(S, 3, d)).astype(np.float32) if act else None,
              rng.normal(size=(S, d, 3)).astype(np.float32))
    sbias = rng.uniform(-0.1, 0.1, size=E).astype(np.float32) if score else None
    cf = 1.0
    C = oracle.capacity(T, E, k, cf)
    out = oracle.forward(x, W_r, W1, W3, W2, k=k, act=act, cf=cf, score=score,
                         priority=priority, select_bias=sbias,
                         Ws1=None if Ws is None else Ws[0], Ws3=None if Ws is None else Ws[1],
                         Ws2=None if Ws is None else Ws[2])
    tk, g, kp, y, aux, zl = py_forward(x, W_r, W1, W3, W2, k, act, C, score, sbias, priority, Ws)
    np.testing.assert_array_equal(out.route.topk, tk)
    np.testing.assert_allclose(out.route.gates, g, rtol=1e-12)
    np.testing.assert_array_equal(out.cap.keep, kp)
    np.testing.assert_allclose(out.y, y, rtol=1e-10, atol=1e-12)
    assert out.aux == pytest.approx(aux, rel=1e-12)
    assert out.zloss == pytest.approx(zl, rel=1e-12)


def test_tiny_config_through_the_oracle():
    inp = remove_near_ties(generate(CONFIGS["tiny"]))
    assert near_tie_rows(inp, oracle_route(inp)).size == 0
    out = oracle_forward(inp)
    s = inp.shape
    assert out.cap.C == 40
    assert out.y.shape == (s.T, s.d) and np.all(np.isfinite(out.y))
    assert out.cap.counts.sum() == s.T * s.k
    assert 0.9 < out.aux < 1.5 and out.zloss > 0
    tk, g, kp, y, aux, zl = py_forward(storage(inp.x), storage(inp.W_r), storage(inp.W1), None,
                                       storage(inp.W2), s.k, s.act, out.cap.C)
    np.testing.assert_array_equal(out.route.topk, tk)
    np.testing.assert_allclose(out.y, y, rtol=1e-10, atol=1e-12)


def test_generator_is_deterministic_and_seeded():
    a = generate(CONFIGS["tiny"])
    b = generate(CONFIGS["tiny"])
    assert torch.equal(a.x, b.x) and torch.equal(a.W1, b.W1)
    c = generate(CONFIGS["tiny"], seed=1)
    assert not torch.equal(a.x, c.x)
