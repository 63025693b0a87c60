"""Pins for the CPU oracle: each test ties it to something other than itself --
values the pages print, closed forms, invariants, and special cases that reduce
to a library routine (scipy, numpy's stable sort, torch float64 matmuls).

Sources by page title: "Lab 18 - Mixture of experts" (sections 1-3),
"Lab 01 - Router, Load Balancing, Capacity & the MoE Layer" (traps),
"Mixture of Experts - parameters without the FLOPs" (section 2).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special as sp
import torch
import torch.nn.functional as Fn

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def route_logits(z, k, score=0, renorm=-1, select_bias=None):
    """Route prescribed logits: d = E and W_r = I, so x = z exactly."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    E = z.shape[1]
    return oracle.route(z, np.eye(E, dtype=np.float32), k, score, renorm, None, select_bias)


# ----------------------------------------------------------------------- softmax

def test_softmax_survives_huge_logits():
    # "Lab 01", where to start step 1: logits of 1000 must not produce NaN
    r = route_logits([[1000.0, 0.0, 0.0, 0.0]], k=1)
    assert np.all(np.isfinite(r.scores))
    np.testing.assert_array_equal(r.scores[0], [1.0, 0.0, 0.0, 0.0])
    assert r.lse[0] == 1000.0
    r2 = route_logits([[1000.0, 1000.0]], k=1)
    np.testing.assert_array_equal(r2.scores[0], [0.5, 0.5])
    assert r2.lse[0] == pytest.approx(1000.0 + math.log(2.0), abs=1e-12)
    r3 = route_logits([[-1000.0, 1000.0, 0.0]], k=2, score=1)
    assert np.all(np.isfinite(r3.scores)) and np.all(np.isfinite(r3.gates))


def test_softmax_matches_library():
    rng = np.random.default_rng(1)
    z = rng.normal(size=(50, 7)).astype(np.float32) * 3
    r = route_logits(z, k=2)
    np.testing.assert_allclose(r.scores, sp.softmax(z.astype(np.float64), axis=1), rtol=1e-13)


# --------------------------------------------------------------------- top-k, gates

def test_topk_best_first_ties_to_lower_index():
    # "Lab 01" traps: break ties by expert index; numpy's stable argsort of the
    # negated keys is the library reference for that order
    z = np.array([[1.0, 3.0, 3.0, 0.0, 3.0],
                  [2.0, 2.0, 2.0, 2.0, 2.0],
                  [0.0, -1.0, 5.0, 5.0, -1.0]], np.float32)
    r = route_logits(z, k=3)
    ref = np.argsort(-z.astype(np.float64), axis=1, kind="stable")[:, :3]
    np.testing.assert_array_equal(r.topk, ref)
    np.testing.assert_array_equal(r.topk[0], [1, 2, 4])
    np.testing.assert_array_equal(r.topk[1], [0, 1, 2])


def test_topk_matches_stable_sort_random():
    rng = np.random.default_rng(2)
    z = rng.integers(-3, 4, size=(200, 9)).astype(np.float32)   # many exact ties
    r = route_logits(z, k=4)
    ref = np.argsort(-z.astype(np.float64), axis=1, kind="stable")[:, :4]
    np.testing.assert_array_equal(r.topk, ref)


@pytest.mark.parametrize("k", [2, 3, 5])
def test_renormalized_gates_equal_softmax_over_selected_logits(k):
    # "Lab 18" section 1: dividing the full softmax by the selected mass equals a
    # softmax over the selected logits
    rng = np.random.default_rng(3 + k)
    z = rng.normal(size=(64, 8)).astype(np.float32) * 2
    r = route_logits(z, k=k)
    sel = np.take_along_axis(z.astype(np.float64), r.topk.astype(np.int64), axis=1)
    np.testing.assert_allclose(r.gates, sp.softmax(sel, axis=1), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r.gates.sum(axis=1), 1.0, rtol=1e-13)


def test_raw_gate_for_top1_is_the_max_probability():
    # "Lab 18" section 1: Switch keeps the raw p_i when k = 1 (renormalizing would give 1)
    rng = np.random.default_rng(4)
    z = rng.normal(size=(64, 6)).astype(np.float32)
    r = route_logits(z, k=1)
    np.testing.assert_allclose(r.gates[:, 0], sp.softmax(z.astype(np.float64), axis=1).max(axis=1),
                               rtol=1e-13)
    assert np.all(r.gates[:, 0] < 1.0)
    forced = route_logits(z, k=1, renorm=1)
    np.testing.assert_array_equal(forced.gates, 1.0)


def test_sigmoid_gates_use_scores_without_selection_bias():
    # "Lab 18" section 2: the bias steers selection but not the gate values
    z = np.array([[2.0, 1.0, 0.0, -1.0]], np.float32)
    bias = np.array([0.0, 0.0, 5.0, 0.0], np.float32)     # lifts expert 2 into the top 2
    r = route_logits(z, k=2, score=1, select_bias=bias)
    np.testing.assert_array_equal(r.topk[0], [2, 0])
    s = sp.expit(z[0].astype(np.float64))
    np.testing.assert_allclose(r.gates[0], s[[2, 0]] / s[[2, 0]].sum(), rtol=1e-13)
    np.testing.assert_allclose(r.scores[0], s, rtol=1e-14)
    r0 = route_logits(z, k=2, score=1)
    np.testing.assert_array_equal(r0.topk[0], [0, 1])


def test_bf16_inputs_are_widened_exactly():
    rng = np.random.default_rng(5)
    xf = torch.tensor(rng.normal(size=(16, 24)), dtype=torch.float32).to(torch.bfloat16)
    W = rng.normal(size=(24, 5)).astype(np.float32) * 0.1
    bits = xf.view(torch.int16).numpy().view(np.uint16)
    r_bf = oracle.route(bits, W, 2)
    r_f = oracle.route(xf.to(torch.float32).numpy(), W, 2)
    np.testing.assert_array_equal(r_bf.z, r_f.z)
    np.testing.assert_allclose(r_bf.z, xf.double().numpy() @ W.astype(np.float64), rtol=1e-12,
                               atol=1e-13)


# ------------------------------------------------------------------------ losses

def test_aux_loss_worked_example_0_92():
    # "Lab 18" section 2: E=2, 90% of tokens at a 0.5/0.5 tie (-> expert 0 by the
    # index tie-break), 10% certain of expert 1: aux = 0.92.  Routing the tied
    # tokens to expert 1 instead would give 1.10.
    g = golden("aux_loss_tie_example.json")
    z = np.array([[0.0, 0.0]] * 90 + [[-1000.0, 1000.0]] * 10, np.float32)
    r = route_logits(z, k=g["k"])
    cap = oracle.capacity_walk(r.topk, g["E"], math.inf)
    aux, _ = oracle.losses(r.scores, cap.counts, r.lse, g["k"])
    assert aux == pytest.approx(g["aux"], abs=1e-12)
    np.testing.assert_array_equal(cap.counts, [90, 10])


def test_aux_loss_is_one_when_balanced_and_E_when_collapsed():
    # "Lab 18" section 2 / "Lab 01" step 3: uniform routing gives exactly 1, total
    # collapse gives E; f divides by the T k slots
    E, k, T = 8, 2, 64
    t = np.arange(T)
    a = t % E
    b = (a + 1 + (t // E) % (E - 1)) % E
    rng = np.random.default_rng(6)
    z = rng.normal(size=(T, E)) * 0.1 - 3.0
    z[t, a] = 2.0
    z[t, b] = 1.0
    r = route_logits(z.astype(np.float32), k=k)
    cap = oracle.capacity_walk(r.topk, E, math.inf)
    np.testing.assert_array_equal(cap.counts, np.full(E, T * k // E))
    aux, _ = oracle.losses(r.scores, cap.counts, r.lse, k)
    assert aux == pytest.approx(1.0, abs=1e-12)
    zc = np.full((T, E), -1000.0, np.float32)
    zc[:, 0] = 1000.0
    rc = route_logits(zc, k=1)
    capc = oracle.capacity_walk(rc.topk, E, math.inf)
    auxc, _ = oracle.losses(rc.scores, capc.counts, rc.lse, 1)
    assert auxc == pytest.approx(float(E), abs=1e-12)


def test_aux_loss_uses_full_softmax_not_gates():
    # "Lab 18" common bugs: P from renormalized gates ignores the unselected mass
    rng = np.random.default_rng(7)
    z = rng.normal(size=(32, 4)).astype(np.float32)
    r = route_logits(z, k=2)
    cap = oracle.capacity_walk(r.topk, 4, math.inf)
    aux, _ = oracle.losses(r.scores, cap.counts, r.lse, 2)
    p = sp.softmax(z.astype(np.float64), axis=1)
    f = np.bincount(r.topk.reshape(-1), minlength=4) / (32 * 2)
    assert aux == pytest.approx(4 * float((f * p.mean(axis=0)).sum()), rel=1e-13)


def test_sigmoid_aux_is_one_when_balanced():
    E, k, T = 4, 2, 16
    t = np.arange(T)
    a = t % E
    b = (a + 1 + (t // E) % (E - 1)) % E
    z = np.full((T, E), -2.0)
    z[t, a] = 2.0
    z[t, b] = 1.0
    r = route_logits(z.astype(np.float32), k=k, score=1)
    cap = oracle.capacity_walk(r.topk, E, math.inf)
    aux, _ = oracle.losses(r.scores, cap.counts, r.lse, k, score=1)
    assert aux == pytest.approx(1.0, abs=1e-12)


def test_router_z_loss_matches_definition():
    # "Lab 18" section 2: L_z = mean over tokens of logsumexp(z)^2
    rng = np.random.default_rng(8)
    z = rng.normal(size=(40, 6)).astype(np.float32) * 4
    r = route_logits(z, k=2)
    cap = oracle.capacity_walk(r.topk, 6, math.inf)
    _, zl = oracle.losses(r.scores, cap.counts, r.lse, 2)
    ref = float(np.mean(sp.logsumexp(z.astype(np.float64), axis=1) ** 2))
    assert zl == pytest.approx(ref, rel=1e-13)
    zeros = route_logits(np.zeros((5, 6), np.float32), k=2)
    _, zl0 = oracle.losses(zeros.scores, np.array([5, 5, 0, 0, 0, 0]), zeros.lse, 2)
    assert zl0 == pytest.approx(math.log(6.0) ** 2, rel=1e-14)


# ---------------------------------------------------------------------- capacity

def test_capacity_worked_example():
    g = golden("capacity_worked_example.json")
    assert oracle.capacity(g["T"], g["E"], g["k"], g["cf"]) == g["C"]
    assert g["T"] * g["k"] // g["E"] == g["balanced_load"]


def test_capacity_factor_below_one_raises():
    # "Lab 01" traps: capacity_factor < 1.0 must raise
    with pytest.raises(oracle.OracleError):
        oracle.capacity(4096, 8, 2, 0.99)
    with pytest.raises(oracle.OracleError):
        oracle.capacity_walk(np.zeros((4, 1), np.int32), 2, 0.5)
    with pytest.raises(oracle.OracleError):
        oracle.capacity(16, 4, 1, float("nan"))
    assert oracle.capacity(4096, 8, 1, 1.0) == 512
    assert oracle.capacity(100, 8, 2, math.inf) == 100


def test_capacity_ceil_formula_values():
    assert oracle.capacity(64, 4, 2, 1.25) == 40
    assert oracle.capacity(16384, 64, 6, 1.5) == 2304
    assert oracle.capacity(8192, 8, 2, 1.25) == 2560
    assert oracle.capacity(10, 3, 1, 1.0) == 4          # ceil(10/3)


def test_capacity_above_T_is_held_at_T_and_changes_no_decision():
    # a token's k experts are distinct ("Lab 18" section 1, top-k), so an
    # expert receives at most T assignments: any C >= T keeps everything
    assert oracle.capacity(64, 4, 2, 1e20) == 64
    assert oracle.capacity(10, 2, 2, 1.25) == 10        # ceil(12.5) = 13 > T
    rng = np.random.default_rng(5)
    topk = np.stack([rng.choice(2, size=2, replace=False) for _ in range(10)]).astype(np.int32)
    held = oracle.capacity_walk(topk, 2, 1.25)
    unclamped = oracle.capacity_walk(topk, 2, C=13)
    assert held.keep.all() and unclamped.keep.all() and held.n_dropped == 0
    big = oracle.capacity_walk(np.zeros((64, 1), np.int32), 4, 1e20)
    assert big.keep.all() and big.n_dropped == 0


def test_token_order_fcfs_keeps_the_earliest_tokens():
    # "Lab 01" step 4: first come first served in token order
    T, E, k = 16, 4, 1
    topk = np.zeros((T, k), np.int32)
    topk[5, 0] = 3
    cap = oracle.capacity_walk(topk, E, 1.0)                # C = 4
    assert cap.C == 4
    kept_tokens = np.nonzero(cap.keep[:, 0])[0]
    np.testing.assert_array_equal(kept_tokens, [0, 1, 2, 3, 5])
    np.testing.assert_array_equal(cap.counts, [15, 0, 0, 1])
    np.testing.assert_array_equal(cap.pos[:7, 0], [0, 1, 2, 3, 4, 0, 5])
    assert cap.n_dropped == 11
    np.testing.assert_array_equal(cap.dropped, 1 - cap.keep[:, 0])


def test_rank_major_token0_loses_its_second_choice():
    g = golden("rank_major_priority_example.json")
    topk = np.array(g["topk"], np.int32)
    rm = oracle.capacity_walk(topk, g["E"], C=g["C"], priority=1)
    np.testing.assert_array_equal(rm.keep, g["rank_major_keep"])
    to = oracle.capacity_walk(topk, g["E"], C=g["C"], priority=0)
    np.testing.assert_array_equal(to.keep, g["token_order_keep"])


@pytest.mark.parametrize("priority", [0, 1])
def test_capacity_positions_equal_one_hot_cumsum(priority):
    # "Lab 18" tips: flatten in priority order, one-hot, cumulative sum; the
    # entry of the assignment's own expert minus one is its queue position
    rng = np.random.default_rng(9 + priority)
    T, E, k = 300, 7, 3
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    cap = oracle.capacity_walk(topk, E, 1.1, priority)
    flat = topk.reshape(-1) if priority == 0 else topk.T.reshape(-1)
    onehot = np.eye(E, dtype=np.int64)[flat]
    pos_flat = np.take_along_axis(np.cumsum(onehot, axis=0), flat[:, None], axis=1)[:, 0] - 1
    pos = pos_flat.reshape(T, k) if priority == 0 else pos_flat.reshape(k, T).T
    np.testing.assert_array_equal(cap.pos, pos)
    np.testing.assert_array_equal(cap.keep, (pos < cap.C).astype(np.uint8))
    np.testing.assert_array_equal(cap.counts, np.bincount(flat, minlength=E))


# --------------------------------------------------------------------- forward

def _torch_ffn(x, W1, W3, W2, act):
    h = x @ W1.T
    if act == 0:
        h = Fn.gelu(h, approximate="none")
    else:
        h = Fn.silu(h) * (x @ W3.T)
    return h @ W2.T


def _rand_layer(rng, T, d, E, F, act, S=0, Fs=0):
    x = rng.normal(size=(T, d)).astype(np.float32)
    W_r = (rng.normal(size=(d, E)) * 0.3).astype(np.float32)
    W1 = (rng.normal(size=(E, F, d)) / math.sqrt(d)).astype(np.float32)
    W3 = (rng.normal(size=(E, F, d)) / math.sqrt(d)).astype(np.float32) if act else None
    W2 = (rng.normal(size=(E, d, F)) / math.sqrt(F)).astype(np.float32)
    sh = (None, None, None)
    if S:
        sh = ((rng.normal(size=(S, Fs, d)) / math.sqrt(d)).astype(np.float32),
              (rng.normal(size=(S, Fs, d)) / math.sqrt(d)).astype(np.float32) if act else None,
              (rng.normal(size=(S, d, Fs)) / math.sqrt(Fs)).astype(np.float32))
    return x, W_r, W1, W3, W2, sh


@pytest.mark.parametrize("act,S", [(0, 0), (1, 0), (1, 2), (0, 1)])
def test_k_equals_E_is_a_dense_soft_mixture(act, S):
    # k == E renormalizes by a mass of 1, so y = sum_i p_i FFN_i(x) + shared:
    # a dense mixture computed here with torch float64 matmuls, torch's exact
    # GELU and SiLU.  Catches transposed operands (d != F), swapped W1/W3 and a
    # wrong activation.
    rng = np.random.default_rng(10 + act + S)
    T, d, E, F, Fs = 12, 6, 3, 10, 5
    x, W_r, W1, W3, W2, (Ws1, Ws3, Ws2) = _rand_layer(rng, T, d, E, F, act, S, Fs)
    out = oracle.forward(x, W_r, W1, W3, W2, k=E, act=act, cf=math.inf, Ws1=Ws1, Ws3=Ws3,
                         Ws2=Ws2)
    X = torch.tensor(x, dtype=torch.float64)
    p = torch.softmax(X @ torch.tensor(W_r, dtype=torch.float64), dim=1)
    ref = torch.zeros(T, d, dtype=torch.float64)
    for e in range(E):
        w3 = None if W3 is None else torch.tensor(W3[e], dtype=torch.float64)
        ref += p[:, e:e + 1] * _torch_ffn(X, torch.tensor(W1[e], dtype=torch.float64), w3,
                                          torch.tensor(W2[e], dtype=torch.float64), act)
    for s in range(S):
        w3 = None if Ws3 is None else torch.tensor(Ws3[s], dtype=torch.float64)
        ref += _torch_ffn(X, torch.tensor(Ws1[s], dtype=torch.float64), w3,
                          torch.tensor(Ws2[s], dtype=torch.float64), act)
    np.testing.assert_allclose(out.y, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_single_expert_is_a_plain_mlp():
    rng = np.random.default_rng(20)
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, 9, 8, 1, 16, 1)
    out = oracle.forward(x, W_r, W1, W3, W2, k=1, act=1, cf=1.0)
    np.testing.assert_array_equal(out.route.gates, 1.0)          # softmax of one logit
    X = torch.tensor(x, dtype=torch.float64)
    ref = _torch_ffn(X, torch.tensor(W1[0], dtype=torch.float64),
                     torch.tensor(W3[0], dtype=torch.float64),
                     torch.tensor(W2[0], dtype=torch.float64), 1)
    np.testing.assert_allclose(out.y, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_dropped_tokens_get_nothing_and_kept_tokens_their_gated_expert():
    # "Lab 18" section 3: a dropped slot contributes nothing; a token with every
    # slot dropped reaches the next layer only through the residual (y = 0 here)
    rng = np.random.default_rng(21)
    T, d, E, F = 16, 8, 4, 12
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, T, d, E, F, 0)
    bias = np.array([8.0, 0.0, 0.0, 0.0], np.float32)       # everyone picks expert 0
    out = oracle.forward(x, W_r, W1, W3, W2, k=1, act=0, cf=1.0, logit_bias=bias)
    assert np.all(out.route.topk[:, 0] == 0)
    C = out.cap.C
    assert C == 4
    X = torch.tensor(x, dtype=torch.float64)
    z = X @ torch.tensor(W_r, dtype=torch.float64) + torch.tensor(bias, dtype=torch.float64)
    p0 = torch.softmax(z, dim=1)[:, 0:1]
    ref = p0 * _torch_ffn(X, torch.tensor(W1[0], dtype=torch.float64), None,
                          torch.tensor(W2[0], dtype=torch.float64), 0)
    np.testing.assert_allclose(out.y[:C], ref.numpy()[:C], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(out.y[C:], 0.0)
    np.testing.assert_array_equal(out.cap.dropped, [0] * C + [1] * (T - C))


def test_one_slot_per_expert_at_most_E_tokens_get_output():
    # "Lab 18" what-to-implement row 5: with one slot per expert at most four
    # tokens (E = 4) get output
    rng = np.random.default_rng(22)
    T, d, E, F = 32, 8, 4, 8
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, T, d, E, F, 0)
    for priority in (0, 1):
        out = oracle.forward(x, W_r, W1, W3, W2, k=2, act=0, cf=1.0, priority=priority,
                             capacity_override=1)
        nonzero = np.count_nonzero(np.abs(out.y).sum(axis=1))
        assert nonzero <= E
        assert out.cap.keep.sum() == E


def test_shared_expert_removes_the_fully_dropped_failure():
    # "Phase 02" takeaways: a shared expert gives every token some FFN
    rng = np.random.default_rng(23)
    T, d, E, F, Fs = 16, 8, 4, 8, 6
    x, W_r, W1, W3, W2, (Ws1, Ws3, Ws2) = _rand_layer(rng, T, d, E, F, 1, 1, Fs)
    bias = np.array([9.0, 0.0, 0.0, 0.0], np.float32)
    out = oracle.forward(x, W_r, W1, W3, W2, k=1, act=1, cf=1.0, logit_bias=bias, Ws1=Ws1,
                         Ws3=Ws3, Ws2=Ws2)
    dropped = np.nonzero(out.cap.dropped)[0]
    assert dropped.size > 0
    X = torch.tensor(x, dtype=torch.float64)
    shared = _torch_ffn(X, torch.tensor(Ws1[0], dtype=torch.float64),
                        torch.tensor(Ws3[0], dtype=torch.float64),
                        torch.tensor(Ws2[0], dtype=torch.float64), 1).numpy()
    np.testing.assert_allclose(out.y[dropped], shared[dropped], rtol=1e-11, atol=1e-12)


def test_token_subset_matches_full_forward():
    rng = np.random.default_rng(24)
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, 20, 8, 4, 8, 1)
    full = oracle.forward(x, W_r, W1, W3, W2, k=2, act=1, cf=1.0)
    sub = oracle.forward(x, W_r, W1, W3, W2, k=2, act=1, cf=1.0, tokens=[19, 3, 7])
    np.testing.assert_array_equal(sub.y, full.y[[19, 3, 7]])


# ----------------------------------------------------------- parameter counting

def test_param_counts_match_the_table():
    for row in golden("param_counts.json")["rows"]:
        total, active = oracle.moe_param_counts(row["d"], row["d_ff"], row["E"], row["k"],
                                                row["n_shared"])
        assert round(total / 1e6, 1) == row["total_M"]
        assert round(active / 1e6, 1) == row["active_M"]


def test_sparsity_ratio_is_one_when_k_equals_E():
    # "Lab 01" traps: top_k == n_experts must give sparsity exactly 1.0
    assert oracle.sparsity_ratio(1024, 512, 8, 8) == 1.0
    assert oracle.sparsity_ratio(1024, 512, 8, 2) == 0.25
