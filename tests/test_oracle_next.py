"""Pins of the oracle's batch-prioritized capacity, sequence-wise balance loss
and auxiliary-loss-free bias update against closed forms, properties the
pages state, and brute force by another method on small inputs."""
import numpy as np
import pytest

import oracle


# ------------------------------------------------------- batch-prioritized capacity

def test_scored_capacity_hand_example():
    # One expert, two slots, four tokens scored 0.1, 0.9, 0.5, 0.7: the two
    # highest scores (tokens 1 and 3) are kept; the queue runs 1, 3, 2, 0.
    topk = np.zeros((4, 1), np.int32)
    cap = oracle.capacity_walk(topk, 1, C=2, priority=2,
                               sel_scores=np.array([[0.1], [0.9], [0.5], [0.7]]))
    assert cap.pos.ravel().tolist() == [3, 0, 2, 1]
    assert cap.keep.ravel().tolist() == [0, 1, 0, 1]
    assert cap.dropped.tolist() == [1, 0, 1, 0]
    assert cap.n_dropped == 2 and cap.counts.tolist() == [4]


def test_scored_capacity_with_equal_scores_is_token_order():
    rng = np.random.default_rng(3)
    T, E, k = 97, 6, 3
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    flat = oracle.capacity_walk(topk, E, C=40, priority=2,
                                sel_scores=np.full((T, k), 0.25, np.float32))
    tok = oracle.capacity_walk(topk, E, C=40, priority=0)
    assert np.array_equal(flat.pos, tok.pos) and np.array_equal(flat.keep, tok.keep)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_scored_capacity_equals_rank_by_counting(seed):
    # pos of an assignment = number of assignments to the same expert that
    # outrank it (higher score, or equal score and earlier in token/slot
    # order): counted pairwise here, sorted-and-walked in the oracle.
    rng = np.random.default_rng(seed)
    T, E, k, C = 41, 5, 2, 7
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    sel = (rng.integers(0, 6, size=(T, k)) / 8).astype(np.float32)   # many equal scores
    cap = oracle.capacity_walk(topk, E, C=C, priority=2, sel_scores=sel)
    f_e, f_s = topk.ravel(), sel.ravel()
    A = T * k
    for a in range(A):
        ahead = sum(1 for b in range(A)
                    if f_e[b] == f_e[a] and (f_s[b] > f_s[a] or (f_s[b] == f_s[a] and b < a)))
        assert cap.pos.ravel()[a] == ahead
        assert cap.keep.ravel()[a] == (ahead < C)
    assert cap.counts.tolist() == np.bincount(f_e, minlength=E).tolist()
    assert cap.dropped.tolist() == [int(not cap.keep[t].any()) for t in range(T)]


def test_scored_capacity_keeps_the_highest_scores_of_each_expert():
    rng = np.random.default_rng(5)
    T, E, k = 300, 4, 2
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    sel = rng.random((T, k)).astype(np.float32)
    cap = oracle.capacity_walk(topk, E, 1.0, priority=2, sel_scores=sel)
    for e in range(E):
        m = topk == e
        kept, lost = sel[m & (cap.keep == 1)], sel[m & (cap.keep == 0)]
        if len(kept) and len(lost):
            assert kept.min() >= lost.max()


def test_forward_batch_prioritized_uses_router_scores():
    # Through the forward: the kept assignments of each expert are its
    # highest-probability ones, and selected_scores is the full softmax value.
    rng = np.random.default_rng(8)
    T, d, E, k, F = 64, 16, 4, 2, 8
    x = rng.standard_normal((T, d)).astype(np.float32)
    W_r = rng.standard_normal((d, E)).astype(np.float32)
    W1 = rng.standard_normal((E, F, d)).astype(np.float32)
    W2 = rng.standard_normal((E, d, F)).astype(np.float32)
    out = oracle.forward(x, W_r, W1, None, W2, k=k, act=0, cf=1.0, priority=2)
    sel = oracle.selected_scores(out.route.scores, out.route.topk)
    assert np.array_equal(sel, np.take_along_axis(out.route.scores, out.route.topk.astype(int),
                                                  1).astype(np.float32))
    direct = oracle.capacity_walk(out.route.topk, E, 1.0, priority=2, sel_scores=sel)
    assert np.array_equal(direct.keep, out.cap.keep)


# -------------------------------------------------------- sequence-wise balance loss

def _seq_loss_loop(scores, topk, k, L, score):
    T, E = scores.shape
    vals = []
    for b in range(T // L):
        rows = range(b * L, (b + 1) * L)
        cnt = [0] * E
        for t in rows:
            for j in range(k):
                cnt[topk[t, j]] += 1
        P = [0.0] * E
        for t in rows:
            norm = sum(scores[t]) if score == 1 else 1.0
            for i in range(E):
                P[i] += scores[t, i] / norm
        vals.append(E * sum(cnt[i] / (L * k) * P[i] / L for i in range(E)))
    return sum(vals) / len(vals), vals


@pytest.mark.parametrize("score", [0, 1])
def test_seq_loss_agrees_with_python_loop(score):
    rng = np.random.default_rng(11 + score)
    T, E, k, L = 48, 5, 2, 12
    z = rng.standard_normal((T, E))
    scores = np.exp(z) / np.exp(z).sum(1, keepdims=True) if score == 0 else 1 / (1 + np.exp(-z))
    topk = np.argsort(-scores, axis=1, kind="stable")[:, :k].astype(np.int32)
    mean, per = oracle.seq_losses(scores, topk, k, L, score)
    ref_mean, ref = _seq_loss_loop(scores, topk, k, L, score)
    assert abs(mean - ref_mean) < 1e-12
    assert np.allclose(per, ref, rtol=0, atol=1e-12)


def test_seq_loss_of_one_sequence_is_the_batch_loss():
    rng = np.random.default_rng(2)
    T, E, k = 40, 6, 2
    z = rng.standard_normal((T, E))
    p = np.exp(z) / np.exp(z).sum(1, keepdims=True)
    topk = np.argsort(-p, axis=1, kind="stable")[:, :k].astype(np.int32)
    counts = np.bincount(topk.ravel(), minlength=E).astype(np.int32)
    aux, _ = oracle.losses(p, counts, np.zeros(T), k)
    mean, _ = oracle.seq_losses(p, topk, k, T)
    assert abs(mean - aux) < 1e-12


def test_seq_loss_sees_per_sequence_collapse_the_batch_loss_misses():
    # Two sequences, each sent wholly (p = 1) to its own expert: the batch is
    # balanced (Switch loss 1), each sequence collapsed (loss E = 2).
    L, E = 8, 2
    p = np.zeros((2 * L, E))
    p[:L, 0] = 1.0
    p[L:, 1] = 1.0
    topk = np.argmax(p, 1).astype(np.int32)[:, None]
    mean, per = oracle.seq_losses(p, topk, 1, L)
    assert per.tolist() == [2.0, 2.0] and mean == 2.0
    aux, _ = oracle.losses(p, np.bincount(topk.ravel(), minlength=E).astype(np.int32),
                           np.zeros(2 * L), 1)
    assert aux == 1.0


def test_seq_loss_rejects_a_partial_sequence():
    with pytest.raises(oracle.OracleError):
        oracle.seq_losses(np.full((10, 2), 0.5), np.zeros((10, 1), np.int32), 1, 4)


# ----------------------------------------------------------- bias update (V3 balancing)

def test_bias_update_closed_form():
    g = np.float32(1e-3)
    b = np.array([0.5, -0.25, 0.0, 1e-3], np.float32)
    # T k = 8 slots over E = 4 experts: balanced load 2
    out = oracle.bias_update([3, 1, 2, 2], 4, 2, 1e-3, b)
    want = np.array([b[0] - g, b[1] + g, b[2], b[3]], np.float32)
    assert out.tobytes() == want.tobytes()


def test_bias_update_compares_with_a_fractional_balanced_load():
    # T k / E = 1.5: two tokens on expert 0 is over, one on expert 1 is under
    out = oracle.bias_update([2, 1], 3, 1, 0.5, [0.0, 0.0])
    assert out.tolist() == [-0.5, 0.5]


def test_bias_update_balances_selection_without_touching_gates():
    # A router skewed by fixed logit offsets, sigmoid scores with a selection
    # bias: repeated steps bring the loads together, while the gates stay the
    # renormalized sigmoid scores of the selected experts (no bias in them).
    rng = np.random.default_rng(4)
    T, d, E, k = 512, 16, 8, 2
    x = rng.standard_normal((T, d)).astype(np.float32)
    W_r = (rng.standard_normal((d, E)) * 0.3).astype(np.float32)
    lb = np.linspace(1.0, -1.0, E).astype(np.float32)
    bias = np.zeros(E, np.float32)
    spread = []
    for step in range(150):
        r = oracle.route(x, W_r, k, score=1, logit_bias=lb, select_bias=bias)
        counts = np.bincount(r.topk.ravel(), minlength=E)
        spread.append(counts.max() - counts.min())
        bias = oracle.bias_update(counts.astype(np.int32), T, k, 0.01, bias)
    assert spread[-1] < spread[0] / 4
    s_sel = np.take_along_axis(r.scores, r.topk.astype(int), 1)
    assert np.allclose(r.gates, s_sel / s_sel.sum(1, keepdims=True), rtol=0, atol=1e-15)
