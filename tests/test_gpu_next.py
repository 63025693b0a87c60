"""GPU parity of the rows beyond the forward pass: batch-prioritized capacity,
the sequence-wise balance loss and the auxiliary-loss-free bias step, through
the C ABI, against the oracle on the same seeded inputs.

Bar: capacity results and the bias step bit-exact; the sequence-wise loss
within 1e-5 relative (as the batch losses); the forward with the score order
at the bf16 bar of test_gpu_parity.py.
"""
import math

import numpy as np
import pytest
import torch

from moe_inputs import CONFIGS, PRIORITY_SCORE, generate, shrink
from support import oracle_forward, oracle_route, remove_near_ties
import oracle

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_54_b200 as moe

LOSS_RTOL = 1e-5


def _assignments(T, E, k, seed, levels, skew=False):
    """Seeded top-k indices (k distinct experts per token) and router scores
    [T, E] on `levels` values in [0, 1), so that equal scores are common; a
    few scores are -0.0 (equal to +0.0)."""
    g = torch.Generator().manual_seed(seed)
    topk = torch.rand((T, E), generator=g).argsort(dim=1)[:, :k].to(torch.int32)
    if skew and k < E:
        # every token's first choice is expert 0: one list of T entries
        rest = torch.rand((T, E - 1), generator=g).argsort(dim=1)[:, : k - 1] + 1
        topk = torch.cat([torch.zeros((T, 1), dtype=torch.int64), rest], 1).to(torch.int32)
    scores = torch.randint(0, levels, (T, E), generator=g).to(torch.float32) / levels
    neg = torch.rand((T, E), generator=g) < 0.01
    scores[neg & (scores == 0)] = -0.0
    return topk, scores


def _offsets(kept):
    off = [0]
    for c in kept:
        off.append(off[-1] + (int(c) + 127) // 128 * 128)
    return off


CAP_CASES = [
    # T, E, k, cf, levels, skew
    (1000, 8, 2, 1.0, 16, False),
    (4096, 8, 1, 1.0, 1000, False),
    (333, 64, 6, 1.5, 8, False),
    (4096, 256, 8, 1.0, 50, False),
    (257, 1, 1, 1.0, 4, False),
    (2048, 4, 4, 1.0, 3, False),
    (16384, 64, 6, 1.5, 100000, False),
    (16384, 8, 2, 1.25, 7, True),
    (300, 8, 2, math.inf, 5, False),
]


@pytest.mark.parametrize("case", CAP_CASES, ids=lambda c: "T{}_E{}_k{}_cf{}_{}".format(*c[:4], "skew" if c[5] else "u"))
def test_capacity_scored_is_bit_exact(case):
    T, E, k, cf, levels, skew = case
    topk, scores = _assignments(T, E, k, seed=T + E + k, levels=levels, skew=skew)
    cfg = moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=cf, priority=PRIORITY_SCORE)
    out = moe.moe_capacity_scored(cfg, topk.cuda(), scores.cuda())
    torch.cuda.synchronize()
    ref = oracle.capacity_walk(topk.numpy(), E, cf, priority=2,
                               sel_scores=oracle.selected_scores(scores.numpy(), topk.numpy()))
    np.testing.assert_array_equal(out.counts.cpu().numpy(), ref.counts)
    np.testing.assert_array_equal(out.pos.cpu().numpy(), ref.pos)
    np.testing.assert_array_equal(out.keep.cpu().numpy(), ref.keep)
    np.testing.assert_array_equal(out.dropped.cpu().numpy(), ref.dropped)
    assert int(out.n_dropped.item()) == ref.n_dropped
    kept = np.minimum(ref.counts, ref.C)
    np.testing.assert_array_equal(out.kept.cpu().numpy(), kept)
    np.testing.assert_array_equal(out.offsets.cpu().numpy(), _offsets(kept))


def test_capacity_scored_with_equal_scores_matches_token_order():
    T, E, k = 1500, 16, 4
    topk, _ = _assignments(T, E, k, seed=5, levels=2)
    flat = torch.full((T, E), 0.5)
    scored = moe.moe_capacity_scored(
        moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=1.0, priority=2),
        topk.cuda(), flat.cuda())
    token = moe.moe_capacity(moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=1.0),
                             topk.cuda())
    torch.cuda.synchronize()
    assert torch.equal(scored.pos, token.pos) and torch.equal(scored.keep, token.keep)
    assert torch.equal(scored.dropped, token.dropped)


SCORED_FWD = {
    "switch_small": shrink(CONFIGS["switch"], T=1000, d=256, d_ff=512, priority=PRIORITY_SCORE),
    "mixtral_small": shrink(CONFIGS["mixtral"], T=700, d=512, d_ff=384, cf=1.0, zipf_s=1.1,
                            priority=PRIORITY_SCORE),
    "deepseek_v3_small": shrink(CONFIGS["deepseek_v3"], T=333, d=192, d_ff=128, d_ff_shared=192,
                                cf=1.0, priority=PRIORITY_SCORE),
}


def _uncertain_experts(ref, E, rel=1e-5):
    """Experts whose capacity boundary falls between two scores closer than
    rel: there either side of the pair is a correct keep set in fp32."""
    sel = oracle.selected_scores(ref.route.scores, ref.route.topk).astype(np.float64)
    out = set()
    for e in range(E):
        s = np.sort(sel[ref.route.topk == e])[::-1]
        C = ref.cap.C
        if len(s) > C > 0 and s[C - 1] - s[C] <= rel * max(abs(s[C - 1]), 1e-30):
            out.add(e)
    return out


@pytest.mark.parametrize("name", list(SCORED_FWD))
def test_forward_with_score_priority_matches_the_oracle(name):
    shape = SCORED_FWD[name]
    inp = remove_near_ties(generate(shape, device="cuda"))
    ref = oracle_forward(inp)
    fwd = moe.MoEForward(moe.moe_config(shape), "cuda")
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    fwd(inp.x, w)
    torch.cuda.synchronize()
    assert moe.moe_device_status(fwd.ws) == 0
    topk = fwd.topk.cpu().numpy()
    np.testing.assert_array_equal(topk, ref.route.topk)
    np.testing.assert_array_equal(fwd.counts.cpu().numpy(), ref.cap.counts)
    assert int(fwd.n_dropped.item()) == ref.cap.n_dropped
    assert ref.cap.n_dropped > 0   # the order matters only when something is dropped
    unsure = _uncertain_experts(ref, shape.E)
    sure = ~np.isin(topk, list(unsure)) if unsure else np.ones_like(topk, dtype=bool)
    keep = fwd.keep.cpu().numpy()
    np.testing.assert_array_equal(keep[sure], ref.cap.keep[sure])
    sel = oracle.selected_scores(ref.route.scores, ref.route.topk).astype(np.float64)
    for e in unsure:   # valid: the kept ones of e are its highest-scored, C of them
        m = topk == e
        assert keep[m].sum() == min(m.sum(), ref.cap.C)
        kept_s, dropped_s = sel[m & (keep == 1)], sel[m & (keep == 0)]
        if kept_s.size and dropped_s.size:
            # every kept score is at least every dropped score of the expert,
            # up to the fp32 near-tie window
            lo, hi = kept_s.min(), dropped_s.max()
            assert lo >= hi - 1e-5 * max(abs(hi), 1e-30), (e, lo, hi)
    tokens = np.nonzero(sure.all(axis=1))[0]
    assert tokens.size >= 0.9 * shape.T
    got = fwd.y[torch.as_tensor(tokens, device="cuda")].double().cpu().numpy()
    want = ref.y[tokens]
    scale = np.abs(want).max()
    frob = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300)
    assert frob <= 1e-2 and np.abs(got - want).max() <= 2e-2 * scale
    assert float(fwd.aux.item()) == pytest.approx(ref.aux, rel=LOSS_RTOL)


SEQ_CASES = {
    "switch": (shrink(CONFIGS["switch"], T=1024, d=256, d_ff=512), [32, 256, 1024]),
    "deepseekmoe": (shrink(CONFIGS["deepseekmoe"], T=1024, d=128, d_ff=128, d_ff_shared=128),
                    [64, 512]),
    "deepseek_v3": (shrink(CONFIGS["deepseek_v3"], T=512, d=192, d_ff=128, d_ff_shared=192),
                    [32, 128, 512]),
    "mixtral_full": (CONFIGS["mixtral"], [4096]),
}


@pytest.mark.parametrize("name", list(SEQ_CASES))
def test_seq_balance_loss_matches_the_oracle(name):
    shape, lengths = SEQ_CASES[name]
    inp = remove_near_ties(generate(shape, device="cuda"))
    cfg = moe.moe_config(shape)
    topk, _, partials, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    r = oracle_route(inp)
    np.testing.assert_array_equal(topk.cpu().numpy(), r.topk)
    for L in lengths:
        loss, per = moe.moe_seq_balance_loss(cfg, L, topk, partials)
        torch.cuda.synchronize()
        mean, per_ref = oracle.seq_losses(r.scores, r.topk, shape.k, L, shape.score)
        np.testing.assert_allclose(per.double().cpu().numpy(), per_ref, rtol=LOSS_RTOL)
        assert float(loss.item()) == pytest.approx(mean, rel=LOSS_RTOL)
    if name != "mixtral_full":
        # one sequence spanning the batch is the batch Switch loss
        counts = np.bincount(r.topk.ravel(), minlength=shape.E).astype(np.int32)
        aux, _ = oracle.losses(r.scores, counts, r.lse, shape.k, shape.score)
        loss, _ = moe.moe_seq_balance_loss(cfg, shape.T, topk, partials)
        assert float(loss.item()) == pytest.approx(aux, rel=LOSS_RTOL)


@pytest.mark.parametrize("E,T,k", [(8, 4096, 2), (256, 4096, 8), (3, 7, 1), (64, 16384, 6)])
def test_bias_update_is_bit_exact(E, T, k):
    g = torch.Generator().manual_seed(E * 7 + k)
    counts = torch.randint(0, 2 * T * k // E + 2, (E,), generator=g).to(torch.int32)
    if T * k % E == 0:
        counts[0] = T * k // E   # exactly balanced: unchanged
    bias = (torch.randn(E, generator=g) * 0.1).to(torch.float32)
    cfg = moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=1.0)
    dev_bias = bias.cuda()
    moe.moe_bias_update(cfg, counts.cuda(), 1e-3, dev_bias)
    torch.cuda.synchronize()
    want = oracle.bias_update(counts.numpy(), T, k, 1e-3, bias.numpy())
    assert dev_bias.cpu().numpy().tobytes() == want.tobytes()


def test_bias_steps_balance_the_gpu_router():
    """DeepSeek-V3-shaped router with skewed logits: route, count, step the
    selection bias, repeatedly, all on the GPU; the load spread shrinks."""
    shape = shrink(CONFIGS["deepseek_v3"], T=2048, d=256, d_ff=128, d_ff_shared=128, E=32,
                   k=4, zipf_s=1.1)
    inp = generate(shape, device="cuda")
    cfg = moe.moe_config(shape)
    bias = torch.zeros(shape.E, dtype=torch.float32, device="cuda")
    spread = []
    for _ in range(200):
        topk, _, _, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, bias)
        cap = moe.moe_capacity(cfg, topk)
        c = cap.counts.cpu()
        spread.append(int(c.max() - c.min()))
        moe.moe_bias_update(cfg, cap.counts, 0.01, bias)
    assert spread[-1] < spread[0] / 3, spread[::20]


@pytest.mark.parametrize("shards,cf", [(3, 1.0), (2, 1.25), (4, math.inf)])
def test_sharded_capacity_equals_the_whole_batch(shards, cf):
    """A token-ordered batch split into shards (run one after another on this
    GPU, the all-gather of counts done by stacking): each shard's keep, drop
    and positions equal the whole batch's bit for bit, and the losses from the
    shards' counts and loss rows match the whole batch's within 1e-5 (the
    router splits K differently for a shard, so its loss rows may differ in
    the last bits)."""
    Tl, E, k, d = 1024, 16, 4, 256
    shape = shrink(CONFIGS["deepseekmoe"], T=Tl * shards, d=d, E=E, k=k, d_ff=128,
                   d_ff_shared=128, cf=cf, zipf_s=1.1)
    inp = remove_near_ties(generate(shape, device="cuda"))
    cfg_all = moe.moe_config(shape)
    topk, _, part, _, _ = moe.moe_route(cfg_all, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    whole = moe.moe_capacity(cfg_all, topk)
    C = moe.moe_capacity_value(cfg_all)
    cfg_one = moe.moe_config(shape, T=Tl)
    local = [moe.moe_capacity(cfg_one, topk[i * Tl:(i + 1) * Tl].contiguous())
             for i in range(shards)]
    shard_counts = torch.stack([c.counts for c in local])
    base = torch.zeros(E, dtype=torch.int64, device="cuda")
    kept_sum = torch.zeros(E, dtype=torch.int64, device="cuda")
    nd = 0
    for i in range(shards):
        rows = slice(i * Tl, (i + 1) * Tl)
        out = moe.moe_capacity_sharded(cfg_one, C, shard_counts, i, topk[rows].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(out.keep, whole.keep[rows])
        assert torch.equal(out.dropped, whole.dropped[rows])
        e = topk[rows].long()
        assert torch.equal(out.pos.long() + base[e], whole.pos[rows].long())
        assert torch.equal(out.counts, local[i].counts)
        kept_sum += out.kept.long()
        nd += int(out.n_dropped.item())
        base += out.counts.long()
    assert torch.equal(kept_sum, whole.kept.long())
    assert nd == int(whole.n_dropped.item())
    if cf == 1.0:
        assert nd > 0
    # losses: counts summed, loss rows concatenated in shard order
    part_l = [moe.moe_route(cfg_one, inp.x[i * Tl:(i + 1) * Tl].contiguous(), inp.W_r,
                            inp.logit_bias, inp.select_bias)[2] for i in range(shards)]
    aux_s, z_s = moe.moe_losses(cfg_all, shard_counts.sum(0).to(torch.int32), torch.cat(part_l))
    aux_w, z_w = moe.moe_losses(cfg_all, whole.counts, part)
    torch.cuda.synchronize()
    assert aux_s.item() == pytest.approx(aux_w.item(), rel=LOSS_RTOL)
    assert z_s.item() == pytest.approx(z_w.item(), rel=LOSS_RTOL)
