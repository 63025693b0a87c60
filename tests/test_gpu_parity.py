"""End-to-end parity of the CUDA path (through the C ABI) with the CPU oracle
on the same seeded inputs.

Bar (from the layer's specification):
  - routing indices, per-expert counts, queue positions, keep/drop masks and
    the dropped-token set: bit-exact;
  - fp32 layers: max |y - y_ref| <= 1e-4 max|y_ref|;
  - bf16 layers: relative Frobenius error <= 1e-2 and max abs error
    <= 2e-2 max|y_ref|;
  - aux loss and z-loss: within 1e-5 relative.
Inputs are redrawn wherever two neighbouring selection keys among the top k+1
are closer than 1e-4 (see support.remove_near_ties).
"""
import math

import numpy as np
import pytest
import torch

from moe_inputs import CONFIGS, generate, mixtral_variant, shrink, balanced_assignment
from support import oracle_forward, oracle_route, remove_near_ties, storage, near_tie_rows
import oracle

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_54_b200 as moe

LOSS_RTOL = 1e-5


def run_stages(inp):
    """All six stages through the per-stage ABI calls."""
    s = inp.shape
    cfg = moe.moe_config(s)
    topk, gates, part, logits, scores = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias,
                                                      inp.select_bias, want_logits=True,
                                                      want_scores=True)
    cap = moe.moe_capacity(cfg, topk)
    x_perm = moe.moe_dispatch(cfg, inp.x, topk, cap.pos, cap.keep, cap.offsets)
    Y, Ysh, ws = moe.moe_expert_ffn(cfg, x_perm, cap.offsets, inp.W1, inp.W3, inp.W2, inp.x,
                                    inp.Ws1, inp.Ws3, inp.Ws2)
    y = moe.moe_combine(cfg, Y, Ysh, gates, topk, cap.pos, cap.keep, cap.offsets)
    aux, zl = moe.moe_losses(cfg, cap.counts, part)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    return dict(topk=topk, gates=gates, logits=logits, scores=scores, cap=cap, y=y, aux=aux,
                zloss=zl)


def run_forward(inp):
    """The launch configuration the benchmark times: one moe_forward call."""
    s = inp.shape
    cfg = moe.moe_config(s)
    fwd = moe.MoEForward(cfg, inp.x.device)
    w = moe.weights_struct(inp.W_r, inp.W1, inp.W2, inp.W3, inp.logit_bias, inp.select_bias,
                           inp.Ws1, inp.Ws3, inp.Ws2)
    fwd(inp.x, w)
    torch.cuda.synchronize()
    assert moe.moe_device_status(fwd.ws) == 0
    return fwd


def check_y(shape, got, ref):
    got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    if shape.dtype == 0:
        assert err.max() <= 1e-4 * scale, f"max abs err {err.max():.3e} vs max|y| {scale:.3e}"
    else:
        frob = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
        assert frob <= 1e-2, f"relative Frobenius error {frob:.3e}"
        assert err.max() <= 2e-2 * scale, f"max abs err {err.max():.3e} vs max|y| {scale:.3e}"


def check_losses(aux, zl, ref):
    assert float(aux.item()) == pytest.approx(ref.aux, rel=LOSS_RTOL)
    assert float(zl.item()) == pytest.approx(ref.zloss, rel=LOSS_RTOL)


def check_routing(topk, gates, ref, rtol=1e-5):
    np.testing.assert_array_equal(topk.cpu().numpy(), ref.route.topk)
    np.testing.assert_allclose(gates.double().cpu().numpy(), ref.route.gates, rtol=rtol, atol=1e-6)


def check_capacity(counts, keep, dropped, ref, pos=None, n_dropped=None):
    np.testing.assert_array_equal(counts.cpu().numpy(), ref.cap.counts)
    np.testing.assert_array_equal(keep.cpu().numpy(), ref.cap.keep)
    np.testing.assert_array_equal(dropped.cpu().numpy(), ref.cap.dropped)
    if pos is not None:
        np.testing.assert_array_equal(pos.cpu().numpy(), ref.cap.pos)
    if n_dropped is not None:
        assert int(n_dropped.item()) == ref.cap.n_dropped


def tile_stratified_tokens(topk, pos, keep, E, seed=54, tile=128):
    """Tokens that reach every tile of every expert segment: for each expert,
    one kept row drawn at random inside each 128-row tile of its segment (so
    both 128-row halves of every 256-row SM-pair tile, and a varying TMEM lane
    and epilogue warp), plus the segment's first and last kept rows; mapped
    back to the token that owns the row."""
    rng = np.random.default_rng(seed)
    kept_rows = {}
    t_idx, j_idx = np.nonzero(keep)
    for t, j in zip(t_idx, j_idx):
        kept_rows.setdefault(int(topk[t, j]), {})[int(pos[t, j])] = int(t)
    tokens = set()
    for e in range(E):
        rows = kept_rows.get(e)
        if not rows:
            continue
        n = len(rows)
        assert sorted(rows) == list(range(n)), "kept positions of an expert are 0..kept-1"
        tokens.add(rows[0])
        tokens.add(rows[n - 1])
        for lo in range(0, n, tile):
            hi = min(lo + tile, n)
            tokens.add(rows[int(rng.integers(lo, hi))])
    return tokens


SMALL = {
    "tiny": CONFIGS["tiny"],
    "switch_small": shrink(CONFIGS["switch"], T=1000, d=256, d_ff=512),
    "mixtral_small": shrink(CONFIGS["mixtral"], T=700, d=512, d_ff=384),
    "mixtral_small_rank_major": shrink(CONFIGS["mixtral"], T=700, d=512, d_ff=384, priority=1,
                                       cf=1.0, zipf_s=1.1),
    "deepseekmoe_small": shrink(CONFIGS["deepseekmoe"], T=900, d=128, d_ff=128,
                                d_ff_shared=128),
    "deepseek_v3_small": shrink(CONFIGS["deepseek_v3"], T=333, d=192, d_ff=128,
                                d_ff_shared=192),
    "k_equals_E": shrink(CONFIGS["mixtral"], T=200, d=128, d_ff=128, E=4, k=4, cf=math.inf),
    "single_expert": shrink(CONFIGS["mixtral"], T=130, d=64, d_ff=64, E=1, k=1, cf=1.0),
    # T k = 512 E: the expert GEMMs run SM-pair (256-row) tiles over the full
    # Mixtral-shaped K (d = 4096, d_ff = 14336), many tiles per SM pair, odd
    # trailing 128-row halves; every token compared
    "mixtral_full_k_pair": shrink(CONFIGS["mixtral"], T=2048),
    # SM-pair tiles with GELU, and (top-1, no shared expert) the forward's
    # gate fused into GEMM2; 5 of the 8 segments end in an odd 128-row half
    # tile (the pair's second CTA computes rows it does not store)
    "switch_pair": shrink(CONFIGS["switch"], T=4096, d=512, d_ff=1024),
    # SM-pair SwiGLU tiles, fewer than the clusters in GEMM2 (36 tiles for 74
    # SM pairs) and about one per cluster in GEMM1, short K
    "mixtral_pair_few_tiles": shrink(CONFIGS["mixtral"], T=2048, d=512, d_ff=1024),
    # SM-pair SwiGLU tiles with two shared experts over T = 1900 rows: the
    # shared set ends in an odd, ragged 128-row half tile
    "deepseekmoe_pair": shrink(CONFIGS["deepseekmoe"], T=1900, d=256, d_ff=256,
                               d_ff_shared=256, E=16),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_every_token_matches_the_oracle(name):
    """Sizes the oracle finishes in seconds, several tiles and a ragged tail;
    every output row compared."""
    inp = remove_near_ties(generate(SMALL[name], device="cuda"))
    ref = oracle_forward(inp)
    out = run_stages(inp)
    check_routing(out["topk"], out["gates"], ref)
    check_capacity(out["cap"].counts, out["cap"].keep, out["cap"].dropped, ref, out["cap"].pos,
                   out["cap"].n_dropped)
    check_y(inp.shape, out["y"], ref.y)
    check_losses(out["aux"], out["zloss"], ref)
    np.testing.assert_allclose(out["logits"].double().cpu().numpy(), ref.route.z, rtol=1e-4,
                               atol=1e-4)
    fwd = run_forward(inp)
    assert torch.equal(fwd.topk, out["topk"])
    check_losses(fwd.aux, fwd.zloss, ref)
    if inp.shape.k == 1 and inp.shape.n_shared == 0:
        # the forward fuses this layer's combine into the expert GEMM (y rounded
        # once, not twice): its own comparison with the oracle
        check_y(inp.shape, fwd.y, ref.y)
    else:   # the same kernels as the stage calls
        assert torch.equal(fwd.y, out["y"])
        assert torch.equal(fwd.aux, out["aux"]) and torch.equal(fwd.zloss, out["zloss"])


def run_fused_combine(inp, gather, direct=False):
    """The combine's gate fused into GEMM2 (moe_expert_ffn_slots), then the
    ordered slot sum (moe_combine_slots); gather: the dispatch fused into GEMM1
    too (moe_dispatch_rows).  direct (k = 1, no shared expert): GEMM2 writes y
    itself, the dispatch zeroes the rows of dropped tokens."""
    s = inp.shape
    cfg = moe.moe_config(s)
    topk, gates, _, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    cap = moe.moe_capacity(cfg, topk)
    R = moe.moe_perm_rows(cfg)
    y = torch.full((s.T, s.d), float("nan"), dtype=inp.x.dtype, device="cuda")
    if gather:
        slot = moe.moe_dispatch_rows(cfg, topk, cap.pos, cap.keep, cap.offsets)
        x_perm = None
    else:
        slot = torch.empty((R,), dtype=torch.int32, device="cuda")
        x_perm = moe.moe_dispatch(cfg, inp.x, topk, cap.pos, cap.keep, cap.offsets,
                                  src_slot=slot, zero_rows=y if direct else None)
    Y_slot, Ysh, ws = moe.moe_expert_ffn_slots(cfg, x_perm, inp.x, slot, cap.offsets, cap.kept,
                                               gates, inp.W1, inp.W3, inp.W2, inp.Ws1, inp.Ws3,
                                               inp.Ws2, Y_slot=y if direct else None)
    if not direct:
        moe.moe_combine_slots(cfg, Y_slot, Ysh, cap.keep, y=y)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    return y, topk, cap


FUSED = [n for n in SMALL if n != "mixtral_full_k_pair"]


@pytest.mark.parametrize("gather", [False, True], ids=["copy", "gather"])
@pytest.mark.parametrize("name", FUSED)
def test_fused_combine_matches_the_oracle(name, gather):
    """NEXT-2: the gate applied in GEMM2's epilogue, each kept row written to
    its assignment's row, then a plain ordered sum of a token's contiguous
    rows; with and without the dispatch fused into GEMM1.  Every token
    compared with the oracle (dropped slots contribute nothing, fully dropped
    tokens get the shared experts or 0)."""
    inp = remove_near_ties(generate(SMALL[name], device="cuda"))
    ref = oracle_forward(inp)
    y, topk, cap = run_fused_combine(inp, gather)
    np.testing.assert_array_equal(topk.cpu().numpy(), ref.route.topk)
    np.testing.assert_array_equal(cap.keep.cpu().numpy(), ref.cap.keep)
    check_y(inp.shape, y, ref.y)
    if inp.shape.k == 1 and inp.shape.n_shared == 0 and not gather:
        y2, _, _ = run_fused_combine(inp, gather, direct=True)
        check_y(inp.shape, y2, ref.y)
        assert not torch.isnan(y2.float()).any()   # dropped tokens' rows were zeroed


def test_drops_happen_and_dropped_tokens_get_zero():
    """Zipf-skewed Switch-style routing at cf = 1: tokens are dropped, and a
    fully dropped token's output is exactly zero (the residual is the
    caller's)."""
    inp = remove_near_ties(generate(SMALL["switch_small"], device="cuda"))
    ref = oracle_forward(inp)
    assert ref.cap.n_dropped > 0
    fwd = run_forward(inp)
    dropped = np.nonzero(ref.cap.dropped)[0]
    assert dropped.size > 0
    assert torch.count_nonzero(fwd.y[torch.as_tensor(dropped, device="cuda")]).item() == 0


@pytest.mark.parametrize("name", ["tiny", "switch", "mixtral", "deepseekmoe", "deepseek_v3"])
def test_full_size_config(name):
    """Full sizes, launched as the benchmark launches them: routing, capacity
    and drops bit-exact on every token, losses on every token, y on a
    tile-stratified sample of tokens the oracle computes one by one (a row in
    every 128-row tile of every expert segment, each segment's first and last
    kept rows, the first and last token and a dropped token)."""
    shape = CONFIGS[name]
    inp = remove_near_ties(generate(shape, device="cuda"))
    fwd = run_forward(inp)
    r = oracle_route(inp)
    cap = oracle.capacity_walk(r.topk, shape.E, shape.cf, shape.priority)
    aux, zl = oracle.losses(r.scores, cap.counts, r.lse, shape.k, shape.score)
    np.testing.assert_array_equal(fwd.topk.cpu().numpy(), r.topk)
    np.testing.assert_allclose(fwd.gates.double().cpu().numpy(), r.gates, rtol=1e-5, atol=1e-6)
    np.testing.assert_array_equal(fwd.counts.cpu().numpy(), cap.counts)
    np.testing.assert_array_equal(fwd.keep.cpu().numpy(), cap.keep)
    np.testing.assert_array_equal(fwd.dropped.cpu().numpy(), cap.dropped)
    assert int(fwd.n_dropped.item()) == cap.n_dropped
    assert float(fwd.aux.item()) == pytest.approx(aux, rel=LOSS_RTOL)
    assert float(fwd.zloss.item()) == pytest.approx(zl, rel=LOSS_RTOL)
    # y on a tile-stratified sample: every 128-row tile of every expert
    # segment (both halves of each SM-pair tile) holds a compared row
    tokens = tile_stratified_tokens(r.topk, cap.pos, cap.keep, shape.E)
    tokens |= {0, shape.T - 1}
    dropped = np.nonzero(cap.dropped)[0]
    if dropped.size:
        tokens.add(int(dropped[0]))
    tokens = np.array(sorted(tokens), dtype=np.int32)
    y_ref = oracle.ffn_tokens(storage(inp.x), r.topk, r.gates, cap.keep, storage(inp.W1),
                              storage(inp.W3), storage(inp.W2), shape.act, storage(inp.Ws1),
                              storage(inp.Ws3), storage(inp.Ws2), tokens)
    check_y(shape, fwd.y[torch.as_tensor(tokens, device="cuda").long()], y_ref)
    # the per-stage losses call (its partials staged through shared memory in
    # several row tiles at these sizes) gives the forward's bits
    cfg = moe.moe_config(shape)
    topk, _, part, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    aux_s, z_s = moe.moe_losses(cfg, moe.moe_capacity(cfg, topk).counts, part)
    assert torch.equal(aux_s, fwd.aux) and torch.equal(z_s, fwd.zloss)
    del inp, fwd
    torch.cuda.empty_cache()


LONG = {
    # 2048 rows of loss partials with 65 columns (3 row phases, 17 shared tiles)
    "deepseekmoe_long": shrink(CONFIGS["deepseekmoe"], T=65536, d=128, d_ff=128,
                               d_ff_shared=128),
    # 625 rows with 257 columns (one phase, ragged last tile and token block)
    "deepseek_v3_long": shrink(CONFIGS["deepseek_v3"], T=20000, d=128, d_ff=128,
                               d_ff_shared=128),
}


@pytest.mark.parametrize("name", list(LONG))
def test_losses_over_many_token_blocks(name):
    """Both losses over many token blocks: the forward (losses in its capacity
    launch) and the per-stage call against the oracle, and bit for bit against
    each other."""
    shape = LONG[name]
    inp = remove_near_ties(generate(shape, device="cuda"))
    fwd = run_forward(inp)
    r = oracle_route(inp)
    cap = oracle.capacity_walk(r.topk, shape.E, shape.cf, shape.priority)
    aux, zl = oracle.losses(r.scores, cap.counts, r.lse, shape.k, shape.score)
    np.testing.assert_array_equal(fwd.counts.cpu().numpy(), cap.counts)
    assert float(fwd.aux.item()) == pytest.approx(aux, rel=LOSS_RTOL)
    assert float(fwd.zloss.item()) == pytest.approx(zl, rel=LOSS_RTOL)
    cfg = moe.moe_config(shape)
    topk, _, part, _, _ = moe.moe_route(cfg, inp.x, inp.W_r, inp.logit_bias, inp.select_bias)
    aux_s, z_s = moe.moe_losses(cfg, moe.moe_capacity(cfg, topk).counts, part)
    assert torch.equal(aux_s, fwd.aux) and torch.equal(z_s, fwd.zloss)
    del inp, fwd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("kind", ["balanced", "skewed"])
def test_mixtral_balanced_and_skewed(kind):
    shape = mixtral_variant(kind)
    inp = generate(shape, device="cuda")
    if kind == "skewed":
        remove_near_ties(inp)
    fwd = run_forward(inp)
    r = oracle_route(inp)
    cap = oracle.capacity_walk(r.topk, shape.E, shape.cf, shape.priority)
    np.testing.assert_array_equal(fwd.topk.cpu().numpy(), r.topk)
    np.testing.assert_array_equal(fwd.keep.cpu().numpy(), cap.keep)
    if kind == "balanced":
        a, b = balanced_assignment(shape.T, shape.E)
        np.testing.assert_array_equal(r.topk, np.stack([a.numpy(), b.numpy()], axis=1))
        np.testing.assert_array_equal(fwd.counts.cpu().numpy(), np.full(shape.E, 2 * shape.T // shape.E))
        assert int(fwd.n_dropped.item()) == 0
        assert float(fwd.aux.item()) == pytest.approx(1.0, abs=1e-6)
    else:
        assert cap.n_dropped > 0
        assert int(fwd.n_dropped.item()) == cap.n_dropped
    del inp, fwd
    torch.cuda.empty_cache()


def test_zero_tokens_is_a_no_op():
    shape = shrink(CONFIGS["mixtral"], T=0, d=128, d_ff=128)
    cfg = moe.moe_config(shape)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    W_r = torch.randn((128, 8), device="cuda")
    W = torch.randn((8, 128, 128), device="cuda").to(torch.bfloat16)
    y, aux, zl, fwd = moe.moe_forward(cfg, x, W_r, W, W, W3=W)
    torch.cuda.synchronize()
    assert y.shape == (0, 128)
    assert int(fwd.counts.sum().item()) == 0
