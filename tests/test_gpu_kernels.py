"""Stage-level GPU tests through the C ABI: each kernel against a plain
float64 PyTorch (or pure integer) reference of the same operation on the same
inputs.  End-to-end parity with the oracle is in test_gpu_parity.py."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mixture_experts_layer_54_b200 as moe

DEV = "cuda"
BF16_REL_FROB = 1e-2
BF16_MAX_ABS = 2e-2


def _ffn_ref(x, W1, W3, W2, act):
    x, W1, W2 = x.double(), W1.double(), W2.double()
    h = x @ W1.T
    h = Fn.gelu(h) if act == 0 else Fn.silu(h) * (x @ W3.double().T)
    return h @ W2.T


def _close_bf16(got, ref):
    got = got.double().cpu()
    ref = ref.double().cpu()
    err = (got - ref)
    frob = err.norm() / max(ref.norm().item(), 1e-30)
    mx = err.abs().max().item()
    scale = ref.abs().max().item()
    assert frob <= BF16_REL_FROB, f"relative Frobenius error {frob:.3e}"
    assert mx <= BF16_MAX_ABS * scale, f"max abs error {mx:.3e} vs max|y| {scale:.3e}"


def _segments(kept, align=128):
    offsets = [0]
    for c in kept:
        offsets.append(offsets[-1] + (c + align - 1) // align * align)
    return offsets


@pytest.mark.parametrize("pair", [False, True], ids=["1sm", "2sm"])
@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("dims", [(256, 384), (512, 128), (192, 256)])
def test_expert_ffn_grouped_gemm_against_torch(act, dims, pair):
    """Ragged segments (empty, 1 row, 127, 128, 129, several tiles) through the
    tcgen05 grouped GEMM; every kept row compared with its expert's FFN.  T*k
    >= 512*E selects SM-pair (256-row) tiles, smaller T single-SM tiles."""
    d, F = dims
    kept = [0, 1, 127, 128, 129, 300, 5, 260]
    E = len(kept)
    T = 2048 if pair else 400
    cfg = moe.moe_config(T=T, d=d, E=E, k=2, d_ff=F, act=act, dtype=1, cf=math.inf)
    R = moe.moe_perm_rows(cfg)
    offsets = _segments(kept)
    assert offsets[-1] <= R
    g = torch.Generator(device=DEV).manual_seed(7)
    x_perm = torch.randn((R, d), generator=g, device=DEV).to(torch.bfloat16)
    W1 = (torch.randn((E, F, d), generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    W3 = (torch.randn((E, F, d), generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16) \
        if act == 1 else None
    W2 = (torch.randn((E, d, F), generator=g, device=DEV) / math.sqrt(F)).to(torch.bfloat16)
    off_t = torch.tensor(offsets, dtype=torch.int32, device=DEV)
    Y, _, ws = moe.moe_expert_ffn(cfg, x_perm, off_t, W1, W3, W2)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    for e in range(E):
        if kept[e] == 0:
            continue
        rows = slice(offsets[e], offsets[e] + kept[e])
        ref = _ffn_ref(x_perm[rows], W1[e], None if W3 is None else W3[e], W2[e], act)
        _close_bf16(Y[rows], ref)


@pytest.mark.parametrize("act", [0, 1])
def test_pair_gemm_with_many_tiles_per_sm_pair(act):
    """SM-pair tiles where every SM pair runs many tiles in turn (GEMM1: 16 N
    tiles x ~70 row pairs over 74 pairs), so the TMEM double buffer and the
    shared-memory ring wrap many times; ragged segments, every kept row
    compared with its expert's FFN in float64."""
    d, F = 1024, 2048
    kept = [4000, 1, 2900, 0, 5000, 129, 2047, 3300]
    E = len(kept)
    cfg = moe.moe_config(T=16384, d=d, E=E, k=2, d_ff=F, act=act, dtype=1, cf=math.inf)
    R = moe.moe_perm_rows(cfg)
    offsets = _segments(kept)
    assert offsets[-1] <= R
    g = torch.Generator(device=DEV).manual_seed(17 + act)
    x_perm = torch.randn((R, d), generator=g, device=DEV).to(torch.bfloat16)
    W1 = (torch.randn((E, F, d), generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
    W3 = (torch.randn((E, F, d), generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16) \
        if act == 1 else None
    W2 = (torch.randn((E, d, F), generator=g, device=DEV) / math.sqrt(F)).to(torch.bfloat16)
    off_t = torch.tensor(offsets, dtype=torch.int32, device=DEV)
    Y, _, ws = moe.moe_expert_ffn(cfg, x_perm, off_t, W1, W3, W2)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    for e in range(E):
        if kept[e] == 0:
            continue
        rows = slice(offsets[e], offsets[e] + kept[e])
        ref = _ffn_ref(x_perm[rows], W1[e], None if W3 is None else W3[e], W2[e], act)
        _close_bf16(Y[rows], ref)
        # and row by row: no row may be wrong while the segment's norm is fine
        err = (Y[rows].double() - ref).abs().amax(dim=1)
        assert err.max().item() <= BF16_MAX_ABS * ref.abs().max().item()


def test_capacity_with_a_huge_factor_keeps_everything():
    """A finite factor far above T k / E holds C at T: nothing is dropped
    (the integer conversion of ceil(cf T k / E) would overflow otherwise)."""
    T, E, k = 1000, 8, 2
    rng = np.random.default_rng(3)
    topk = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    cfg = moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=1e20)
    assert moe.moe_capacity_value(cfg) == T
    cap = moe.moe_capacity(cfg, torch.tensor(topk, device=DEV))
    torch.cuda.synchronize()
    assert int(cap.n_dropped.item()) == 0
    assert bool(cap.keep.bool().all().item())
    np.testing.assert_array_equal(cap.counts.cpu().numpy(), np.bincount(topk.ravel(), minlength=E))


@pytest.mark.parametrize("act,S,T", [(1, 2, 333), (0, 1, 333), (1, 1, 333), (1, 2, 2100),
                                     (0, 1, 2100)])
def test_shared_experts_against_torch(act, S, T):
    d, F, Fs, E = 256, 128, 192, 4
    cfg = moe.moe_config(T=T, d=d, E=E, k=1, d_ff=F, act=act, dtype=1, cf=math.inf,
                         n_shared=S, d_ff_shared=Fs)
    R = moe.moe_perm_rows(cfg)
    g = torch.Generator(device=DEV).manual_seed(11)
    rnd = lambda *s, sc=1.0: (torch.randn(s, generator=g, device=DEV) * sc).to(torch.bfloat16)
    x = rnd(T, d)
    x_perm = rnd(R, d)
    W1, W2 = rnd(E, F, d, sc=d ** -0.5), rnd(E, d, F, sc=F ** -0.5)
    W3 = rnd(E, F, d, sc=d ** -0.5) if act else None
    Ws1, Ws2 = rnd(S, Fs, d, sc=d ** -0.5), rnd(S, d, Fs, sc=Fs ** -0.5)
    Ws3 = rnd(S, Fs, d, sc=d ** -0.5) if act else None
    off_t = torch.tensor(_segments([T // 4] * E), dtype=torch.int32, device=DEV)
    Y, Ysh, ws = moe.moe_expert_ffn(cfg, x_perm, off_t, W1, W3, W2, x, Ws1, Ws3, Ws2)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    ref = sum(_ffn_ref(x, Ws1[s], None if Ws3 is None else Ws3[s], Ws2[s], act) for s in range(S))
    _close_bf16(Ysh, ref)


def test_expert_ffn_fp32_simt_against_torch():
    d, F, E, T = 32, 64, 4, 64
    kept = [40, 0, 13, 75]
    cfg = moe.moe_config(T=T, d=d, E=E, k=2, d_ff=F, act=0, dtype=0, cf=math.inf, n_shared=1,
                         d_ff_shared=48)
    R = moe.moe_perm_rows(cfg)
    offsets = _segments(kept)
    g = torch.Generator(device=DEV).manual_seed(3)
    x_perm = torch.randn((R, d), generator=g, device=DEV)
    x = torch.randn((T, d), generator=g, device=DEV)
    W1 = torch.randn((E, F, d), generator=g, device=DEV) / math.sqrt(d)
    W2 = torch.randn((E, d, F), generator=g, device=DEV) / math.sqrt(F)
    Ws1 = torch.randn((1, 48, d), generator=g, device=DEV) / math.sqrt(d)
    Ws2 = torch.randn((1, d, 48), generator=g, device=DEV) / math.sqrt(48)
    Y, Ysh, _ = moe.moe_expert_ffn(cfg, x_perm, torch.tensor(offsets, dtype=torch.int32,
                                                             device=DEV), W1, None, W2, x, Ws1,
                                   None, Ws2)
    torch.cuda.synchronize()
    for e in range(E):
        rows = slice(offsets[e], offsets[e] + kept[e])
        if kept[e]:
            ref = _ffn_ref(x_perm[rows], W1[e], None, W2[e], 0)
            err = (Y[rows].double() - ref).abs().max().item()
            assert err <= 1e-4 * ref.abs().max().item()
    ref = _ffn_ref(x, Ws1[0], None, Ws2[0], 0)
    assert (Ysh.double() - ref).abs().max().item() <= 1e-4 * ref.abs().max().item()


@pytest.mark.parametrize("priority", [0, 1])
@pytest.mark.parametrize("T,E,k,cf", [(1000, 8, 2, 1.0), (777, 64, 6, 1.25), (300, 256, 8, 1.0),
                                      (5, 4, 4, 1.0), (1, 3, 1, 1.0),
                                      # many capacity blocks (64 to 256 of 256 tokens),
                                      # a ragged last one
                                      (65536, 8, 2, 1.0), (16384, 64, 6, 1.5),
                                      (20000, 256, 8, 1.0)])
def test_capacity_bit_exact_with_sequential_walk(priority, T, E, k, cf):
    """Skewed random top-k lists (distinct experts per token) against the pages'
    one-hot cumulative-sum formulation, in integers (for long lists, the same
    positions from a stable sort by expert)."""
    rng = np.random.default_rng(T + E + priority)
    w = 1.0 / np.arange(1, E + 1) ** 1.1
    w = w / w.sum()
    if T <= 1000:
        topk = np.stack([rng.choice(E, size=k, replace=False, p=w) for _ in range(T)])
    else:   # k distinct experts per token: the k smallest of exponential keys scaled by w
        keys = rng.exponential(size=(T, E)) / w
        topk = np.argsort(keys, axis=1)[:, :k]
    topk = topk.astype(np.int32)
    cfg = moe.moe_config(T=T, d=64, E=E, k=k, d_ff=64, dtype=1, cf=cf, priority=priority)
    C = moe.moe_capacity_value(cfg)
    out = moe.moe_capacity(cfg, torch.tensor(topk, device=DEV))
    flat = topk.reshape(-1) if priority == 0 else topk.T.reshape(-1)
    if T <= 1000:
        onehot = np.eye(E, dtype=np.int64)[flat]
        pf = np.take_along_axis(np.cumsum(onehot, axis=0), flat[:, None], axis=1)[:, 0] - 1
    else:   # place within the expert's list, the list in priority order (stable sort)
        order = np.argsort(flat, kind="stable")
        first = np.searchsorted(flat[order], np.arange(E))
        pf = np.empty(flat.size, dtype=np.int64)
        pf[order] = np.arange(flat.size) - first[flat[order]]
    pos = pf.reshape(T, k) if priority == 0 else pf.reshape(k, T).T
    counts = np.bincount(flat, minlength=E)
    kept = np.minimum(counts, C)
    keep = (pos < C).astype(np.uint8)
    np.testing.assert_array_equal(out.pos.cpu().numpy(), pos)
    np.testing.assert_array_equal(out.keep.cpu().numpy(), keep)
    np.testing.assert_array_equal(out.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(out.kept.cpu().numpy(), kept)
    np.testing.assert_array_equal(out.dropped.cpu().numpy(), (keep.sum(axis=1) == 0).astype(np.uint8))
    padded = (kept + 127) // 128 * 128
    np.testing.assert_array_equal(out.offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(padded)]))
    assert int(out.n_dropped.item()) == int((counts - kept).sum())


@pytest.mark.parametrize("dtype", [0, 1])
def test_dispatch_and_combine_move_rows_exactly(dtype):
    T, d, E, k = 300, 128, 8, 2
    tdt = torch.bfloat16 if dtype else torch.float32
    rng = np.random.default_rng(5)
    topk = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    cfg = moe.moe_config(T=T, d=d, E=E, k=k, d_ff=64, dtype=dtype, cf=1.0)
    cap = moe.moe_capacity(cfg, torch.tensor(topk, device=DEV))
    x = torch.randn((T, d), device=DEV).to(tdt)
    xp = moe.moe_dispatch(cfg, x, torch.tensor(topk, device=DEV), cap.pos, cap.keep, cap.offsets)
    pos, keep, off = cap.pos.cpu().numpy(), cap.keep.cpu().numpy(), cap.offsets.cpu().numpy()
    xp_c, x_c = xp.cpu(), x.cpu()
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                assert torch.equal(xp_c[off[topk[t, j]] + pos[t, j]], x_c[t])
    # combine: y = sum_j keep g Y_perm[row] + Y_sh + residual, fp32 accumulation in slot order
    Y_perm = torch.randn_like(xp)
    Y_sh = torch.randn((T, d), device=DEV).to(tdt)
    res = torch.randn((T, d), device=DEV).to(tdt)
    gates = torch.rand((T, k), device=DEV)
    y = moe.moe_combine(cfg, Y_perm, Y_sh, gates, torch.tensor(topk, device=DEV), cap.pos,
                        cap.keep, cap.offsets, residual=res)
    ref = torch.zeros((T, d), dtype=torch.float32)
    Yp, g = Y_perm.cpu().float(), gates.cpu()
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                ref[t] = ref[t] + g[t, j] * Yp[off[topk[t, j]] + pos[t, j]]
    ref = ref + Y_sh.cpu().float() + res.cpu().float()
    tol = 1e-6 if dtype == 0 else 8e-3
    assert (y.cpu().float() - ref).abs().max().item() <= tol * max(ref.abs().max().item(), 1.0)


def test_route_logits_and_selection_against_torch():
    T, d, E, k = 1000, 512, 64, 6
    g = torch.Generator(device=DEV).manual_seed(9)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    W_r = torch.randn((d, E), generator=g, device=DEV) * 0.05
    cfg = moe.moe_config(T=T, d=d, E=E, k=k, d_ff=64, dtype=1, cf=1.0)
    topk, gates, part, logits, scores = moe.moe_route(cfg, x, W_r, want_logits=True,
                                                      want_scores=True)
    z = x.double() @ W_r.double()
    # recursive fp32 summation bound: |dz| <= d * 2^-24 * sum |x_c W_c|
    bound = d * 2.0 ** -24 * (x.double().abs() @ W_r.double().abs())
    assert torch.all((logits.double() - z).abs() <= bound + 1e-7)
    p = torch.softmax(z, dim=1)
    assert (scores.double() - p).abs().max().item() < 1e-6
    # top-k of the GPU's own logits, lower index on ties
    lz = logits.double().cpu().numpy()
    ref = np.argsort(-lz, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(topk.cpu().numpy(), ref)
    sel = torch.gather(z, 1, topk.long())
    assert (gates.double() - torch.softmax(sel, dim=1)).abs().max().item() < 1e-5


def test_status_word_is_clear_after_a_normal_call():
    cfg = moe.moe_config(T=128, d=128, E=2, k=1, d_ff=128, act=1, dtype=1, cf=math.inf)
    R = moe.moe_perm_rows(cfg)
    x_perm = torch.zeros((R, 128), dtype=torch.bfloat16, device=DEV)
    W = torch.zeros((2, 128, 128), dtype=torch.bfloat16, device=DEV)
    off = torch.tensor([0, 128, 128], dtype=torch.int32, device=DEV)
    Y, _, ws = moe.moe_expert_ffn(cfg, x_perm, off, W, W, W)
    assert moe.moe_device_status(ws) == 0
    assert torch.count_nonzero(Y[:128]).item() == 0


def test_a_wait_that_runs_out_sets_the_status_and_leaves_the_context_usable():
    """The bounded wait of the expert GEMMs' roles, on a barrier nothing
    arrives on, gives up after its limit and records MOE_ERR_DEVICE_TIMEOUT;
    afterwards the same workspace, cleared, serves a normal call."""
    from mixture_experts_layer_54_b200 import _abi
    cfg = moe.moe_config(T=128, d=128, E=2, k=1, d_ff=128, act=1, dtype=1, cf=math.inf)
    ws = moe.workspace(moe.moe_stage_workspace_size(cfg), DEV)
    moe.moe_clear_device_status(ws)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    moe.moe_probe_wait_timeout(ws, 50_000_000)   # 50 ms
    end.record()
    assert moe.moe_device_status(ws) == _abi.MOE_ERR_DEVICE_TIMEOUT
    assert 40.0 <= start.elapsed_time(end) < 1000.0
    R = moe.moe_perm_rows(cfg)
    g = torch.Generator(device=DEV).manual_seed(1)
    x_perm = torch.randn((R, 128), generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn((2, 128, 128), generator=g, device=DEV) / 12).to(torch.bfloat16)
    off = torch.tensor([0, 128, 128], dtype=torch.int32, device=DEV)
    Y, _, _ = moe.moe_expert_ffn(cfg, x_perm, off, W, W, W, ws=ws)   # clears the word
    assert moe.moe_device_status(ws) == 0
    _close_bf16(Y[:128], _ffn_ref(x_perm[:128], W[0], W[0], W[0], 1))


@pytest.mark.parametrize("case", [
    # T, d, E, k, F, act, S, dtype (pair tiles when T k >= 512 E)
    (2048, 256, 8, 2, 384, 1, 0, 1),     # SM-pair tiles, SwiGLU
    (2048, 192, 4, 2, 256, 0, 1, 1),     # SM-pair tiles, GELU, shared expert
    (333, 128, 16, 3, 128, 1, 2, 1),     # single-SM tiles, shared experts
    (97, 32, 4, 2, 64, 0, 1, 0),         # fp32 SIMT
], ids=["pair_swiglu", "pair_gelu_shared", "1sm_shared", "fp32"])
def test_gathered_expert_ffn_equals_dispatch_then_ffn(case):
    """The dispatch fused into GEMM1 (rows gathered from x through the row
    table) gives exactly the result of the permuted copy followed by the GEMM,
    on every kept row; the row table matches one built on the host."""
    T, d, E, k, F, act, S, dt = case
    cfg = moe.moe_config(T=T, d=d, E=E, k=k, d_ff=F, act=act, dtype=dt, cf=1.0, n_shared=S,
                         d_ff_shared=128 if S else 0)
    tdt = torch.bfloat16 if dt == 1 else torch.float32
    g = torch.Generator(device=DEV).manual_seed(T + E)
    rnd = lambda *s, sc=1.0: (torch.randn(s, generator=g, device=DEV) * sc).to(tdt)
    x = rnd(T, d)
    W1, W2 = rnd(E, F, d, sc=d ** -0.5), rnd(E, d, F, sc=F ** -0.5)
    W3 = rnd(E, F, d, sc=d ** -0.5) if act == 1 else None
    Ws1 = rnd(S, 128, d, sc=d ** -0.5) if S else None
    Ws3 = rnd(S, 128, d, sc=d ** -0.5) if S and act == 1 else None
    Ws2 = rnd(S, d, 128, sc=128 ** -0.5) if S else None
    # skewed random top-k so that some assignments are dropped (cf = 1)
    pick = torch.rand((T, E), generator=g, device=DEV) + torch.linspace(0.5, 0, E, device=DEV)
    topk = pick.argsort(dim=1, descending=True)[:, :k].to(torch.int32).contiguous()
    cap = moe.moe_capacity(cfg, topk)
    slot_copy = torch.full((moe.moe_perm_rows(cfg),), -7, dtype=torch.int32, device=DEV)
    x_perm = moe.moe_dispatch(cfg, x, topk, cap.pos, cap.keep, cap.offsets, src_slot=slot_copy)
    Y_ref, Ysh_ref, ws1 = moe.moe_expert_ffn(cfg, x_perm, cap.offsets, W1, W3, W2, x, Ws1, Ws3,
                                             Ws2)
    rows = moe.moe_dispatch_rows(cfg, topk, cap.pos, cap.keep, cap.offsets)
    Y, Ysh, ws2 = moe.moe_expert_ffn_gather(cfg, x, rows, cap.offsets, W1, W3, W2, Ws1, Ws3, Ws2)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws1) == 0 and moe.moe_device_status(ws2) == 0
    tk, pos, keep = topk.cpu().numpy(), cap.pos.cpu().numpy(), cap.keep.cpu().numpy()
    off = cap.offsets.cpu().numpy()
    assert keep.sum() < T * k   # something was dropped
    # the table: row offsets[e] + pos[t, j] holds assignment t k + j, padding -1
    want = np.full(moe.moe_perm_rows(cfg), -1, np.int32)
    kept_rows = []
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                r = off[tk[t, j]] + pos[t, j]
                want[r] = t * k + j
                kept_rows.append(r)
    np.testing.assert_array_equal(rows.cpu().numpy(), want)
    # the copying dispatch writes the same entries for kept rows, no others
    sc = slot_copy.cpu().numpy()
    np.testing.assert_array_equal(sc[kept_rows], want[kept_rows])
    assert np.all(np.delete(sc, kept_rows) == -7)
    kr = torch.as_tensor(kept_rows, device=DEV, dtype=torch.long)
    assert torch.equal(Y[kr], Y_ref[kr])
    if S:
        assert torch.equal(Ysh, Ysh_ref)


def _check_route(T, d, E, k, score, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    W_r = torch.randn((d, E), generator=g, device=DEV) * 0.05
    sb = ((torch.rand(E, generator=g, device=DEV) - 0.5) * 0.2) if score == 1 else None
    cfg = moe.moe_config(T=T, d=d, E=E, k=k, d_ff=64, dtype=1, cf=1.0, score=score)
    topk, gates, part, logits, scores = moe.moe_route(cfg, x, W_r, None, sb, want_logits=True,
                                                      want_scores=True)
    torch.cuda.synchronize()
    # the logits are the fp32 router: within the recursive-summation bound of x W_r
    z = x.double() @ W_r.double()
    bound = d * 2.0 ** -24 * (x.double().abs() @ W_r.double().abs())
    assert torch.all((logits.double() - z).abs() <= bound + 1e-7)
    key = logits if score == 0 else scores + sb   # fp32, as the kernel ranks
    ref = np.argsort(-key.double().cpu().numpy(), axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(topk.cpu().numpy(), ref)
    sel = torch.gather(scores.double(), 1, topk.long())
    want = sel / sel.sum(1, keepdim=True) if k > 1 else sel
    assert (gates.double() - want).abs().max().item() < 1e-6
    # loss partials: the probability mass per expert and lse^2, summed over the batch
    rows = part.view(-1, E + 1).double()
    assert rows.shape[0] == (T + 31) // 32
    p = scores.double() if score == 0 else scores.double() / scores.double().sum(1, keepdim=True)
    np.testing.assert_allclose(rows[:, :E].sum(0).cpu().numpy(), p.sum(0).cpu().numpy(),
                               rtol=1e-5, atol=1e-4)
    lse = torch.logsumexp(logits.double(), dim=1)
    assert rows[:, E].sum().item() == pytest.approx((lse ** 2).sum().item(), rel=1e-5)
    # each row holds its own 32 tokens
    r0 = rows[0].cpu()
    assert r0[:E].numpy() == pytest.approx(p[:32].sum(0).cpu().numpy(), rel=1e-5, abs=1e-5)


@pytest.mark.parametrize("E,k", [(9, 2), (16, 4), (32, 8), (33, 3), (64, 6), (96, 8), (128, 1),
                                 (129, 5), (200, 8), (256, 8)])
@pytest.mark.parametrize("score", [0, 1], ids=["softmax", "sigmoid"])
def test_route_selection_every_width(E, k, score):
    """The selection at every lane width (1, 2, 4 or 8 experts per lane),
    ragged expert counts included: top-k of the kernel's own fp32 keys with
    ties to the lower index, gates, and the loss partials."""
    _check_route(1000, 256, E, k, score, E * 10 + k + score)


@pytest.mark.parametrize("T,d,E,k", [(1000, 1024, 8, 2), (777, 512, 40, 3),
                                     (16384, 1024, 64, 6), (500, 512, 100, 8)])
def test_route_with_unaligned_router_weights_gives_the_same_bits(T, d, E, k):
    """W_r 16-byte aligned and W_r four bytes off give the same top-k, gates,
    loss partials and logits, bit for bit (the one-kernel router copies W_r in
    4-byte pieces, the three-launch split reads it per element)."""
    g = torch.Generator(device=DEV).manual_seed(T + E)
    x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
    W_r = torch.randn((d, E), generator=g, device=DEV) * 0.05
    buf = torch.empty(d * E + 1, device=DEV)
    W_off = buf[1:].view(d, E)
    W_off.copy_(W_r)
    assert W_r.data_ptr() % 16 == 0 and W_off.data_ptr() % 16 == 4
    cfg = moe.moe_config(T=T, d=d, E=E, k=k, d_ff=64, dtype=1, cf=1.0)
    a = moe.moe_route(cfg, x, W_r, want_logits=True)
    b = moe.moe_route(cfg, x, W_off, want_logits=True)
    torch.cuda.synchronize()
    for u, v in zip(a[:4], b[:4]):
        assert torch.equal(u, v)


@pytest.mark.parametrize("T,d,E,k", [
    (1000, 1024, 4, 1),    # one kernel: 4 experts per token group, K in 4 parts (cluster of 4)
    (777, 512, 8, 2),      # 8 experts per token group, K in 2 parts
    (1000, 1024, 16, 4),   # a warp per token, K in 4 parts
    (600, 512, 40, 3),     # three launches: 48 padded experts, two per lane
    (333, 1024, 64, 6),    # three launches: 64 experts in one chunk, ragged last tile
    (16384, 1024, 8, 2),   # one kernel: 128 tiles, a cluster of 2 per tile (grid within one wave)
    (16384, 1024, 64, 6),  # DeepSeekMoE-shaped: three launches
    (20000, 512, 32, 4),   # three launches, 157 tiles, ragged last tile
    (500, 512, 100, 8),    # three launches: 2 expert chunks x 2 K parts
    (64, 256, 8, 2),       # less than one 128-token tile (one block, K whole)
    (40, 256, 200, 8),     # three launches: 4 expert chunks, two rows of the loss partials
])
@pytest.mark.parametrize("score", [0, 1], ids=["softmax", "sigmoid"])
def test_route_cluster_shapes(T, d, E, k, score):
    """Every way the router splits the work (one kernel: K parts over a
    cluster of 1, 2 or 4 blocks per 128-token tile; three launches: expert
    chunks and K parts): the same checks as above."""
    _check_route(T, d, E, k, score, T + d + E + k + score)
