"""Thin torch-facing binding of the C ABI: same names as the C calls, argument
marshalling only (device pointers, sizes, the current CUDA stream).  Every
step of the layer runs in the library's kernels; output tensors are allocated
here with torch, which is the library's memory manager.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi
from ._abi import MoeConfig, MoeOutputs, MoeWeights, check, lib

DTYPE_F32, DTYPE_BF16 = 0, 1


def moe_config(shape=None, **kw) -> MoeConfig:
    """Build the C config from any object with the layer's attributes
    (T, d, E, k, d_ff, act, dtype, cf, and optionally n_shared, d_ff_shared,
    score, renorm, priority) and/or keyword overrides."""
    def get(name, default=None):
        if name in kw:
            return kw[name]
        if shape is not None and hasattr(shape, name):
            return getattr(shape, name)
        return default
    cf = get("cf", get("capacity_factor", 1.0))
    return MoeConfig(T=get("T"), d=get("d"), E=get("E"), k=get("k"), d_ff=get("d_ff"),
                     n_shared=get("n_shared", 0), d_ff_shared=get("d_ff_shared", 0),
                     act=get("act", 0), score=get("score", 0), renorm=get("renorm", -1),
                     dtype=get("dtype", DTYPE_BF16), priority=get("priority", 0),
                     capacity_factor=float(cf))


def _p(t):
    """Device pointer of a tensor argument (None passes a null pointer).  The
    library reads and writes dense row-major buffers, so a strided view is
    refused rather than read as if it were dense."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("moe ops take contiguous tensors (call .contiguous() on views)")
    if not t.is_cuda:
        raise ValueError("moe ops take CUDA tensors")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device (and the no-allocation
        # capacity call uses that device's static scratch)
        raise ValueError(f"tensor on {t.device} but the current device is "
                         f"cuda:{torch.cuda.current_device()}: use torch.cuda.device(...)")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _tdtype(cfg: MoeConfig):
    return torch.bfloat16 if cfg.dtype == DTYPE_BF16 else torch.float32


def _dev(t):
    return t.device


def moe_validate(cfg: MoeConfig):
    check(lib().moe_validate(ctypes.byref(cfg)), "moe_validate")


def moe_capacity_value(cfg: MoeConfig) -> int:
    C = ctypes.c_int64()
    check(lib().moe_capacity_value(ctypes.byref(cfg), ctypes.byref(C)), "moe_capacity_value")
    return int(C.value)


def moe_perm_rows(cfg: MoeConfig) -> int:
    moe_validate(cfg)
    return int(lib().moe_perm_rows(ctypes.byref(cfg)))


def moe_loss_partials_count(cfg: MoeConfig) -> int:
    moe_validate(cfg)
    return int(lib().moe_loss_partials_count(ctypes.byref(cfg)))


def moe_stage_workspace_size(cfg: MoeConfig) -> int:
    moe_validate(cfg)
    return int(lib().moe_stage_workspace_size(ctypes.byref(cfg)))


def moe_workspace_size(cfg: MoeConfig) -> int:
    moe_validate(cfg)
    return int(lib().moe_workspace_size(ctypes.byref(cfg)))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned uint8 device buffer (torch's allocator aligns to 512)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def moe_route(cfg: MoeConfig, x, W_r, logit_bias=None, select_bias=None, want_logits=False,
              want_scores=False, ws=None):
    dev = _dev(x)
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    T, k, E = cfg.T, cfg.k, cfg.E
    topk = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    partials = torch.empty((max(moe_loss_partials_count(cfg), 1),), dtype=torch.float32,
                           device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev) if want_logits else None
    scores = torch.empty((T, E), dtype=torch.float32, device=dev) if want_scores else None
    check(lib().moe_route(ctypes.byref(cfg), _p(x), _p(W_r), _p(logit_bias), _p(select_bias),
                          _p(topk), _p(gates), _p(partials), _p(logits), _p(scores), _p(ws),
                          ws.numel(), _stream()), "moe_route")
    return topk, gates, partials, logits, scores


@dataclass
class CapacityOut:
    counts: torch.Tensor
    pos: torch.Tensor
    keep: torch.Tensor
    kept: torch.Tensor
    offsets: torch.Tensor
    dropped: torch.Tensor
    n_dropped: torch.Tensor


def moe_capacity(cfg: MoeConfig, topk, ws=None) -> CapacityOut:
    dev = _dev(topk)
    T, k, E = cfg.T, cfg.k, cfg.E
    out = CapacityOut(
        counts=torch.empty((E,), dtype=torch.int32, device=dev),
        pos=torch.empty((T, k), dtype=torch.int32, device=dev),
        keep=torch.empty((T, k), dtype=torch.uint8, device=dev),
        kept=torch.empty((E,), dtype=torch.int32, device=dev),
        offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
        dropped=torch.empty((T,), dtype=torch.uint8, device=dev),
        n_dropped=torch.empty((1,), dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_capacity(ctypes.byref(cfg), _p(topk), _p(out.counts), _p(out.pos),
                             _p(out.keep), _p(out.kept), _p(out.offsets), _p(out.dropped),
                             _p(out.n_dropped), _p(ws), ws.numel(), _stream()), "moe_capacity")
    return out


def moe_capacity_scored(cfg: MoeConfig, topk, scores, ws=None) -> CapacityOut:
    """Batch-prioritized capacity: scores [T, E] fp32 are moe_route's
    scores_out; cfg.priority must be 2 (score order)."""
    dev = _dev(topk)
    T, k, E = cfg.T, cfg.k, cfg.E
    out = CapacityOut(
        counts=torch.empty((E,), dtype=torch.int32, device=dev),
        pos=torch.empty((T, k), dtype=torch.int32, device=dev),
        keep=torch.empty((T, k), dtype=torch.uint8, device=dev),
        kept=torch.empty((E,), dtype=torch.int32, device=dev),
        offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
        dropped=torch.empty((T,), dtype=torch.uint8, device=dev),
        n_dropped=torch.empty((1,), dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_capacity_scored(ctypes.byref(cfg), _p(topk), _p(scores), _p(out.counts),
                                    _p(out.pos), _p(out.keep), _p(out.kept), _p(out.offsets),
                                    _p(out.dropped), _p(out.n_dropped), _p(ws), ws.numel(),
                                    _stream()), "moe_capacity_scored")
    return out


def moe_capacity_sharded(cfg: MoeConfig, capacity: int, shard_counts, shard: int, topk,
                         ws=None) -> CapacityOut:
    """Capacity of one shard of a token-ordered batch split across ranks:
    shard_counts [n_shards, E] int32 are every shard's per-expert counts (see
    gather_shard_counts), `capacity` the whole batch's C."""
    dev = _dev(topk)
    T, k, E = cfg.T, cfg.k, cfg.E
    out = CapacityOut(
        counts=torch.empty((E,), dtype=torch.int32, device=dev),
        pos=torch.empty((T, k), dtype=torch.int32, device=dev),
        keep=torch.empty((T, k), dtype=torch.uint8, device=dev),
        kept=torch.empty((E,), dtype=torch.int32, device=dev),
        offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
        dropped=torch.empty((T,), dtype=torch.uint8, device=dev),
        n_dropped=torch.empty((1,), dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_capacity_sharded(ctypes.byref(cfg), int(capacity), _p(shard_counts),
                                     int(shard_counts.shape[0]), int(shard), _p(topk),
                                     _p(out.counts), _p(out.pos), _p(out.keep), _p(out.kept),
                                     _p(out.offsets), _p(out.dropped), _p(out.n_dropped), _p(ws),
                                     ws.numel(), _stream()), "moe_capacity_sharded")
    return out


def gather_shard_counts(counts, group=None):
    """All-gather of every rank's per-expert counts [E] into [world, E], rank
    order (the one exchange the token-order capacity needs across shards)."""
    import torch.distributed as dist
    parts = [torch.empty_like(counts) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, counts, group=group)
    return torch.stack(parts)


def shard_losses(cfg_global: MoeConfig, counts, loss_partials, group=None):
    """Switch loss and z-loss of the whole batch from the shards' own counts and
    loss partials: counts all-reduced (sum), partial rows all-gathered in rank
    order (every shard's token count a multiple of 32, so the rows line up
    with the whole batch's), then moe_losses on the whole batch's config."""
    import torch.distributed as dist
    total = counts.clone()
    dist.all_reduce(total, group=group)
    rows = [torch.empty_like(loss_partials) for _ in range(dist.get_world_size(group))]
    dist.all_gather(rows, loss_partials, group=group)
    return moe_losses(cfg_global, total, torch.cat(rows))


def moe_seq_balance_loss(cfg: MoeConfig, seq_len: int, topk, loss_partials, per_seq=None,
                         loss=None):
    """Sequence-wise balance loss over sequences of seq_len tokens; returns
    (loss [1], per_seq [T / seq_len]) as device fp32 tensors."""
    dev = _dev(topk)
    if per_seq is None:
        per_seq = torch.empty((max(cfg.T // max(seq_len, 1), 1),), dtype=torch.float32,
                              device=dev)
    if loss is None:
        loss = torch.empty((1,), dtype=torch.float32, device=dev)
    check(lib().moe_seq_balance_loss(ctypes.byref(cfg), int(seq_len), _p(topk),
                                     _p(loss_partials), _p(per_seq), _p(loss), _stream()),
          "moe_seq_balance_loss")
    return loss, per_seq


def moe_bias_update(cfg: MoeConfig, counts, gamma: float, select_bias):
    """One auxiliary-loss-free balancing step on select_bias (in place)."""
    check(lib().moe_bias_update(ctypes.byref(cfg), _p(counts), ctypes.c_float(gamma),
                                _p(select_bias), _stream()), "moe_bias_update")
    return select_bias


def moe_capacity_noalloc(cfg: MoeConfig, topk) -> CapacityOut:
    """moe_capacity with the library's own static scratch instead of a
    workspace (for callers that cannot allocate device memory)."""
    dev = _dev(topk)
    T, k, E = cfg.T, cfg.k, cfg.E
    out = CapacityOut(
        counts=torch.empty((E,), dtype=torch.int32, device=dev),
        pos=torch.empty((T, k), dtype=torch.int32, device=dev),
        keep=torch.empty((T, k), dtype=torch.uint8, device=dev),
        kept=torch.empty((E,), dtype=torch.int32, device=dev),
        offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
        dropped=torch.empty((T,), dtype=torch.uint8, device=dev),
        n_dropped=torch.empty((1,), dtype=torch.int32, device=dev))
    check(lib().moe_capacity_noalloc(ctypes.byref(cfg), _p(topk), _p(out.counts), _p(out.pos),
                                     _p(out.keep), _p(out.kept), _p(out.offsets),
                                     _p(out.dropped), _p(out.n_dropped), _stream()),
          "moe_capacity_noalloc")
    return out


def moe_dispatch(cfg: MoeConfig, x, topk, pos, keep, offsets, x_perm=None, src_slot=None,
                 zero_rows=None):
    """Permuted rows; with src_slot (an int32 [moe_perm_rows] tensor) also the
    assignment t k + j each kept row holds; with zero_rows ([T, d]) the rows of
    tokens whose every slot was dropped are zeroed there."""
    if x_perm is None:
        x_perm = torch.empty((moe_perm_rows(cfg), cfg.d), dtype=_tdtype(cfg), device=_dev(x))
    check(lib().moe_dispatch(ctypes.byref(cfg), _p(x), _p(topk), _p(pos), _p(keep), _p(offsets),
                             _p(x_perm), _p(src_slot), _p(zero_rows), _stream()), "moe_dispatch")
    return x_perm


def moe_dispatch_rows(cfg: MoeConfig, topk, pos, keep, offsets, src_slot=None):
    """The dispatch as a row table: src_slot[r] = t k + j, the assignment whose
    token row goes to permuted row r (-1 for padding rows), for the GEMMs that
    gather their rows from x."""
    if src_slot is None:
        src_slot = torch.empty((moe_perm_rows(cfg),), dtype=torch.int32, device=_dev(offsets))
    check(lib().moe_dispatch_rows(ctypes.byref(cfg), _p(topk), _p(pos), _p(keep), _p(offsets),
                                  _p(src_slot), _stream()), "moe_dispatch_rows")
    return src_slot


def moe_expert_ffn_gather(cfg: MoeConfig, x, src_slot, offsets, W1, W3, W2, Ws1=None, Ws3=None,
                          Ws2=None, ws=None, Y_perm=None, Y_shared=None):
    """moe_expert_ffn with the dispatch fused in: routed rows read from x
    through src_slot."""
    dev = _dev(x)
    if Y_perm is None:
        Y_perm = torch.empty((moe_perm_rows(cfg), cfg.d), dtype=_tdtype(cfg), device=dev)
    if cfg.n_shared > 0 and Y_shared is None:
        Y_shared = torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=dev)
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_expert_ffn_gather(ctypes.byref(cfg), _p(x), _p(src_slot), _p(offsets),
                                      _p(W1), _p(W3), _p(W2), _p(Ws1), _p(Ws3), _p(Ws2),
                                      _p(Y_perm), _p(Y_shared), _p(ws), ws.numel(), _stream()),
          "moe_expert_ffn_gather")
    return Y_perm, Y_shared, ws


def moe_expert_ffn_slots(cfg: MoeConfig, x_perm, x, src_slot, offsets, kept, gates, W1, W3, W2,
                         Ws1=None, Ws3=None, Ws2=None, ws=None, Y_slot=None, Y_shared=None):
    """moe_expert_ffn with the combine's gate in GEMM2's epilogue: Y_slot
    [T k, d], row t k + j = gates[t, j] * FFN(x_t) for kept slots (others not
    written).  x_perm None: rows gathered from x through src_slot."""
    dev = _dev(src_slot)
    if Y_slot is None:
        Y_slot = torch.empty((cfg.T * cfg.k, cfg.d), dtype=_tdtype(cfg), device=dev)
    if cfg.n_shared > 0 and Y_shared is None:
        Y_shared = torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=dev)
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_expert_ffn_slots(ctypes.byref(cfg), _p(x_perm), _p(x), _p(src_slot),
                                     _p(offsets), _p(kept), _p(gates), _p(W1), _p(W3), _p(W2),
                                     _p(Ws1), _p(Ws3), _p(Ws2), _p(Y_slot), _p(Y_shared), _p(ws),
                                     ws.numel(), _stream()), "moe_expert_ffn_slots")
    return Y_slot, Y_shared, ws


def moe_combine_slots(cfg: MoeConfig, Y_slot, Y_shared, keep, residual=None, y=None):
    """y[t] = sum of the kept rows t k + j of Y_slot (+ Y_shared[t])
    (+ residual[t]), fp32 in slot order."""
    if y is None:
        y = torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=_dev(Y_slot))
    check(lib().moe_combine_slots(ctypes.byref(cfg), _p(Y_slot), _p(Y_shared), _p(keep),
                                  _p(residual), _p(y), _stream()), "moe_combine_slots")
    return y


def moe_expert_ffn(cfg: MoeConfig, x_perm, offsets, W1, W3, W2, x=None, Ws1=None, Ws3=None,
                   Ws2=None, ws=None, Y_perm=None, Y_shared=None):
    dev = _dev(x_perm)
    if Y_perm is None:
        Y_perm = torch.empty((moe_perm_rows(cfg), cfg.d), dtype=_tdtype(cfg), device=dev)
    if cfg.n_shared > 0 and Y_shared is None:
        Y_shared = torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=dev)
    if ws is None:
        ws = workspace(moe_stage_workspace_size(cfg), dev)
    check(lib().moe_expert_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(W1), _p(W3),
                               _p(W2), _p(x), _p(Ws1), _p(Ws3), _p(Ws2), _p(Y_perm),
                               _p(Y_shared), _p(ws), ws.numel(), _stream()), "moe_expert_ffn")
    return Y_perm, Y_shared, ws


def moe_combine(cfg: MoeConfig, Y_perm, Y_shared, gates, topk, pos, keep, offsets,
                residual=None, y=None):
    if y is None:
        y = torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=_dev(Y_perm))
    check(lib().moe_combine(ctypes.byref(cfg), _p(Y_perm), _p(Y_shared), _p(gates), _p(topk),
                            _p(pos), _p(keep), _p(offsets), _p(residual), _p(y), _stream()),
          "moe_combine")
    return y


def moe_losses(cfg: MoeConfig, counts, partials):
    dev = _dev(counts)
    aux = torch.empty((1,), dtype=torch.float32, device=dev)
    zl = torch.empty((1,), dtype=torch.float32, device=dev)
    check(lib().moe_losses(ctypes.byref(cfg), _p(counts), _p(partials), _p(aux), _p(zl),
                           _stream()), "moe_losses")
    return aux, zl


def moe_device_status(ws) -> int:
    st = ctypes.c_int32()
    check(lib().moe_device_status(_p(ws), ctypes.byref(st), _stream()), "moe_device_status")
    return int(st.value)


def moe_clear_device_status(ws):
    check(lib().moe_clear_device_status(_p(ws), _stream()), "moe_clear_device_status")


def moe_probe_wait_timeout(ws, timeout_ns: int):
    """Diagnostic: one bounded wait that must run out and set the status word."""
    check(lib().moe_probe_wait_timeout(_p(ws), int(timeout_ns), _stream()),
          "moe_probe_wait_timeout")


def weights_struct(W_r, W1, W2, W3=None, logit_bias=None, select_bias=None, Ws1=None, Ws3=None,
                   Ws2=None) -> MoeWeights:
    def v(t):
        return None if t is None else _p(t).value
    return MoeWeights(W_r=v(W_r), logit_bias=v(logit_bias), select_bias=v(select_bias),
                      W1=v(W1), W3=v(W3), W2=v(W2), Ws1=v(Ws1), Ws3=v(Ws3), Ws2=v(Ws2))


class MoEForward:
    """Reusable forward of one layer: owns the workspace and the outputs, so
    repeated calls allocate nothing (the benchmark and CUDA-graph friendly
    form of moe_forward)."""

    def __init__(self, cfg: MoeConfig, device, keep_routing: bool = True):
        self.cfg = cfg
        moe_validate(cfg)
        dev = torch.device(device)
        T, k, E = cfg.T, cfg.k, cfg.E
        self.ws = workspace(moe_workspace_size(cfg), dev)
        self.y = torch.empty((T, cfg.d), dtype=_tdtype(cfg), device=dev)
        self.aux = torch.empty((1,), dtype=torch.float32, device=dev)
        self.zloss = torch.empty((1,), dtype=torch.float32, device=dev)
        self.topk = self.gates = self.keep = self.dropped = self.counts = self.n_dropped = None
        if keep_routing:
            self.topk = torch.empty((T, k), dtype=torch.int32, device=dev)
            self.gates = torch.empty((T, k), dtype=torch.float32, device=dev)
            self.keep = torch.empty((T, k), dtype=torch.uint8, device=dev)
            self.dropped = torch.empty((T,), dtype=torch.uint8, device=dev)
            self.counts = torch.empty((E,), dtype=torch.int32, device=dev)
            self.n_dropped = torch.empty((1,), dtype=torch.int32, device=dev)

        def v(t):
            return None if t is None else t.data_ptr()
        self._out = MoeOutputs(y=v(self.y), topk_idx=v(self.topk), gates=v(self.gates),
                               keep=v(self.keep), dropped=v(self.dropped),
                               counts=v(self.counts), n_dropped=v(self.n_dropped),
                               aux=v(self.aux), zloss=v(self.zloss))

    def __call__(self, x, weights: MoeWeights):
        check(lib().moe_forward(ctypes.byref(self.cfg), ctypes.byref(weights), _p(x),
                                ctypes.byref(self._out), _p(self.ws), self.ws.numel(), _stream()),
              "moe_forward")
        return self.y


class HostStream:
    """Runs the layer over batches that live in pinned host memory, the way a
    server feeds it: batch i + 1's copy to the device and batch i - 1's copy
    back overlap batch i's kernels.  `depth` device slots (input buffer, layer
    state, output) rotate; copies in run on one side stream, copies out on
    another, the layer (moe_forward) on the caller's current stream, ordered by
    events only.  This class orders copies; it computes nothing itself."""

    def __init__(self, cfg: MoeConfig, device, weights: MoeWeights, depth: int = 2):
        dev = torch.device(device)
        self.weights = weights
        self.depth = depth
        self.fwd = [MoEForward(cfg, dev, keep_routing=False) for _ in range(depth)]
        self.x_dev = [torch.empty((cfg.T, cfg.d), dtype=_tdtype(cfg), device=dev)
                      for _ in range(depth)]
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]
        self.ev_in, self.ev_done, self.ev_out = ev(), ev(), ev()
        self.n = 0

    def start_after(self, event):
        """Make the next copies wait for `event` (e.g. the start of a timed region)."""
        self.s_in.wait_event(event)
        self.s_out.wait_event(event)

    def submit(self, x_host, y_host, loss_host=None):
        """Queue one batch: x_host [T, d] pinned in, y_host [T, d] (and loss_host
        [2] = aux, z) pinned out.  Returns the event after which the outputs
        hold this batch's results."""
        slot = self.n % self.depth
        comp = torch.cuda.current_stream()
        fwd = self.fwd[slot]
        with torch.cuda.stream(self.s_in):
            self.s_in.wait_event(self.ev_done[slot])     # slot's input no longer read
            self.x_dev[slot].copy_(x_host, non_blocking=True)
            self.ev_in[slot].record(self.s_in)
        comp.wait_event(self.ev_in[slot])
        comp.wait_event(self.ev_out[slot])                # slot's output already copied out
        fwd(self.x_dev[slot], self.weights)
        self.ev_done[slot].record(comp)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.ev_done[slot])
            y_host.copy_(fwd.y, non_blocking=True)
            if loss_host is not None:
                loss_host[0:1].copy_(fwd.aux, non_blocking=True)
                loss_host[1:2].copy_(fwd.zloss, non_blocking=True)
            self.ev_out[slot].record(self.s_out)
        self.n += 1
        return self.ev_out[slot]

    def drain(self):
        """Make the current stream wait until every queued batch is copied out."""
        comp = torch.cuda.current_stream()
        for e in self.ev_out:
            comp.wait_event(e)


def moe_forward(cfg: MoeConfig, x, W_r, W1, W2, W3=None, logit_bias=None, select_bias=None,
                Ws1=None, Ws3=None, Ws2=None):
    """One-shot forward: returns (y, aux, zloss, MoEForward state with routing)."""
    fwd = MoEForward(cfg, x.device)
    w = weights_struct(W_r, W1, W2, W3, logit_bias, select_bias, Ws1, Ws3, Ws2)
    fwd(x, w)
    return fwd.y, fwd.aux, fwd.zloss, fwd


__all__ = ["moe_config", "moe_validate", "moe_capacity_value", "moe_perm_rows",
           "moe_capacity_noalloc",
           "moe_loss_partials_count", "moe_stage_workspace_size", "moe_workspace_size",
           "workspace", "moe_route", "moe_capacity", "moe_dispatch", "moe_expert_ffn",
           "moe_combine", "moe_losses", "moe_device_status", "weights_struct", "MoEForward",
           "HostStream", "moe_forward", "CapacityOut", "StagedForward", "moe_capacity_scored",
           "moe_seq_balance_loss", "moe_bias_update", "moe_clear_device_status",
           "moe_probe_wait_timeout", "moe_dispatch_rows", "moe_expert_ffn_gather",
           "moe_expert_ffn_slots", "moe_combine_slots",
           "moe_capacity_sharded", "gather_shard_counts", "shard_losses"]


class StagedForward:
    """The forward as its stage calls on preallocated buffers: the kernels
    moe_forward runs, except that the losses are a launch of their own (the
    forward computes them in the capacity launch, with the same bits);
    `events`, when given, are seven CUDA events recorded before, between and
    after the stages so each stage's device time can be read (route, capacity,
    dispatch, expert_ffn, combine, losses).  A top-1 layer without shared
    experts has its combine in the expert GEMM (the combine stage is empty)."""

    STAGES = ("route", "capacity", "dispatch", "expert_ffn", "combine", "losses")

    def __init__(self, cfg: MoeConfig, device):
        moe_validate(cfg)
        self.cfg = cfg
        dev = torch.device(device)
        T, k, E, d = cfg.T, cfg.k, cfg.E, cfg.d
        dt = _tdtype(cfg)
        R = moe_perm_rows(cfg)
        e = lambda shape, t: torch.empty(shape, dtype=t, device=dev)
        self.topk, self.gates = e((T, k), torch.int32), e((T, k), torch.float32)
        self.partials = e((max(moe_loss_partials_count(cfg), 1),), torch.float32)
        self.counts, self.kept = e((E,), torch.int32), e((E,), torch.int32)
        self.offsets, self.n_dropped = e((E + 1,), torch.int32), e((1,), torch.int32)
        self.pos, self.keep = e((T, k), torch.int32), e((T, k), torch.uint8)
        self.dropped = e((T,), torch.uint8)
        self.x_perm, self.Y_perm = e((R, d), dt), e((R, d), dt)
        self.Y_sh = e((T, d), dt) if cfg.n_shared > 0 else None
        self.y = e((T, d), dt)
        self.aux, self.zloss = e((1,), torch.float32), e((1,), torch.float32)
        # batch-prioritized capacity ranks by the router scores [T, E]
        self.scores = e((T, E), torch.float32) if cfg.priority == 2 else None
        self.ws = workspace(moe_stage_workspace_size(cfg), dev)
        # one slot per token and no shared expert: the combine's gate runs in the
        # expert GEMM, which writes y (as moe_forward does)
        self.fused_combine = cfg.k == 1 and cfg.n_shared == 0
        self.slot = e((R,), torch.int32) if self.fused_combine else None

    def __call__(self, x, W_r, W1, W2, W3=None, logit_bias=None, select_bias=None, Ws1=None,
                 Ws3=None, Ws2=None, events=None):
        L, c, s = lib(), ctypes.byref(self.cfg), _stream()
        rec = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        rec(0)
        check(L.moe_route(c, _p(x), _p(W_r), _p(logit_bias), _p(select_bias), _p(self.topk),
                          _p(self.gates), _p(self.partials), None, _p(self.scores), _p(self.ws),
                          self.ws.numel(), s), "moe_route")
        rec(1)
        if self.scores is not None:
            check(L.moe_capacity_scored(c, _p(self.topk), _p(self.scores), _p(self.counts),
                                        _p(self.pos), _p(self.keep), _p(self.kept),
                                        _p(self.offsets), _p(self.dropped), _p(self.n_dropped),
                                        _p(self.ws), self.ws.numel(), s), "moe_capacity_scored")
        else:
            check(L.moe_capacity(c, _p(self.topk), _p(self.counts), _p(self.pos), _p(self.keep),
                                 _p(self.kept), _p(self.offsets), _p(self.dropped),
                                 _p(self.n_dropped), _p(self.ws), self.ws.numel(), s),
                  "moe_capacity")
        rec(2)
        fused = self.fused_combine
        check(L.moe_dispatch(c, _p(x), _p(self.topk), _p(self.pos), _p(self.keep),
                             _p(self.offsets), _p(self.x_perm), _p(self.slot),
                             _p(self.y) if fused else None, s), "moe_dispatch")
        rec(3)
        if fused:
            check(L.moe_expert_ffn_slots(c, _p(self.x_perm), _p(x), _p(self.slot),
                                         _p(self.offsets), _p(self.kept), _p(self.gates), _p(W1),
                                         _p(W3), _p(W2), None, None, None, _p(self.y), None,
                                         _p(self.ws), self.ws.numel(), s), "moe_expert_ffn_slots")
        else:
            check(L.moe_expert_ffn(c, _p(self.x_perm), _p(self.offsets), _p(W1), _p(W3), _p(W2),
                                   _p(x), _p(Ws1), _p(Ws3), _p(Ws2), _p(self.Y_perm),
                                   _p(self.Y_sh), _p(self.ws), self.ws.numel(), s),
                  "moe_expert_ffn")
        rec(4)
        if not fused:   # (fused: the combine ran in the expert GEMM)
            check(L.moe_combine(c, _p(self.Y_perm), _p(self.Y_sh), _p(self.gates), _p(self.topk),
                                _p(self.pos), _p(self.keep), _p(self.offsets), None, _p(self.y),
                                s), "moe_combine")
        rec(5)
        check(L.moe_losses(c, _p(self.counts), _p(self.partials), _p(self.aux), _p(self.zloss),
                           s), "moe_losses")
        rec(6)
        return self.y
