"""Seeded synthetic inputs for the token-choice MoE forward pass.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no router, no top-k, no capacity, no FFN), so that both
the CUDA library's tests and the CPU oracle can take their inputs from it
without sharing any computation.

Workloads are shaped like the layers the pages discuss ("Lab 18 - Mixture of
experts", section 1 parameter table and DeepSeek-V3 note; cs336 lecture 4,
"DeepSeek v1 -> V2 -> V3"):

  tiny         T=64    d=32   E=4   F=64    k=2 GELU    fp32  cf=1.25
  switch       T=4096  d=1024 E=8   F=4096  k=1 GELU    bf16  cf=1.0, Zipf-skewed router
  mixtral      T=8192  d=4096 E=8   F=14336 k=2 SwiGLU  bf16  cf=1.25
  deepseekmoe  T=16384 d=1024 E=64  F=512   k=6 SwiGLU  bf16  cf=1.5, 2 shared (Fs=512)
  deepseek_v3  T=4096  d=7168 E=256 F=2048  k=8 SwiGLU  bf16  no capacity, sigmoid
               scores + selection bias U(-0.1, 0.1), 1 shared (Fs=2048)

Every tensor is drawn from a torch.Generator seeded with 54000 + the config's
index, on the device asked for, in a fixed order.  Near-tie filtering needs the
router's arithmetic and therefore lives with the tests, which use
``resample_rows`` to redraw the rows they reject.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

ACT_GELU, ACT_SWIGLU = 0, 1
SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1
PRIORITY_TOKEN, PRIORITY_RANK, PRIORITY_SCORE = 0, 1, 2


@dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    d: int
    E: int
    k: int
    d_ff: int
    act: int
    dtype: int
    cf: float
    n_shared: int = 0
    d_ff_shared: int = 0
    score: int = SCORE_SOFTMAX
    renorm: int = -1            # -1: renormalize exactly when k > 1
    priority: int = PRIORITY_TOKEN
    router_std: float | None = None   # None: 1/sqrt(d)
    zipf_s: float = 0.0               # > 0: per-expert logit offsets -s*ln(rank)
    select_bias: float = 0.0          # > 0: selection bias ~ U(-v, v)
    seed_index: int = 0
    variant: str = "default"


CONFIGS: dict[str, MoEShape] = {
    "tiny": MoEShape("tiny", T=64, d=32, E=4, k=2, d_ff=64, act=ACT_GELU, dtype=DTYPE_F32,
                     cf=1.25, router_std=0.02, seed_index=0),
    "switch": MoEShape("switch", T=4096, d=1024, E=8, k=1, d_ff=4096, act=ACT_GELU,
                       dtype=DTYPE_BF16, cf=1.0, router_std=0.02, zipf_s=1.1, seed_index=1),
    "mixtral": MoEShape("mixtral", T=8192, d=4096, E=8, k=2, d_ff=14336, act=ACT_SWIGLU,
                        dtype=DTYPE_BF16, cf=1.25, seed_index=2),
    "deepseekmoe": MoEShape("deepseekmoe", T=16384, d=1024, E=64, k=6, d_ff=512,
                            act=ACT_SWIGLU, dtype=DTYPE_BF16, cf=1.5, n_shared=2,
                            d_ff_shared=512, router_std=0.02, seed_index=3),
    "deepseek_v3": MoEShape("deepseek_v3", T=4096, d=7168, E=256, k=8, d_ff=2048,
                            act=ACT_SWIGLU, dtype=DTYPE_BF16, cf=math.inf, n_shared=1,
                            d_ff_shared=2048, score=SCORE_SIGMOID, select_bias=0.1,
                            seed_index=4),
}
CONFIG_ORDER = ["tiny", "switch", "mixtral", "deepseekmoe", "deepseek_v3"]


def mixtral_variant(kind: str) -> MoEShape:
    """The Mixtral-shaped layer run with balanced prescribed logits or with a
    Zipf-skewed router."""
    base = CONFIGS["mixtral"]
    if kind == "balanced":
        return replace(base, variant="balanced")
    if kind == "skewed":
        return replace(base, variant="skewed", zipf_s=1.1)
    return base


def shrink(shape: MoEShape, **kw) -> MoEShape:
    """Same layer family at other sizes (for parity cases the oracle finishes
    quickly)."""
    return replace(shape, **kw)


@dataclass
class Inputs:
    shape: MoEShape
    x: torch.Tensor                 # [T, d]  fp32 or bf16
    W_r: torch.Tensor               # [d, E]  fp32
    logit_bias: torch.Tensor | None  # [E] fp32
    select_bias: torch.Tensor | None  # [E] fp32
    W1: torch.Tensor                # [E, F, d]
    W3: torch.Tensor | None         # [E, F, d] (SwiGLU)
    W2: torch.Tensor                # [E, d, F]
    Ws1: torch.Tensor | None = None  # [S, Fs, d]
    Ws3: torch.Tensor | None = None
    Ws2: torch.Tensor | None = None  # [S, d, Fs]
    seed: int = 0
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "Inputs":
        def mv(t):
            return None if t is None else t.to(device)
        return Inputs(self.shape, mv(self.x), mv(self.W_r), mv(self.logit_bias),
                      mv(self.select_bias), mv(self.W1), mv(self.W3), mv(self.W2),
                      mv(self.Ws1), mv(self.Ws3), mv(self.Ws2), self.seed, dict(self.extra))


def torch_dtype(code: int):
    return torch.float32 if code == DTYPE_F32 else torch.bfloat16


def _normal(shape, std, dtype, gen, device, chunk_dim0=True):
    """N(0, std^2) drawn in fp32, scaled, then rounded to dtype; drawn slice by
    slice along dim 0 so the fp32 temporary stays small."""
    out = torch.empty(shape, dtype=dtype, device=device)
    if len(shape) == 3 and chunk_dim0:
        for i in range(shape[0]):
            out[i].copy_(torch.randn(shape[1:], generator=gen, device=device,
                                     dtype=torch.float32).mul_(std))
    else:
        out.copy_(torch.randn(shape, generator=gen, device=device, dtype=torch.float32).mul_(std))
    return out


def seed_for(shape: MoEShape) -> int:
    return 54000 + shape.seed_index


def generate(shape: MoEShape, device="cpu", seed: int | None = None) -> Inputs:
    """Draw one layer's inputs and weights.

    x ~ N(0, 1); router W_r ~ N(0, router_std^2) (default 1/d); expert weights
    ~ N(0, 1/fan_in) (fan_in = d for W1/W3, F for W2; tiny uses exactly this);
    Zipf offsets -s*ln(rank_e) with rank a seeded permutation of 1..E;
    selection bias ~ U(-v, v).
    """
    device = torch.device(device)
    seed = seed_for(shape) if seed is None else seed
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = torch_dtype(shape.dtype)
    T, d, E, F = shape.T, shape.d, shape.E, shape.d_ff
    x = _normal((T, d), 1.0, dt, g, device)
    rstd = shape.router_std if shape.router_std is not None else 1.0 / math.sqrt(d)
    W_r = _normal((d, E), rstd, torch.float32, g, device)
    logit_bias = None
    if shape.zipf_s > 0:
        rank = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
        logit_bias = (-shape.zipf_s * torch.log(rank)).to(torch.float32)
    select_bias = None
    if shape.score == SCORE_SIGMOID and shape.select_bias > 0:
        u = torch.rand((E,), generator=g, device=device, dtype=torch.float32)
        select_bias = (u * 2.0 - 1.0) * shape.select_bias
    W1 = _normal((E, F, d), 1.0 / math.sqrt(d), dt, g, device)
    W3 = _normal((E, F, d), 1.0 / math.sqrt(d), dt, g, device) if shape.act == ACT_SWIGLU else None
    W2 = _normal((E, d, F), 1.0 / math.sqrt(F), dt, g, device)
    Ws1 = Ws3 = Ws2 = None
    if shape.n_shared > 0:
        S, Fs = shape.n_shared, shape.d_ff_shared
        Ws1 = _normal((S, Fs, d), 1.0 / math.sqrt(d), dt, g, device)
        if shape.act == ACT_SWIGLU:
            Ws3 = _normal((S, Fs, d), 1.0 / math.sqrt(d), dt, g, device)
        Ws2 = _normal((S, d, Fs), 1.0 / math.sqrt(Fs), dt, g, device)
    inp = Inputs(shape, x, W_r, logit_bias, select_bias, W1, W3, W2, Ws1, Ws3, Ws2, seed)
    if shape.variant == "balanced":
        inp.x = balanced_tokens(shape, W_r, g, device)
    return inp


def balanced_assignment(T: int, E: int):
    """Prescribed top-2 of token t: a = t mod E, b = (a + 1 + (t // E) mod (E - 1)) mod E.
    Every block of E consecutive tokens gives each expert one first and one
    second choice, so each expert receives exactly 2T/E assignments."""
    t = torch.arange(T)
    a = t % E
    b = (a + 1 + (t // E) % (E - 1)) % E
    return a, b


def balanced_tokens(shape: MoEShape, W_r: torch.Tensor, g, device) -> torch.Tensor:
    """Rows x_t whose router logits are prescribed: 2 for the first choice, 1 for
    the second, -1 + N(0, 0.1^2) elsewhere.  x_t is the least-norm solution of
    W_r^T x = z* plus N(0, 1) noise projected off the column space of W_r."""
    T, d, E = shape.T, shape.d, shape.E
    a, b = balanced_assignment(T, E)
    zt = -1.0 + 0.1 * torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    zt = zt.to(torch.float64)
    rows = torch.arange(T, device=device)
    zt[rows, a.to(device)] = 2.0
    zt[rows, b.to(device)] = 1.0
    W = W_r.to(torch.float64)
    G_inv = torch.linalg.inv(W.T @ W)
    noise = torch.randn((T, d), generator=g, device=device, dtype=torch.float32).to(torch.float64)
    noise = noise - (noise @ W) @ G_inv @ W.T
    x = zt @ G_inv @ W.T + noise
    return x.to(torch_dtype(shape.dtype))


def resample_rows(inp: Inputs, rows, attempt: int) -> None:
    """Redraw x rows (in place) from a generator seeded by (seed, attempt)."""
    rows = torch.as_tensor(rows, dtype=torch.long)
    if rows.numel() == 0:
        return
    dev = inp.x.device
    g = torch.Generator(device=dev)
    g.manual_seed(inp.seed * 1000 + 7919 * (attempt + 1))
    fresh = torch.randn((rows.numel(), inp.shape.d), generator=g, device=dev, dtype=torch.float32)
    inp.x[rows.to(dev)] = fresh.to(inp.x.dtype)


__all__ = ["MoEShape", "CONFIGS", "CONFIG_ORDER", "Inputs", "generate", "mixtral_variant",
           "shrink", "resample_rows", "balanced_assignment", "seed_for", "torch_dtype",
           "ACT_GELU", "ACT_SWIGLU", "SCORE_SOFTMAX", "SCORE_SIGMOID", "DTYPE_F32",
           "DTYPE_BF16", "PRIORITY_TOKEN", "PRIORITY_RANK", "PRIORITY_SCORE"]
