"""Seeded synthetic workloads for the Monarch attention forward.

This module holds the five workload shapes and the seeded input recipes.  It
contains none of the operator's arithmetic: it only draws random tensors, so
both the CUDA path (tests, bench) and the fp64 oracle's tests can use it.

The pages (MonarchRT: Efficient Attention for Real-Time Video Generation,
gist.science/zh/paper/2602.12271, section 4 "Results") measure kernel latency
at 720p and end-to-end generation with Self-Forcing at 480p but print no
tensor shapes; these synthetic shapes stand in for those workloads:
a Wan-style latent grid of 30x52 (480p) or 45x80 (720p) tokens per frame,
21 latent frames per clip, 12 heads of width 128.

Recipe (every draw on a CPU ``torch.Generator`` seeded with the workload's
index, fp32 draws in the order Q, K, V, then extras, then cast):
  0 tiny_fp32     Q, K, V iid N(0,1) * d^-1/2, kept fp32.
  1 chunk_bf16    Q, K, V iid N(0,1).
  2 fullclip_bf16 Q, K, V iid N(0,1); then R (8 x d) iid N(0,1) and the
                  shared positional term 0.5 * u(n) R added to Q and K, where
                  u(n) = [cos 2pi t/T, sin 2pi t/T, cos 2pi h/H, sin 2pi h/H,
                  cos 2pi w/W, sin 2pi w/W, cos 2pi(h/H+w/W), sin 2pi(h/H+w/W)]
                  (periodic and separable, like the positional part of the
                  attention map the pages describe; unit variance per entry).
  3 tiled_bf16    Q, K, V iid N(0,1).
  4 large_bf16    Q, K, V iid N(0,1); then randperm(N)[:5% of N] picks key
                  rows that are multiplied by 4 in every batch and head
                  (a stand-in for the sparse semantic outliers).
  5 chunk_ar_bf16 the last chunk of a 21-frame clip generated
                  autoregressively: Q, K, V of the 3 new frames iid N(0,1);
                  the 18 context frames' keys and stage-1 outputs iid N(0,1),
                  drawn by generate_context from a generator seeded
                  1000 + index.
  6 fullclip_row_bf16  the full-clip grid under the (f*h, w) split; Q, K, V
                  iid N(0,1).
  7 bwd_chunk_f32 gradients on the chunk shape in fp32: Q, K, V iid
                  N(0,1) * d^-1/4 (moderate logits for the exact path); dO the
                  same, drawn by generate_upstream from a generator seeded
                  2000 + index.
  8 bwd_chunk_bf16 gradients on the chunk shape in bf16 (tensor cores):
                  Q, K, V iid N(0,1), as chunk_bf16; dO iid N(0,1), drawn by
                  generate_upstream from a generator seeded 2000 + index.
  9 bwd_fullclip_bf16 gradients on the full-clip grid in bf16: Q, K, V and
                  dO iid N(0,1).
"""
from __future__ import annotations

import dataclasses
import math

import torch

FACT_FRAME = 0
FACT_TILED = 1
FACT_ROW = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    dtype: str  # "f32" or "bf16"
    fact: int = FACT_FRAME
    tile_h: int = 0
    tile_w: int = 0
    extra: str = ""  # "scaled", "positional", "outliers" or ""
    T_ctx: int = 0   # context frames before the chunk (autoregressive chunk workloads)
    grad: bool = False  # gradient workload: dQ, dK, dV for an upstream gradient dO

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def m(self) -> int:
        """Tokens per stage-1 block."""
        if self.fact == FACT_TILED:
            return self.tile_h * self.tile_w
        if self.fact == FACT_ROW:
            return self.W
        return self.H * self.W

    @property
    def N_ctx(self) -> int:
        return self.T_ctx * self.H * self.W

    @property
    def b(self) -> int:
        """Keys per stage-2 group: one spatial position across frames (context
        included), or for the (f*h, w) split one column across frames and rows."""
        if self.fact == FACT_ROW:
            return self.T * self.H
        return self.T + self.T_ctx

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*N*(m+b)*d per (batch, head), no padding; a
        gradient workload counts 10*d per (query, key) pair (S, dP, dQ, dK, dV)."""
        per_pair = 10.0 if self.grad else 4.0
        return per_pair * self.N * (self.m + self.b) * self.d * self.B * self.heads

    @property
    def io_bytes(self) -> int:
        """Minimum HBM bytes: read Q, K, V once, write O once; a chunk also
        reads the context's K and Y1 and writes the new frames' Y1."""
        es = 4 if self.dtype == "f32" else 2
        if self.grad:  # read Q, K, V, dO; write dQ, dK, dV
            return 7 * self.N * self.B * self.heads * self.d * es
        rows = 4 * self.N + (self.N + 2 * self.N_ctx if self.T_ctx else 0)
        return rows * self.B * self.heads * self.d * es

    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = [
    Workload(0, "tiny_fp32", 1, 2, 64, 4, 8, 8, "f32", extra="scaled"),
    Workload(1, "chunk_bf16", 1, 12, 128, 3, 30, 52, "bf16"),
    Workload(2, "fullclip_bf16", 1, 12, 128, 21, 30, 52, "bf16", extra="positional"),
    Workload(3, "tiled_bf16", 1, 12, 128, 21, 30, 52, "bf16", FACT_TILED, 10, 13),
    Workload(4, "large_bf16", 2, 12, 128, 21, 45, 80, "bf16", extra="outliers"),
    Workload(5, "chunk_ar_bf16", 1, 12, 128, 3, 30, 52, "bf16", T_ctx=18),
    Workload(6, "fullclip_row_bf16", 1, 12, 128, 21, 30, 52, "bf16", FACT_ROW),
    Workload(7, "bwd_chunk_f32", 1, 12, 128, 3, 30, 52, "f32", grad=True),
    Workload(8, "bwd_chunk_bf16", 1, 12, 128, 3, 30, 52, "bf16", grad=True),
    Workload(9, "bwd_fullclip_bf16", 1, 12, 128, 21, 30, 52, "bf16", grad=True),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def positional_features(T: int, H: int, W: int) -> torch.Tensor:
    """u(n) for every token n = (t*H + h)*W + w, shape [N, 8] (float64)."""
    t = torch.arange(T, dtype=torch.float64).view(T, 1, 1).expand(T, H, W)
    h = torch.arange(H, dtype=torch.float64).view(1, H, 1).expand(T, H, W)
    w = torch.arange(W, dtype=torch.float64).view(1, 1, W).expand(T, H, W)
    tp = 2 * math.pi
    feats = [torch.cos(tp * t / T), torch.sin(tp * t / T),
             torch.cos(tp * h / H), torch.sin(tp * h / H),
             torch.cos(tp * w / W), torch.sin(tp * w / W),
             torch.cos(tp * (h / H + w / W)), torch.sin(tp * (h / H + w / W))]
    return torch.stack([f.reshape(-1) for f in feats], dim=1)


def generate(wl: Workload, seed: int | None = None, B: int | None = None,
             heads: int | None = None):
    """Seeded (Q, K, V) on the CPU, shape [B, heads, N, d], workload dtype.

    ``B``/``heads`` may be lowered for a bounded sample; the first draws are
    then those of the smaller tensor, so a sample is not a slice of the full
    workload -- both sides of any comparison must use the same call.
    """
    seed = wl.index if seed is None else seed
    B = wl.B if B is None else B
    heads = wl.heads if heads is None else heads
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, heads, wl.N, wl.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if wl.extra == "scaled":
        s = wl.d ** -0.5
        q.mul_(s); k.mul_(s); v.mul_(s)
    elif wl.extra == "positional":
        R = torch.randn((8, wl.d), generator=g, dtype=torch.float32)
        pos = (0.5 * positional_features(wl.T, wl.H, wl.W).float() @ R)  # [N, d]
        q.add_(pos); k.add_(pos)
    elif wl.grad and wl.dtype == "f32":
        s = wl.d ** -0.25
        q.mul_(s); k.mul_(s); v.mul_(s)
    elif wl.extra == "outliers":
        n_out = (wl.N * 5) // 100
        rows = torch.randperm(wl.N, generator=g)[:n_out]
        k[:, :, rows, :] *= 4.0
    dt = wl.torch_dtype()
    return q.to(dt), k.to(dt), v.to(dt)


def random_inputs(B, heads, T, H, W, d, dtype=torch.bfloat16, seed=0, scale=1.0):
    """Seeded iid N(0, scale^2) inputs for ad-hoc shapes (edge-case tests)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, heads, T * H * W, d)
    out = []
    for _ in range(3):
        x = torch.randn(shape, generator=g, dtype=torch.float32) * scale
        out.append(x.to(dtype))
    return tuple(out)


def generate_context(wl: Workload, seed: int | None = None, B: int | None = None,
                     heads: int | None = None):
    """Seeded context (K_ctx, Y1_ctx) of a chunk workload on the CPU, shape
    [B, heads, T_ctx*H*W, d], workload dtype."""
    seed = 1000 + wl.index if seed is None else seed
    B = wl.B if B is None else B
    heads = wl.heads if heads is None else heads
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, heads, wl.N_ctx, wl.d)
    kc = torch.randn(shape, generator=g, dtype=torch.float32)
    yc = torch.randn(shape, generator=g, dtype=torch.float32)
    dt = wl.torch_dtype()
    return kc.to(dt), yc.to(dt)


def generate_upstream(wl: Workload, seed: int | None = None, heads: int | None = None):
    """Seeded upstream gradient dO of a gradient workload, shape [B, heads, N, d]."""
    seed = 2000 + wl.index if seed is None else seed
    heads = wl.heads if heads is None else heads
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    do = torch.randn((wl.B, heads, wl.N, wl.d), generator=g, dtype=torch.float32)
    if wl.dtype == "f32":
        do.mul_(wl.d ** -0.25)
    return do.to(wl.torch_dtype())
