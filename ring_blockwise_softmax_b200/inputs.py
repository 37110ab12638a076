"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention or merge arithmetic.  Both the CUDA path's tests/bench and the CPU
oracle consume what it produces, so the two sides always see identical values.

Draws are made on the host with a seeded ``torch.Generator`` (one independent
stream per tensor) in fp32 and then rounded to the workload's dtype
(round-to-nearest-even for bf16).  The oracle widens those exact values to fp64.

The five workloads follow the shapes and value distributions of the pages'
problems: a small fp32 check, a causal bf16 ring with contiguous shards, a long
causal striped ring, a wide-logit non-causal stress case with a 16-way merge,
and the tabular row-axis layout of intelliparadigm.com "Mosaic多轴注意力分片"
§2.2/§3.1 (a [batch, rows, features, embed] tensor, 4 heads of 24 dims,
attention over the rows axis for each feature).  No dataset is involved.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    H: int
    N: int
    d: int
    causal: bool
    P: int
    layout: str  # "contiguous" | "striped"
    qk_sigma: float = 1.0
    v_dist: str = "normal"  # "normal" (sigma 1) | "uniform" (U(-1, 1))
    tabular: tuple | None = None  # (batch, rows, features, embed, heads) for the row-axis layout
    H_kv: int | None = None  # K/V heads (grouped-query attention); None = H
    window: int | None = None  # causal sliding window (positions); None = none

    @property
    def seed(self) -> int:
        return 1000 + self.cfg

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """Algorithmic forward FLOPs: 4*B*H*N^2*d, halved when causal; with a sliding window of w
        positions, 4*B*H*d per visible pair, sum_i min(i + 1, w) pairs per head."""
        if self.window is not None:
            w, n = self.window, self.N
            pairs = w * (w + 1) / 2 + (n - w) * w if w < n else n * (n + 1) / 2
            return 4.0 * self.B * self.H * self.d * pairs
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


WORKLOADS = {
    1: Workload(1, "fp32 non-causal B=1 H=2 N=256 d=64, ring P=4 contiguous", "f32", 1, 2, 256, 64, False, 4,
                "contiguous"),
    2: Workload(2, "bf16 causal B=2 H=16 N=8192 d=64, ring P=8 contiguous", "bf16", 2, 16, 8192, 64, True, 8,
                "contiguous"),
    3: Workload(3, "bf16 causal B=1 H=32 N=32768 d=128, ring P=8 striped", "bf16", 1, 32, 32768, 128, True, 8,
                "striped"),
    4: Workload(4, "bf16 non-causal B=1 H=8 N=16384 d=128, Q,K~N(0,4), V~U(-1,1), ring P=16 contiguous", "bf16",
                1, 8, 16384, 128, False, 16, "contiguous", qk_sigma=2.0, v_dist="uniform"),
    5: Workload(5, "bf16 tabular [1,150000,8,96], 4 heads x d=24, row-axis attention, ring P=8 contiguous",
                "bf16", 1, 32, 150000, 24, False, 8, "contiguous", tabular=(1, 150000, 8, 96, 4)),
}


def _gen(seed: int, sub: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 16 + sub)
    return g


def _torch_dtype(dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def draw(shape, seed: int, sub: int, dist: str = "normal", sigma: float = 1.0, dtype: str = "bf16"):
    """One seeded tensor on the host: N(0, sigma^2) or U(-1, 1), rounded to ``dtype``."""
    g = _gen(seed, sub)
    if dist == "normal":
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if sigma != 1.0:
            x.mul_(sigma)
    elif dist == "uniform":
        x = torch.rand(shape, generator=g, dtype=torch.float32).mul_(2.0).sub_(1.0)
    else:
        raise ValueError(dist)
    return x.to(_torch_dtype(dtype))


def make_qkv(w: Workload, seed: int | None = None, N: int | None = None):
    """Q, K, V as [B, H, N, d] host tensors (views of one storage each).

    For the tabular workload each of Q, K, V is a [batch, rows, features, embed]
    tensor; head h of feature f is the slice embed[h*24:(h+1)*24] and the
    attention axis is rows, so the [B, H, N, d] view has H = features*heads,
    stride(H) = 24, stride(N) = features*embed.  ``N`` overrides the sequence
    length (the same layout at a smaller size, for tests).
    """
    seed = w.seed if seed is None else seed
    n = w.N if N is None else N
    if w.tabular is not None:
        batch, _, feats, embed, heads = w.tabular
        hd = embed // heads
        out = []
        for sub in range(3):
            dist = w.v_dist if sub == 2 else "normal"
            sigma = 1.0 if sub == 2 else w.qk_sigma
            t = draw((batch, n, feats, embed), seed, sub, dist, sigma, w.dtype)
            out.append(t.as_strided((batch, feats * heads, n, hd),
                                    (n * feats * embed, hd, feats * embed, 1)))
        return tuple(out)
    shape = (w.B, w.H, n, w.d)
    kv_shape = (w.B, w.H if w.H_kv is None else w.H_kv, n, w.d)
    q = draw(shape, seed, 0, "normal", w.qk_sigma, w.dtype)
    k = draw(kv_shape, seed, 1, "normal", w.qk_sigma, w.dtype)
    v = draw(kv_shape, seed, 2, w.v_dist, 1.0, w.dtype)
    return q, k, v


def make_small(B, H, N, d, dtype="bf16", seed=0, qk_sigma=1.0, v_dist="normal", Nk=None):
    """A [B, H, N, d] problem of arbitrary size (tests); Nk sets a different key count."""
    nk = N if Nk is None else Nk
    q = draw((B, H, N, d), seed, 0, "normal", qk_sigma, dtype)
    k = draw((B, H, nk, d), seed, 1, "normal", qk_sigma, dtype)
    v = draw((B, H, nk, d), seed, 2, v_dist, 1.0, dtype)
    return q, k, v


def make_merge_inputs(k: int, rows: int, d: int, seed: int = 1104, empty_frac: float = 0.0):
    """k fp32 partial outputs [k, rows, d] ~ U(-1, 1) and partial LSEs [k, rows] ~ 7 + N(0, 4).

    ``empty_frac`` of the (partial, row) entries are empty partials: O = 0, LSE = -inf.
    """
    o = draw((k, rows, d), seed, 0, "uniform", 1.0, "f32")
    lse = draw((k, rows), seed, 1, "normal", 2.0, "f32").add_(7.0)
    if empty_frac > 0:
        u = torch.rand((k, rows), generator=_gen(seed, 2))
        empty = u < empty_frac
        lse[empty] = float("-inf")
        o[empty] = 0.0
    return o, lse
