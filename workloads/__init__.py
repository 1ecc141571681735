"""Seeded synthetic inputs for causal prefill attention.

This module only draws random tensors with the shapes and value structure of
the workloads (Gaussian Q/K/V, per-channel lognormal scales, outlier
channels, rotary position embedding).  It holds none of the attention
method's arithmetic, and both the CUDA path's tests/benchmark and the CPU
oracle read their inputs from here.

Workloads (the pages benchmark Gaussian inputs and captured layers of
Mistral-7B, Qwen3-8B and DeepSeek-V2-Lite; no weights or activations are
available, so layer-shaped synthetic tensors stand in for the captured ones):

  tiny      B=1 Hq=Hkv=2  S=256   d=128      Q,K,V iid N(0,1), seed 0
  gqa       B=1 Hq=32 Hkv=8 S=4096 d=128     Q,K = N(0,1) * lognormal(0,0.5)
                                              channel scale, then RoPE
                                              (theta 1e6); V ~ N(0,1)
  long      B=1 Hq=32 Hkv=8 S=16384 d=128    Q,K = N(0,1), 4 outlier channels
                                              per head x20, then RoPE; V N(0,1)
  long_shared  as long, but the 4 outlier channels of a kv head are shared
                                              by its keys and its query heads,
                                              and Q,K are scaled by
                                              1/sqrt(1 + 4(20^2 - 1)/d) so that
                                              E|q|^2 = d as for N(0,1) rows
  mla       B=1 Hq=Hkv=16 S=16384 dqk=192 dv=128   iid N(0,1)
  gauss     B=1 Hq=Hkv=32 d=128, S in {4K,8K,16K,32K}  iid N(0,1)
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    dqk: int
    dv: int
    dist: str  # "iid", "lognormal_rope", "outlier_rope", "shared_outlier_rope"
    seed: int

    @property
    def Sq(self) -> int:
        return self.S

    @property
    def Sk(self) -> int:
        return self.S

    def causal_flops(self) -> float:
        """2*B*Hq*S^2*(dqk+dv)/2: the causal half of both contractions."""
        return 2.0 * self.B * self.Hq * self.S * self.S * (self.dqk + self.dv) / 2.0

    def with_S(self, S: int) -> "Workload":
        return replace(self, S=S, name="%s_S%d" % (self.name.split("_S")[0], S))


WORKLOADS = {
    "tiny": Workload("tiny", 1, 256, 2, 2, 128, 128, "iid", 0),
    "gqa": Workload("gqa", 1, 4096, 32, 8, 128, 128, "lognormal_rope", 1),
    "long": Workload("long", 1, 16384, 32, 8, 128, 128, "outlier_rope", 2),
    "mla": Workload("mla", 1, 16384, 16, 16, 192, 128, "iid", 3),
    "gauss": Workload("gauss", 1, 32768, 32, 32, 128, 128, "iid", 4),
    "long_shared": Workload("long_shared", 1, 16384, 32, 8, 128, 128, "shared_outlier_rope", 5),
}

GAUSS_SWEEP = (4096, 8192, 16384, 32768)


def get(name: str, S: int | None = None) -> Workload:
    w = WORKLOADS[name]
    return w.with_S(S) if S is not None else w


def _rope(x: torch.Tensor, theta: float) -> torch.Tensor:
    """Rotate-half rotary embedding over positions 0..S-1 (layout B,S,H,d)."""
    B, S, H, d = x.shape
    half = d // 2
    inv = theta ** (-torch.arange(0, half, dtype=torch.float64) * 2.0 / d)
    ang = torch.arange(S, dtype=torch.float64)[:, None] * inv[None, :]
    cos = torch.cos(ang).to(torch.float32)[None, :, None, :]
    sin = torch.sin(ang).to(torch.float32)[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def _qk(g: torch.Generator, B, S, H, d, dist) -> torch.Tensor:
    x = torch.randn((B, S, H, d), generator=g, dtype=torch.float32)
    if dist == "lognormal_rope":
        sc = torch.exp(0.5 * torch.randn((H, d), generator=g, dtype=torch.float32))
        x = _rope(x * sc, 1e6)
    elif dist == "outlier_rope":
        mult = torch.ones((H, d), dtype=torch.float32)
        for h in range(H):
            ch = torch.randperm(d, generator=g)[:4]
            mult[h, ch] = 20.0
        x = _rope(x * mult, 1e6)
    return x


def _shared_outliers(g: torch.Generator, B, S, Hq, Hkv, d, mult=20.0):
    """Q and K with 4 outlier channels per kv head, the same channels for the
    keys of that head and for its query heads, each tensor scaled so that a
    row's expected squared norm stays d; then RoPE (theta 1e6)."""
    m = torch.ones((Hkv, d), dtype=torch.float32)
    for h in range(Hkv):
        m[h, torch.randperm(d, generator=g)[:4]] = mult
    norm = 1.0 / float((1.0 + 4.0 * (mult * mult - 1.0) / d) ** 0.5)
    q = torch.randn((B, S, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, S, Hkv, d), generator=g, dtype=torch.float32)
    q = _rope(q * m.repeat_interleave(Hq // Hkv, dim=0) * norm, 1e6)
    k = _rope(k * m * norm, 1e6)
    return q, k


def make_inputs(w: Workload, seed: int | None = None):
    """Return fp32 CPU tensors q (B,S,Hq,dqk), k (B,S,Hkv,dqk), v (B,S,Hkv,dv)."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    if w.dist == "shared_outlier_rope":
        q, k = _shared_outliers(g, w.B, w.S, w.Hq, w.Hkv, w.dqk)
        v = torch.randn((w.B, w.S, w.Hkv, w.dv), generator=g, dtype=torch.float32)
        return q, k, v
    q = _qk(g, w.B, w.S, w.Hq, w.dqk, w.dist)
    k = _qk(g, w.B, w.S, w.Hkv, w.dqk, w.dist)
    v = torch.randn((w.B, w.S, w.Hkv, w.dv), generator=g, dtype=torch.float32)
    return q, k, v


def make_custom(B, Sq, Sk, Hq, Hkv, dqk, dv, seed=0, std=1.0):
    """iid N(0, std^2) tensors of arbitrary shape (edge-case tests)."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, Sq, Hq, dqk), generator=g) * std
    k = torch.randn((B, Sk, Hkv, dqk), generator=g) * std
    v = torch.randn((B, Sk, Hkv, dv), generator=g)
    return q, k, v


def sample_rows(B: int, Hq: int, Sq: int, every: int = 64):
    """Deterministic row sample for large S: every `every`-th query row of
    every (batch, head), plus the last row; flat ids (b*Hq + h)*Sq + i."""
    rows = []
    for bh in range(B * Hq):
        idx = list(range(0, Sq, every))
        if idx[-1] != Sq - 1:
            idx.append(Sq - 1)
        rows.extend(bh * Sq + i for i in idx)
    return torch.tensor(rows, dtype=torch.int64)
