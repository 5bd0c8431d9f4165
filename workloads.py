"""Seeded synthetic inputs for the five attention workloads.

This module only draws random tensors; it holds none of the attention or
thinning arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA library
read the tensors it returns, so the two sides always see identical bf16/fp32
inputs.

Every (batch, head) slice is drawn from its own ``torch.Generator`` seeded
from ``(data_seed, b, h)``, so a single slice can be regenerated without
drawing the whole tensor (the oracle's sampled checks rely on that).

Workloads (shapes from the Thinformer README's stated layouts, "Getting
Started": query (B,T,H,E), key (B,S,H,E), value (B,S,H,D)):

  tiny     B=1  H=1  T=S=256        E=D=64  fp32  q,k,v ~ N(0,1)
  vit      B=64 H=1  T=S=3136       E=D=64  bf16  q,k = E^-1/4 (Z + 0.5 A U^T), v ~ N(0,1)
           (T2T-ViT token-to-token shape: 56x56 patches; A (S,8) per token,
            U (E,8) ~ N(0,1)/sqrt(8) shared by q and k of one (b,h))
  biggan   B=32 H=1  T=4096 S=1024  E=64 D=256 bf16 q,k,v ~ N(0,1)
           (BigGAN self-attention shape: 64x64 map, keys 2x2 max-pooled;
            keys are drawn directly at the pooled size)
  express32k   B=1 H=32 T=32768  E=D=128 bf16 causal; q,k = E^-1/4 N(0,1) then
               RoPE (base 10000, pairs (2i,2i+1), angle t*10000^(-2i/E)); v ~ N(0,1)
  express128k  B=1 H=32 T=131072 E=D=128 bf16 causal; same generator, seed 3
  express32k_a the express32k tensors through the page-literal cache (n_out = 128)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    S: int
    E: int
    D: int
    dtype: str            # "fp32" | "bf16"
    causal: bool
    g: int                # oversampling parameter of KH-Compress
    seed: int             # Philox seed of the thinning decisions
    data_seed: int        # seed of the synthetic tensors
    kind: str             # "iid" | "rank8" | "rope"
    n_exact: int = 0      # Express exact phase (causal only); the cache size n_out for cache "A"
    batch: int = 0        # Express thin batch (causal only, cache "B")
    cache: str = "B"      # causal only: "B" nodes of a 4-ary counter, "A" the page-literal cache

    @property
    def mode(self) -> int:
        """The library's `causal` argument: 0 Thinformer, 1 Express, 2 Express with the page-literal cache."""
        return 0 if not self.causal else (2 if self.cache == "A" else 1)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.E)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, 256, 64, 64, "fp32", False, 2, 1, 0, "iid"),
    "vit": Workload("vit", 64, 1, 3136, 3136, 64, 64, "bf16", False, 2, 2, 1, "rank8"),
    "biggan": Workload("biggan", 32, 1, 4096, 1024, 64, 256, "bf16", False, 3, 3, 2, "iid"),
    "express32k": Workload("express32k", 1, 32, 32768, 32768, 128, 128, "bf16", True, 2, 1, 0,
                           "rope", n_exact=1024, batch=1024),
    "express128k": Workload("express128k", 1, 32, 131072, 131072, 128, 128, "bf16", True, 2, 4, 3,
                            "rope", n_exact=2048, batch=2048),
    "express32k_a": Workload("express32k_a", 1, 32, 32768, 32768, 128, 128, "bf16", True, 2, 1, 0,
                             "rope", n_exact=128, cache="A"),
}


def _gen(data_seed: int, b: int, h: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(((data_seed * 1_000_003 + b) * 1_000_033 + h) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _rope(x: torch.Tensor) -> torch.Tensor:
    """Rotate consecutive pairs (2i, 2i+1) of each row t by t * 10000^(-2i/E)."""
    T, E = x.shape
    i = torch.arange(E // 2, dtype=torch.float64)
    inv = torch.pow(torch.tensor(10000.0, dtype=torch.float64), -2.0 * i / E)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * inv[None, :]
    c, s = torch.cos(ang).float(), torch.sin(ang).float()
    x0, x1 = x[:, 0::2], x[:, 1::2]
    out = torch.empty_like(x)
    out[:, 0::2] = x0 * c - x1 * s
    out[:, 1::2] = x0 * s + x1 * c
    return out


def slice_qkv(w: Workload, b: int, h: int, T: int | None = None, S: int | None = None):
    """Draw q (T,E), k (S,E), v (S,D) of one (b,h) slice, cast to the workload dtype.

    ``T``/``S`` override the workload's lengths (used for reduced test sizes);
    the draw order is fixed so a slice is a pure function of (w, b, h, T, S).
    """
    T = w.T if T is None else T
    S = (T if w.causal else w.S) if S is None else S
    g = _gen(w.data_seed, b, h)
    E, D = w.E, w.D
    if w.kind == "iid":
        q = torch.randn(T, E, generator=g)
        k = torch.randn(S, E, generator=g)
    elif w.kind == "rank8":
        U = torch.randn(E, 8, generator=g) / math.sqrt(8.0)
        q = torch.randn(T, E, generator=g) + 0.5 * torch.randn(T, 8, generator=g) @ U.T
        k = torch.randn(S, E, generator=g) + 0.5 * torch.randn(S, 8, generator=g) @ U.T
        q, k = q * E ** -0.25, k * E ** -0.25
    elif w.kind == "rope":
        q = _rope(torch.randn(T, E, generator=g) * E ** -0.25)
        k = _rope(torch.randn(S, E, generator=g) * E ** -0.25)
    else:
        raise ValueError(w.kind)
    v = torch.randn(S, D, generator=g)
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def make_qkv(w: Workload, T: int | None = None, S: int | None = None,
             heads: Iterable[int] | None = None, b0: int = 0):
    """Full (B,T,H,E), (B,S,H,E), (B,S,H,D) tensors on the CPU.

    ``heads`` restricts to a subset of heads (the H axis then has len(heads)); ``b0`` is the
    index of batch row 0 in a larger problem (rows b0 .. b0+B-1 of it are drawn).
    """
    T = w.T if T is None else T
    S = (T if w.causal else w.S) if S is None else S
    hs = list(range(w.H)) if heads is None else list(heads)
    dt = w.torch_dtype
    q = torch.empty(w.B, T, len(hs), w.E, dtype=dt)
    k = torch.empty(w.B, S, len(hs), w.E, dtype=dt)
    v = torch.empty(w.B, S, len(hs), w.D, dtype=dt)
    for b in range(w.B):
        for j, h in enumerate(hs):
            qs, ks, vs = slice_qkv(w, b0 + b, h, T, S)
            q[b, :, j], k[b, :, j], v[b, :, j] = qs, ks, vs
    return q, k, v
