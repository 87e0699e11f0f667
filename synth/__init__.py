"""Seeded synthetic video-latent Q/K/V for the adaptive block-sparse attention path.

This module only *makes inputs*. It holds none of the method's arithmetic (no
reordering, pooling, scoring, routing or attention) and is the one piece of code
that both the CPU oracle and the CUDA path consume.

Workload recipe (the pages' workload is Wan2.2 I2V latents, which are not
available; these synthetic tensors stand in for them):

* the latent grid is T x Y x X tokens in natural raster order ``n = (t*Y + y)*X + x``;
* per head h, random Fourier features of the integer coordinate p = (t, y, x):
  ``phi_h(p) = [cos(W_h p); sin(W_h p)]`` with ``W_h`` of shape (d/2, 3), entries
  N(0, sigma^2).  Q and K share ``phi_h`` so Q K^T behaves like a Gaussian
  locality kernel over the video grid;
* ``Q = a_h * phi_h + noise_std * eps_Q``, ``K = a_h * phi_h + noise_std * eps_K``,
  ``V ~ N(0, 1)``;
* the per-head scale a_h is fixed, log-uniform in [lo, hi], or alternating
  between two values over even/odd heads (the head-heterogeneity stress case);
* everything is drawn in float32 from ``numpy.random.default_rng(seed)`` in the
  order: H uniforms (for a_h, always drawn), W (H, d/2, 3), then for each batch b
  and head h: eps_Q, eps_K, V (each N x d); then rounded to bfloat16 with
  round-to-nearest-even on the bit pattern.

Tensors come back as ``uint16`` bit patterns of bfloat16, shape [B, H, N, d].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "Config", "CONFIGS", "bf16_bits", "bf16_to_f32", "make_qkv", "head_scales",
]


@dataclasses.dataclass(frozen=True)
class Config:
    """One workload: geometry, routing parameters and generator parameters."""

    name: str
    B: int
    H: int
    d: int
    T: int
    Y: int
    X: int
    tt: int
    ty: int
    tx: int
    p: float
    k: int
    a_mode: str = "loguniform"        # "fixed" | "loguniform" | "alternating"
    a_lo: float = 0.5                  # fixed value, or log-uniform low, or even-head value
    a_hi: float = 4.0                  # log-uniform high, or odd-head value
    noise_std: float = 1.0
    sigma: float = 0.3
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T * self.Y * self.X

    @property
    def S(self) -> int:
        return self.tt * self.ty * self.tx

    @property
    def Nb(self) -> int:
        return self.N // self.S

    def with_(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The workloads.  "tiny" is the small case the oracle finishes in milliseconds;
# "wan480p" / "wan720p" are single Wan-like attention layers; "stress720p" is the
# head-heterogeneity case; the sweep varies p and tile size around wan720p.
CONFIGS = {
    "tiny": Config("tiny", B=1, H=2, d=64, T=4, Y=8, X=8, tt=1, ty=8, tx=8,
                   p=0.9, k=1, a_mode="fixed", a_lo=2.0,
                   noise_std=math.sqrt(0.5), sigma=0.3, seed=0),
    "wan480p": Config("wan480p", B=1, H=40, d=128, T=20, Y=32, X=48, tt=2, ty=8, tx=8,
                      p=0.9, k=4),
    "wan720p": Config("wan720p", B=1, H=40, d=128, T=20, Y=48, X=80, tt=2, ty=8, tx=8,
                      p=0.9, k=4),
    "stress720p": Config("stress720p", B=1, H=40, d=128, T=20, Y=48, X=80, tt=2, ty=8, tx=8,
                         p=0.95, k=4, a_mode="alternating", a_lo=4.0, a_hi=0.3),
}


def sweep_configs() -> list:
    """p in {0.8, 0.9, 0.95, 0.99, 1.0} x tile {1x8x8, 2x8x8} at 720p scale, k=4."""
    out = []
    base = CONFIGS["wan720p"]
    for tile in ((1, 8, 8), (2, 8, 8)):
        for p in (0.8, 0.9, 0.95, 0.99, 1.0):
            out.append(base.with_(name=f"sweep_p{p}_t{tile[0]}x{tile[1]}x{tile[2]}",
                                  p=p, tt=tile[0], ty=tile[1], tx=tile[2]))
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def head_scales(cfg: Config, u: np.ndarray) -> np.ndarray:
    """Per-head a_h from the H uniforms u (always drawn, so the stream stays aligned)."""
    if cfg.a_mode == "fixed":
        return np.full(cfg.H, cfg.a_lo, dtype=np.float64)
    if cfg.a_mode == "loguniform":
        lo, hi = math.log(cfg.a_lo), math.log(cfg.a_hi)
        return np.exp(lo + u.astype(np.float64) * (hi - lo))
    if cfg.a_mode == "alternating":
        return np.where(np.arange(cfg.H) % 2 == 0, cfg.a_lo, cfg.a_hi).astype(np.float64)
    raise ValueError(f"unknown a_mode {cfg.a_mode!r}")


def _coords(cfg: Config) -> np.ndarray:
    t, y, x = np.meshgrid(np.arange(cfg.T), np.arange(cfg.Y), np.arange(cfg.X), indexing="ij")
    return np.stack([t.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.float64)  # [N, 3]


def make_qkv(cfg: Config, heads: Optional[Sequence[int]] = None):
    """Return (q, k, v) as bf16 bit patterns [B, H', N, d] in natural token order.

    ``heads`` selects a subset of heads (the random stream is still consumed for
    every head in order, so head h is identical whether or not others are kept).
    """
    if cfg.d % 2:
        raise ValueError("head_dim must be even")
    rng = np.random.default_rng(cfg.seed)
    u = rng.random(cfg.H)
    a = head_scales(cfg, u)
    W = rng.standard_normal((cfg.H, cfg.d // 2, 3), dtype=np.float32).astype(np.float64) * cfg.sigma
    keep = list(range(cfg.H)) if heads is None else list(heads)
    pos = {h: n for n, h in enumerate(keep)}
    coords = _coords(cfg)
    N, d = cfg.N, cfg.d
    q = np.empty((cfg.B, len(keep), N, d), dtype=np.uint16)
    k = np.empty_like(q)
    v = np.empty_like(q)
    feats = {}
    for b in range(cfg.B):
        for h in range(cfg.H):
            eq = rng.standard_normal((N, d), dtype=np.float32)
            ek = rng.standard_normal((N, d), dtype=np.float32)
            vv = rng.standard_normal((N, d), dtype=np.float32)
            if h not in pos:
                continue
            if h not in feats:
                ph = coords @ W[h].T                      # [N, d/2]
                feats[h] = (a[h] * np.concatenate([np.cos(ph), np.sin(ph)], axis=1)).astype(np.float32)
            f = feats[h]
            s = np.float32(cfg.noise_std)
            q[b, pos[h]] = bf16_bits(f + s * eq)
            k[b, pos[h]] = bf16_bits(f + s * ek)
            v[b, pos[h]] = bf16_bits(vv)
    return q, k, v
