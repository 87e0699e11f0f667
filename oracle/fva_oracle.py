"""CPU oracle for FVAttn-style adaptive block-sparse attention (TEST INFRASTRUCTURE ONLY).

This is the plain, slow, obviously-correct restatement of what the hot path
computes.  It exists to check the CUDA path and is used only by the tests, the
smoke entry and the CPU-baseline leg of the benchmark; the product never
imports, calls or links it, and it shares no code with the CUDA library.

Source of every step: "FVAttn: Adaptive Sparse Attention with Runtime Load
Balancing for Video Generation" (the paper page), whose abstract, §2 background
on dynamic sparse routing and §3.1 pipeline overview describe the routing
frontend (video-aware block organisation, pooled Q/K block similarities, a Top-p
CDF threshold with a Top-k safety floor, mask materialisation and runtime repair)
and then block-sparse attention.  Where the page is silent the readings are:

* blocks are 3D box tiles of tt x ty x tx tokens, numbered in raster order of
  the tile grid (or, with order="hilbert", along the Hilbert curve of the §3.1
  overview, see tile_order); tokens inside a tile are in raster order;
* "pooled" = arithmetic mean over the tile's tokens, in float64, of the
  bfloat16 inputs;
* block importance = row softmax over key blocks of Qbar_i . Kbar_j / sqrt(d);
* the ranking used by the CDF threshold is by logit, descending, ties to the
  lower key-block index ("larger logit first" is the same order as larger
  probability, but logits do not underflow to equal zeros);
* "reaches" means ">=": n_p = min{n : C_n >= p}; for p >= 1 every block is kept;
* the Top-k floor is a union: keep the first max(n_p, min(k, Nb)) blocks of the
  ranking;
* repair forces the diagonal block (self-attention, so query block i and key
  block i cover the same tokens), then compacts each row into an ascending list;
* per-head realised workload W_h = number of kept block pairs of head h
  (the workload definition in §2, sequence parallelism);
* attention is bidirectional (no causal mask), scale 1/sqrt(d), over exactly
  the kept key blocks;
* the work list is every (b, h, i) item ordered by kept-block count descending,
  ties by item id ascending (longest processing time first).

Pins (tests/test_oracle_pins.py) tie each function to something other than
itself: hand-derived fixtures under tests/golden/, brute-force subset
enumeration, library routines (torch scaled_dot_product_attention, torch.topk),
closed forms and invariants.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable, Optional

import numpy as np

__all__ = [
    "Geometry", "hilbert_index_3d", "tile_order", "tile_source_index", "reorder", "inverse_reorder", "bf16_bits_to_f64",
    "pool_blocks", "block_logits", "row_softmax", "rank_order", "topp_keep",
    "RouteResult", "route", "RepairResult", "repair", "lpt_worklist",
    "attention_items", "attention", "dense_attention", "tie_flags", "sasa_extend", "sasa_augment",
]


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Batch B, heads H, latent grid T x Y x X, head_dim d, tile tt x ty x tx."""

    B: int
    H: int
    T: int
    Y: int
    X: int
    d: int
    tt: int
    ty: int
    tx: int
    order: str = "raster"   # numbering of the tiles: "raster" or "hilbert"

    @property
    def N(self) -> int:
        return self.T * self.Y * self.X

    @property
    def S(self) -> int:
        return self.tt * self.ty * self.tx

    @property
    def Nb(self) -> int:
        return self.N // self.S

    def check(self) -> None:
        if self.T % self.tt or self.Y % self.ty or self.X % self.tx:
            raise ValueError("latent grid must be divisible by the tile")

    @staticmethod
    def of(cfg, order: str = "raster") -> "Geometry":
        return Geometry(cfg.B, cfg.H, cfg.T, cfg.Y, cfg.X, cfg.d, cfg.tt, cfg.ty, cfg.tx, order)


# --------------------------------------------------------------------------------------
# Step 1: video-aware block organisation (abstract; §3.1 overview, block reordering).
# --------------------------------------------------------------------------------------
def hilbert_index_3d(c: tuple, bits: int) -> int:
    """Position of grid cell c = (c0, c1, c2), each in [0, 2^bits), along the 3D Hilbert
    curve of the 2^bits cube: Skilling's method ("Programming the Hilbert curve", 2004),
    restated.  The coordinates are turned into the curve's "transposed" index: for each
    bit level from the top, the lower bits are reflected or exchanged with the first
    coordinate (undoing the curve's rotations), then the coordinates are Gray-coded;
    the index is the transposed bits read level by level, c0 first."""
    X = [int(v) for v in c]
    n = 3
    M = 1 << (bits - 1)
    Q = M
    while Q > 1:
        P = Q - 1
        for i in range(n):
            if X[i] & Q:
                X[0] ^= P
            else:
                t = (X[0] ^ X[i]) & P
                X[0] ^= t
                X[i] ^= t
        Q >>= 1
    for i in range(1, n):
        X[i] ^= X[i - 1]
    t = 0
    Q = M
    while Q > 1:
        if X[n - 1] & Q:
            t ^= Q - 1
        Q >>= 1
    for i in range(n):
        X[i] ^= t
    h = 0
    for j in range(bits - 1, -1, -1):
        for i in range(n):
            h = (h << 1) | ((X[i] >> j) & 1)
    return h


def tile_order(g: Geometry) -> np.ndarray:
    """order[b] = raster index of the tile numbered b.  Raster numbering is the identity.
    Hilbert numbering (the §3.1 overview reorders blocks along a Hilbert curve so that
    spatially adjacent tokens fall into nearby blocks): the tile grid (nT, nY, nX) sits
    in the smallest 2^bits cube that holds it, and its tiles are numbered by ascending
    Hilbert index of (bt, by, bx) in that cube (a generalisation to grids whose sides are
    not powers of two: cells outside the grid are skipped)."""
    g.check()
    nT, nY, nX = g.T // g.tt, g.Y // g.ty, g.X // g.tx
    if g.order == "raster":
        return np.arange(nT * nY * nX, dtype=np.int64)
    if g.order != "hilbert":
        raise ValueError(f"unknown tile order {g.order!r}")
    bits = max(1, int(max(nT, nY, nX) - 1).bit_length())
    keys = []
    for bt in range(nT):
        for by in range(nY):
            for bx in range(nX):
                keys.append((hilbert_index_3d((bt, by, bx), bits), (bt * nY + by) * nX + bx))
    keys.sort()
    return np.array([r for _, r in keys], dtype=np.int64)


def tile_source_index(g: Geometry) -> np.ndarray:
    """src[n'] = natural token index n of the token placed at reordered position n'.

    Position n' = b * S + r, with b the number of the tile (tile_order: raster index of
    the tile over the tile grid (T/tt, Y/ty, X/tx), or its Hilbert rank) and r the raster
    index of the token inside the tile over (tt, ty, tx).  The natural index is
    n = (t * Y + y) * X + x.
    """
    g.check()
    nT, nY, nX = g.T // g.tt, g.Y // g.ty, g.X // g.tx
    npos = np.arange(g.N, dtype=np.int64)
    b, r = np.divmod(npos, g.S)
    b = tile_order(g)[b]
    bt, rem = np.divmod(b, nY * nX)
    by, bx = np.divmod(rem, nX)
    lt, rem = np.divmod(r, g.ty * g.tx)
    ly, lx = np.divmod(rem, g.tx)
    t = bt * g.tt + lt
    y = by * g.ty + ly
    x = bx * g.tx + lx
    return (t * g.Y + y) * g.X + x


def reorder(x: np.ndarray, g: Geometry) -> np.ndarray:
    """x [B, H, N, d] natural order -> tile-major order (an exact gather)."""
    return np.ascontiguousarray(x[:, :, tile_source_index(g), :])


def inverse_reorder(xr: np.ndarray, g: Geometry) -> np.ndarray:
    """Inverse of :func:`reorder` (an exact scatter back to natural order)."""
    out = np.empty_like(xr)
    out[:, :, tile_source_index(g), :] = xr
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact: bf16 is the top half of a float32)."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------------------
# Step 2: pooled Q/K block similarities and the Top-p CDF cut with a Top-k floor
# (§2 background: a per-pair importance score turned into a binary block mask;
# Top-p retains the fewest key blocks whose summed normalised importance is at
# least p; the Top-k floor guarantees a minimum number of blocks;
# §3.1 overview: the scores are block-level similarities of pooled Q and K).
# --------------------------------------------------------------------------------------
def pool_blocks(xr_bits: np.ndarray, S: int) -> np.ndarray:
    """Mean of each block's S tokens, float64.  xr_bits [B, H, N, d] bf16 bits (reordered)."""
    B, H, N, d = xr_bits.shape
    x = bf16_bits_to_f64(xr_bits).reshape(B, H, N // S, S, d)
    return x.mean(axis=3)


def block_logits(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """L[b, h, i, j] = Qbar_i . Kbar_j / sqrt(d), float64."""
    d = qbar.shape[-1]
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / np.sqrt(d)


def row_softmax(L: np.ndarray) -> np.ndarray:
    """Softmax over the last axis, max-subtracted, float64."""
    z = np.exp(L - L.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def rank_order(L_row: np.ndarray) -> np.ndarray:
    """Key blocks of one row ordered by logit descending, ties to the lower index."""
    j = np.arange(L_row.shape[0])
    return np.lexsort((j, -L_row))


def topp_keep(L_row: np.ndarray, P_row: np.ndarray, p: float, k: int):
    """One query block's Top-p set with the Top-k floor.

    Returns (order, C, n_p, kk): the ranking, the cumulative mass C[n-1] = C_n of
    the first n ranked blocks, the Top-p count n_p = min{n : C_n >= p}
    (all blocks when p >= 1 or when rounding leaves C_Nb < p) and the floor
    kk = min(k, Nb).  The kept set is order[:max(n_p, kk)].
    """
    Nb = L_row.shape[0]
    order = rank_order(L_row)
    C = np.cumsum(P_row[order])
    if p >= 1.0:
        n_p = Nb
    else:
        hit = np.nonzero(C >= p)[0]
        n_p = int(hit[0]) + 1 if hit.size else Nb
    kk = min(int(k), Nb)
    return order, C, n_p, kk


@dataclasses.dataclass
class RouteResult:
    topp_mask: np.ndarray   # uint8 [B, H, Nb, Nb]: the Top-p set of each row
    topk_idx: np.ndarray    # int32 [B, H, Nb, kk]: the first kk ranked blocks, ascending ids
    L: np.ndarray           # float64 [B, H, Nb, Nb] logits
    P: np.ndarray           # float64 [B, H, Nb, Nb] block probabilities
    n_p: np.ndarray         # int64 [B, H, Nb]
    p: float
    k: int


def route(qr_bits: np.ndarray, kr_bits: np.ndarray, g: Geometry, p: float, k: int) -> RouteResult:
    """Pool, score, and cut every (b, h, query-block) row."""
    if not (0.0 < p <= 1.0) or k < 1:
        raise ValueError("need 0 < p <= 1 and k >= 1")
    B, H, Nb = g.B, g.H, g.Nb
    kk = min(k, Nb)
    L = np.empty((B, H, Nb, Nb), dtype=np.float64)
    mask = np.zeros((B, H, Nb, Nb), dtype=np.uint8)
    topk = np.zeros((B, H, Nb, kk), dtype=np.int32)
    n_p = np.zeros((B, H, Nb), dtype=np.int64)
    for b in range(B):
        for h in range(H):  # one head at a time keeps the float64 copies small
            L[b, h] = block_logits(pool_blocks(qr_bits[b:b + 1, h:h + 1], g.S),
                                   pool_blocks(kr_bits[b:b + 1, h:h + 1], g.S))[0, 0]
    P = row_softmax(L)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                order, _, npi, _ = topp_keep(L[b, h, i], P[b, h, i], p, k)
                mask[b, h, i, order[:npi]] = 1
                topk[b, h, i] = np.sort(order[:kk])
                n_p[b, h, i] = npi
    return RouteResult(mask, topk, L, P, n_p, p, k)


# --------------------------------------------------------------------------------------
# Step 3: runtime mask repair and compaction (abstract: the materialised mask is
# fixed up at run time; §2 sequence parallelism: realised per-head workload).
# --------------------------------------------------------------------------------------
@dataclasses.dataclass
class RepairResult:
    mask: np.ndarray        # uint8 [B, H, Nb, Nb] repaired mask
    counts: np.ndarray      # int32 [B, H, Nb]
    idx: np.ndarray         # int32 [B, H, Nb, Nb], ascending ids, -1 past counts
    head_work: np.ndarray   # int64 [B, H]
    worklist: np.ndarray    # int32 [B * H * Nb], LPT order of items u = (b*H + h)*Nb + i


def lpt_worklist(counts: np.ndarray) -> np.ndarray:
    """Items ordered by count descending, ties by item id ascending."""
    c = counts.reshape(-1).astype(np.int64)
    u = np.arange(c.size)
    return np.lexsort((u, -c)).astype(np.int32)


def repair(topp_mask: np.ndarray, topk_idx: np.ndarray) -> RepairResult:
    """Union of the Top-p mask, the Top-k floor and the diagonal; compact rows."""
    B, H, Nb, _ = topp_mask.shape
    mask = topp_mask.astype(np.uint8).copy()
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                mask[b, h, i, topk_idx[b, h, i]] = 1
                mask[b, h, i, i] = 1
    counts = mask.sum(axis=-1).astype(np.int32)
    idx = np.full((B, H, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                js = np.nonzero(mask[b, h, i])[0]
                idx[b, h, i, : js.size] = js
    head_work = counts.sum(axis=-1).astype(np.int64)
    return RepairResult(mask, counts, idx, head_work, lpt_worklist(counts))


# --------------------------------------------------------------------------------------
# Step 4: block-sparse attention over the kept blocks (§3.1 overview, last
# compute stage; §2 background: only the selected block pairs are evaluated).
# --------------------------------------------------------------------------------------
# --------------------------------------------------------------------------------------
# Slack-aware augmentation, single-GPU reading (§3.3 SASA; the formulas are garbled in the
# page text, the readings are stated here).  The heads are split into num_ranks virtual
# ranks of H / num_ranks consecutive heads (the Ulysses head layout of §2); W_r = sum of
# W_h over the rank's heads and batch items; W* = max_r W_r is the critical path; rank r
# gets the extra budget B_r = floor(alpha * (W* - W_r)) block pairs (alpha: the
# augmentation coefficient, 0 <= alpha <= 1, so W_r + B_r <= W*).  B_r is spread over
# the rank's rows, in item order u = (b*H + h)*Nb + i, round-robin: q = B_r // n_rows
# extra positions each, one more for the first B_r % n_rows rows.  A row extends its
# ranked prefix (the Top-p set with the floor, max(n_p, min(k, Nb)) blocks, following the
# routing's importance order) by its share, capped at Nb: the kept set becomes the first
# min(Nb, prefix + share) ranked blocks plus the diagonal.
# --------------------------------------------------------------------------------------
def sasa_extend(prefix: np.ndarray, head_work: np.ndarray, num_ranks: int, alpha: float) -> np.ndarray:
    """New ranked-prefix length of every row: prefix int [B, H, Nb] (max(n_p, kk) per row),
    head_work int [B, H] (W_h of the current lists).  Returns int64 [B, H, Nb]."""
    B, H, Nb = prefix.shape
    if num_ranks < 1 or H % num_ranks:
        raise ValueError("num_ranks must divide H")
    if not (0.0 <= alpha <= 1.0):
        raise ValueError("need 0 <= alpha <= 1")
    hpr = H // num_ranks
    W = [int(head_work[:, r * hpr:(r + 1) * hpr].sum()) for r in range(num_ranks)]
    Wstar = max(W)
    out = np.array(prefix, dtype=np.int64)
    for r in range(num_ranks):
        budget = int(math.floor(alpha * float(Wstar - W[r])))
        n_rows = B * hpr * Nb
        q, rem = divmod(budget, n_rows)
        pos = 0
        for b in range(B):
            for h in range(r * hpr, (r + 1) * hpr):
                for i in range(Nb):
                    share = q + (1 if pos < rem else 0)
                    out[b, h, i] = min(Nb, int(prefix[b, h, i]) + share)
                    pos += 1
    return out


def sasa_augment(L: np.ndarray, prefix: np.ndarray, head_work: np.ndarray, num_ranks: int,
                 alpha: float) -> RepairResult:
    """Augmented lists: row (b, h, i) keeps the first sasa_extend(...) blocks of its ranking
    (logits L [B, H, Nb, Nb], descending, ties to the lower id) and its diagonal block."""
    B, H, Nb = prefix.shape
    newlen = sasa_extend(prefix, head_work, num_ranks, alpha)
    mask = np.zeros((B, H, Nb, Nb), dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                mask[b, h, i, rank_order(L[b, h, i])[:newlen[b, h, i]]] = 1
                mask[b, h, i, i] = 1
    counts = mask.sum(-1).astype(np.int32)
    idx = np.full((B, H, Nb, Nb), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                nz = np.nonzero(mask[b, h, i])[0]
                idx[b, h, i, :nz.size] = nz
    hw = counts.sum(-1).astype(np.int64)
    return RepairResult(mask, counts, idx, hw, lpt_worklist(counts))


def attention_items(qr_bits, kr_bits, vr_bits, counts, idx, S: int, items: Iterable, scale: Optional[float] = None):
    """Exact float64 output rows of the given items.

    items: iterable of (b, h, i).  Returns {(b, h, i): float64 [S, d]}: for every
    query token of block i, softmax over the tokens of the kept key blocks only
    (scale 1/sqrt(d) unless given), times their values.
    """
    d = qr_bits.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = {}
    for (b, h, i) in items:
        js = idx[b, h, i, : counts[b, h, i]]
        q = bf16_bits_to_f64(qr_bits[b, h, i * S:(i + 1) * S])
        rows = np.concatenate([np.arange(j * S, (j + 1) * S) for j in js])
        kk = bf16_bits_to_f64(kr_bits[b, h, rows])
        vv = bf16_bits_to_f64(vr_bits[b, h, rows])
        s = (q @ kk.T) * scale
        s = s - s.max(axis=1, keepdims=True)
        w = np.exp(s)
        w /= w.sum(axis=1, keepdims=True)
        out[(b, h, i)] = w @ vv
    return out


def attention(qr_bits, kr_bits, vr_bits, counts, idx, S: int, scale: Optional[float] = None) -> np.ndarray:
    """Float64 block-sparse attention output [B, H, N, d] in reordered token order."""
    B, H, N, d = qr_bits.shape
    Nb = N // S
    out = np.empty((B, H, N, d), dtype=np.float64)
    items = [(b, h, i) for b in range(B) for h in range(H) for i in range(Nb)]
    res = attention_items(qr_bits, kr_bits, vr_bits, counts, idx, S, items, scale)
    for (b, h, i), o in res.items():
        out[b, h, i * S:(i + 1) * S] = o
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: Optional[float] = None) -> np.ndarray:
    """Plain float64 softmax(Q K^T * scale) V over the last two axes (all pairs)."""
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(axis=-1, keepdims=True)
    return np.matmul(w, v)


# --------------------------------------------------------------------------------------
# Ties: rows where an implementation that rounds differently may legitimately
# choose a different set.
# --------------------------------------------------------------------------------------
def tie_flags(rr: RouteResult, tol: float = 1e-5):
    """Per-row tie flags (bool [B, H, Nb] each): (t1, t2_topp, t2_topk).

    t1: the cumulative mass at the cut lies within ``tol`` of p, i.e.
        |C_{n_p} - p| <= tol or |C_{n_p - 1} - p| <= tol.
    t2_topp / t2_topk: the last kept and the first dropped ranked blocks at the
        Top-p boundary n_p (resp. the floor boundary kk) have logits within
        tol * max(1, |L|) of each other, so a rounding difference may swap them.
    """
    B, H, R, Nb = rr.L.shape          # R query-block rows, Nb key blocks
    t1 = np.zeros((B, H, R), dtype=bool)
    t2p = np.zeros_like(t1)
    t2k = np.zeros_like(t1)
    for b in range(B):
        for h in range(H):
            for i in range(R):
                order, C, n_p, kk = topp_keep(rr.L[b, h, i], rr.P[b, h, i], rr.p, rr.k)
                Ls = rr.L[b, h, i, order]
                if rr.p < 1.0:
                    if abs(C[n_p - 1] - rr.p) <= tol or (n_p >= 2 and abs(C[n_p - 2] - rr.p) <= tol):
                        t1[b, h, i] = True
                    # when rounding leaves the total mass below p every block is kept
                    if C[-1] < rr.p + tol:
                        t1[b, h, i] = True

                def close(n):
                    return n < Nb and abs(Ls[n - 1] - Ls[n]) <= tol * max(1.0, abs(Ls[n - 1]))
                t2p[b, h, i] = close(n_p)
                t2k[b, h, i] = close(kk)
    return t1, t2p, t2k
