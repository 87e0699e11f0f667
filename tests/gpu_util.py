"""Helpers for the GPU parity tests: move seeded bf16 inputs to the device, run the
library path step by step, and compare with the oracle under the parity rules
(bit-exact integer work modulo flagged ties; attention within max-abs 2e-2 and
relative-L2 5e-3 with the device's own index lists fed to the oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

ATOL = 2e-2
REL_L2 = 5e-3


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return O.bf16_bits_to_f64(to_bits(t))


def run_path(fva, g, q, k, v, p, kfloor, use_lpt=True, want_logits=False):
    """Runs every library step; returns a dict of device results (torch tensors)."""
    dev = {}
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    shp = (g.B, g.H, g.N, g.d)
    qr, kr, vr, outr, out = (torch.empty(shp, dtype=torch.bfloat16, device="cuda") for _ in range(5))
    fva.fva_reorder(qd, qr, g)
    fva.fva_reorder(kd, kr, g)
    fva.fva_reorder(vd, vr, g)
    kk = min(kfloor, g.Nb)
    mask = torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.uint8, device="cuda")
    topk = torch.empty((g.B, g.H, g.Nb, kk), dtype=torch.int32, device="cuda")
    ws = torch.empty((fva.fva_route_workspace_size(g),), dtype=torch.uint8, device="cuda")
    logits = torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.float64, device="cuda") if want_logits else None
    fva.fva_route(qr, kr, g, p, kfloor, mask, topk, ws, logits_out=logits)
    counts = torch.empty((g.B, g.H, g.Nb), dtype=torch.int32, device="cuda")
    idx = torch.full((g.B, g.H, g.Nb, g.Nb), -1, dtype=torch.int32, device="cuda")
    hw = torch.empty((g.B, g.H), dtype=torch.int64, device="cuda")
    wl = torch.empty((g.B * g.H * g.Nb,), dtype=torch.int32, device="cuda")
    fva.fva_repair(mask, topk, g, kfloor, counts, idx, hw, wl)
    # the fused entry point on the same inputs, with and without the route outputs
    fused = dict(counts=torch.empty_like(counts), idx=torch.full_like(idx, -1), head_work=torch.empty_like(hw),
                 worklist=torch.empty_like(wl), mask=torch.empty_like(mask), topk=torch.empty_like(topk))
    fva.fva_route_repair(qr, kr, g, p, kfloor, fused["counts"], fused["idx"], fused["head_work"],
                         fused["worklist"], ws, topp_mask=fused["mask"], topk_idx=fused["topk"])
    bare = dict(counts=torch.empty_like(counts), idx=torch.full_like(idx, -1), head_work=torch.empty_like(hw),
                worklist=torch.empty_like(wl))
    fva.fva_route_repair(qr, kr, g, p, kfloor, bare["counts"], bare["idx"], bare["head_work"], bare["worklist"],
                         ws)
    fva.fva_block_sparse_attn(qr, kr, vr, counts, idx, wl if use_lpt else None, g, 0.0, outr)
    fva.fva_inverse_reorder(outr, out, g)
    out_nat = torch.empty_like(out)
    fva.fva_block_sparse_attn_natural(qr, kr, vr, counts, idx, wl if use_lpt else None, g, 0.0, out_nat)
    torch.cuda.synchronize()
    assert fva.fva_get_device_error() == 0
    # the fused epilogue writes exactly the inverse reorder of the tile-major output
    assert torch.equal(out_nat.view(torch.int16), out.view(torch.int16))
    # pooling done by the reorder pass, then routing from those means
    qbar, kbar = (torch.empty((g.B, g.H, g.Nb, g.d), dtype=torch.float64, device="cuda") for _ in range(2))
    qr2, kr2 = torch.empty_like(qr), torch.empty_like(kr)
    fva.fva_reorder_pool(qd, qr2, qbar, g)
    fva.fva_reorder_pool(kd, kr2, kbar, g)
    pooled = dict(counts=torch.empty_like(counts), idx=torch.full_like(idx, -1), head_work=torch.empty_like(hw),
                  worklist=torch.empty_like(wl), mask=torch.empty_like(mask), topk=torch.empty_like(topk))
    fva.fva_route_repair_pooled(qbar, kbar, g, p, kfloor, pooled["counts"], pooled["idx"], pooled["head_work"],
                                pooled["worklist"], topp_mask=pooled["mask"], topk_idx=pooled["topk"])
    torch.cuda.synchronize()
    assert fva.fva_get_device_error() == 0
    dev.update(qr=qr, kr=kr, vr=vr, mask=mask, topk=topk, logits=logits, counts=counts, idx=idx, head_work=hw,
               worklist=wl, outr=outr, out=out, fused=fused, bare=bare, pooled=pooled, qr2=qr2, kr2=kr2, qbar=qbar,
               kbar=kbar)
    return dev


def check_fused(dev: dict):
    """fva_route_repair gives exactly what fva_route followed by fva_repair gives."""
    for res in (dev["fused"], dev["bare"]):
        for key in ("counts", "head_work", "worklist"):
            assert torch.equal(res[key], dev[key]), key
        Nb = dev["idx"].shape[-1]
        valid = torch.arange(Nb, device=dev["idx"].device)[None, None, None, :] < dev["counts"][..., None]
        assert torch.equal(torch.where(valid, res["idx"], -1), torch.where(valid, dev["idx"], -1))
    assert torch.equal(dev["fused"]["mask"], dev["mask"])
    assert torch.equal(dev["fused"]["topk"], dev["topk"])


def check_pooled(dev: dict, q: np.ndarray, k: np.ndarray, og):
    """fva_reorder_pool reorders exactly like fva_reorder and its means match the oracle's
    pooling; routing from those means gives exactly the lists of the other entry points."""
    assert torch.equal(dev["qr2"].view(torch.int16), dev["qr"].view(torch.int16))
    assert torch.equal(dev["kr2"].view(torch.int16), dev["kr"].view(torch.int16))
    for bar, x in ((dev["qbar"], q), (dev["kbar"], k)):
        want = O.pool_blocks(O.reorder(x, og), og.S)
        assert np.allclose(bar.cpu().numpy(), want, rtol=1e-13, atol=1e-15)
    res = dev["pooled"]
    for key in ("counts", "head_work", "worklist", "mask", "topk"):
        assert torch.equal(res[key], dev[key]), key
    Nb = dev["idx"].shape[-1]
    valid = torch.arange(Nb, device=dev["idx"].device)[None, None, None, :] < dev["counts"][..., None]
    assert torch.equal(torch.where(valid, res["idx"], -1), torch.where(valid, dev["idx"], -1))


TIE_TOL = 1e-5


def _near_top_set(L_row: np.ndarray, members: np.ndarray, n: int, tol: float) -> bool:
    """`members` (bool [Nb], n of them set) is a set of the n highest logits of the row,
    up to swaps of blocks whose logits lie within tol * max(1, |L|) of the n-th
    highest: no member lies clearly below it and no non-member clearly above it."""
    Ls = L_row[O.rank_order(L_row)]
    thr = Ls[n - 1]
    band = tol * max(1.0, abs(thr))
    return not (L_row[members] < thr - band).any() and not (L_row[~members] > thr + band).any()


def valid_tie_topp(L_row, P_row, mask_row, p, tol=TIE_TOL) -> bool:
    """A Top-p set another rounding of the masses may legitimately choose on a tie row:
    a ranked prefix (up to near-equal logits at its end) whose exact mass reaches
    p - tol, and which is minimal within tol (dropping its lowest-ranked block leaves
    less than p + tol).  Keeping every block is valid when the exact total mass lies
    within tol of p or below it."""
    members = mask_row.astype(bool)
    n = int(members.sum())
    Nb = members.size
    if n == 0 or not _near_top_set(L_row, members, n, tol):
        return False
    mass = float(P_row[members].sum())
    if n == Nb and float(P_row.sum()) < p + tol:
        return True
    if mass < p - tol:
        return False
    rank = np.empty(Nb, dtype=np.int64)
    rank[O.rank_order(L_row)] = np.arange(Nb)
    idx = np.nonzero(members)[0]
    last = idx[np.argmax(rank[idx])]
    return mass - float(P_row[last]) < p + tol


def valid_tie_topk(L_row, ids, kk, tol=TIE_TOL) -> bool:
    """kk distinct ascending block ids forming a set of the kk highest logits, up to
    swaps among logits within tol * max(1, |L|) at the floor boundary."""
    ids = np.asarray(ids)
    if ids.size != kk or (np.diff(ids) <= 0).any() or ids.min() < 0 or ids.max() >= L_row.size:
        return False
    members = np.zeros(L_row.size, dtype=bool)
    members[ids] = True
    return _near_top_set(L_row, members, kk, tol)


def check_route(rr: O.RouteResult, mask_dev: np.ndarray, topk_dev: np.ndarray, max_tie_frac=0.02):
    """Bit-exact comparison except rows flagged as ties; a tie row where the device
    differs must still hold a valid answer (valid_tie_topp / valid_tie_topk).
    Returns (n_rows, n_tie_rows, n_diff_rows); every differing row was validated."""
    t1, t2p, t2k = O.tie_flags(rr)
    dm = (mask_dev != rr.topp_mask).any(-1)
    dk = (topk_dev != rr.topk_idx).any(-1)
    bad_m = dm & ~(t1 | t2p)
    bad_k = dk & ~t2k
    assert not bad_m.any(), f"{int(bad_m.sum())} Top-p rows differ without a tie, e.g. {np.argwhere(bad_m)[:5]}"
    assert not bad_k.any(), f"{int(bad_k.sum())} Top-k rows differ without a tie, e.g. {np.argwhere(bad_k)[:5]}"
    kk = rr.topk_idx.shape[-1]
    for b, h, i in np.argwhere(dm):
        assert valid_tie_topp(rr.L[b, h, i], rr.P[b, h, i], mask_dev[b, h, i], rr.p), \
            f"tie row {(b, h, i)}: device Top-p set is not a valid answer"
    for b, h, i in np.argwhere(dk):
        assert valid_tie_topk(rr.L[b, h, i], topk_dev[b, h, i], kk), \
            f"tie row {(b, h, i)}: device floor is not a valid top-{kk} set"
    ties = t1 | t2p | t2k
    assert ties.mean() <= max_tie_frac, f"tie rows {ties.mean():.4f} above {max_tie_frac}"
    return int(ties.size), int(ties.sum()), int((dm | dk).sum())


def check_repair(fva_dev: dict, mask_dev: np.ndarray, topk_dev: np.ndarray):
    """The device repair outputs equal the oracle repair of the device's own route outputs, exactly."""
    rp = O.repair(mask_dev, topk_dev)
    counts = fva_dev["counts"].cpu().numpy()
    idx = fva_dev["idx"].cpu().numpy()
    assert np.array_equal(counts, rp.counts)
    B, H, Nb = counts.shape
    valid = np.arange(Nb)[None, None, None, :] < counts[..., None]
    assert np.array_equal(np.where(valid, idx, -1), rp.idx)
    assert np.array_equal(fva_dev["head_work"].cpu().numpy(), rp.head_work)
    assert np.array_equal(fva_dev["worklist"].cpu().numpy(), rp.worklist)
    return rp


def compare_attention(got: np.ndarray, want: np.ndarray):
    err = np.abs(got - want)
    mx = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert mx <= ATOL, f"max-abs {mx:.3e} > {ATOL}"
    assert rel <= REL_L2, f"rel-L2 {rel:.3e} > {REL_L2}"
    return mx, rel
