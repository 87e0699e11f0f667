"""Planted mistakes in the CPU oracle: each mutant below is one oracle function with one
plausible error (a dropped term, a wrong sign, index or axis, a transposed operand, an
off-by-one at the cut, the wrong tie order).  With the mutant patched in, every pin test
named beside it must fail.  This shows that the pins pin: no mistake of these kinds can
sit in the oracle while its pins stay green.  CPU only; nothing here touches the GPU path.
"""
import math

import numpy as np
import pytest

import oracle as O
import oracle.fva_oracle as OF
import test_oracle_pins as pins

_TILE_ORDER = OF.tile_order


# ---------------------------------------------------------------- the mutants -------
def m_tile_within_xy_swapped(g):
    """Tokens inside a tile walked x-major (lx before ly) instead of raster order."""
    g.check()
    nT, nY, nX = g.T // g.tt, g.Y // g.ty, g.X // g.tx
    npos = np.arange(g.N, dtype=np.int64)
    b, r = np.divmod(npos, g.S)
    b = OF.tile_order(g)[b]
    bt, rem = np.divmod(b, nY * nX)
    by, bx = np.divmod(rem, nX)
    lt, rem = np.divmod(r, g.ty * g.tx)
    lx, ly = np.divmod(rem, g.ty)
    return ((bt * g.tt + lt) * g.Y + by * g.ty + ly) * g.X + bx * g.tx + lx


def m_tile_grid_column_major(g):
    """Tiles numbered with t fastest instead of x fastest."""
    g.check()
    nT, nY, nX = g.T // g.tt, g.Y // g.ty, g.X // g.tx
    npos = np.arange(g.N, dtype=np.int64)
    b, r = np.divmod(npos, g.S)
    b = OF.tile_order(g)[b]
    bx, rem = np.divmod(b, nT * nY)
    by, bt = np.divmod(rem, nT)
    lt, rem = np.divmod(r, g.ty * g.tx)
    ly, lx = np.divmod(rem, g.tx)
    return ((bt * g.tt + lt) * g.Y + by * g.ty + ly) * g.X + bx * g.tx + lx


def m_inverse_gathers(xr, g):
    """Inverse reorder applying the forward gather a second time."""
    return np.ascontiguousarray(xr[:, :, OF.tile_source_index(g), :])


def m_bf16_unshifted(b):
    """bf16 bits read as the low half of a float32."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


def m_pool_sum(xr_bits, S):
    """Block sum without the 1/S."""
    B, H, N, d = xr_bits.shape
    return OF.bf16_bits_to_f64(xr_bits).reshape(B, H, N // S, S, d).sum(axis=3)


def m_pool_strided(xr_bits, S):
    """Mean over tokens S apart instead of S consecutive tokens."""
    B, H, N, d = xr_bits.shape
    return OF.bf16_bits_to_f64(xr_bits).reshape(B, H, S, N // S, d).mean(axis=2)


def m_logits_unscaled(qbar, kbar):
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2))


def m_logits_over_d(qbar, kbar):
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / qbar.shape[-1]


def m_logits_transposed(qbar, kbar):
    """K Q^T: row i holds the scores of key block i."""
    return np.matmul(kbar, np.swapaxes(qbar, -1, -2)) / np.sqrt(qbar.shape[-1])


def m_softmax_wrong_axis(L):
    z = np.exp(L - L.max(axis=-2, keepdims=True))
    return z / z.sum(axis=-2, keepdims=True)


def m_softmax_unshifted(L):
    with np.errstate(over="ignore", invalid="ignore"):
        z = np.exp(L)
        return z / z.sum(axis=-1, keepdims=True)


def m_rank_ties_high(L_row):
    j = np.arange(L_row.shape[0])
    return np.lexsort((-j, -L_row))


def m_rank_ascending(L_row):
    j = np.arange(L_row.shape[0])
    return np.lexsort((j, L_row))


def _topp_with(cut):
    def f(L_row, P_row, p, k):
        Nb = L_row.shape[0]
        order = OF.rank_order(L_row)
        C = np.cumsum(P_row[order])
        n_p = Nb if p >= 1.0 else cut(C, p, Nb)
        return order, C, n_p, min(int(k), Nb)
    return f


def _cut_strict(C, p, Nb):
    """'reaches' read as strictly above p."""
    hit = np.nonzero(C > p)[0]
    return int(hit[0]) + 1 if hit.size else Nb


def _cut_one_short(C, p, Nb):
    """The 0-based position of the first hit used as the count."""
    hit = np.nonzero(C >= p)[0]
    return int(hit[0]) if hit.size else Nb


def _route_with(floor_ids=lambda order, kk: order[:kk], rows="q", cols="k"):
    """route() with a planted mistake: the floor taken from elsewhere in the ranking, or
    the pooled operands wired to the wrong side of the score matrix (rows / cols name
    the tensor whose block means form Qbar / Kbar)."""
    def f(qr_bits, kr_bits, g, p, k):
        src = {"q": qr_bits, "k": kr_bits}
        qr_bits, kr_bits = src[rows], src[cols]
        B, H, Nb = g.B, g.H, g.Nb
        kk = min(k, Nb)
        L = np.empty((B, H, Nb, Nb))
        mask = np.zeros((B, H, Nb, Nb), dtype=np.uint8)
        topk = np.zeros((B, H, Nb, kk), dtype=np.int32)
        n_p = np.zeros((B, H, Nb), dtype=np.int64)
        for b in range(B):
            for h in range(H):
                L[b, h] = OF.block_logits(OF.pool_blocks(qr_bits[b:b + 1, h:h + 1], g.S),
                                          OF.pool_blocks(kr_bits[b:b + 1, h:h + 1], g.S))[0, 0]
        P = OF.row_softmax(L)
        for b in range(B):
            for h in range(H):
                for i in range(Nb):
                    order, _, npi, _ = OF.topp_keep(L[b, h, i], P[b, h, i], p, k)
                    mask[b, h, i, order[:npi]] = 1
                    topk[b, h, i] = np.sort(floor_ids(order, kk))
                    n_p[b, h, i] = npi
        return OF.RouteResult(mask, topk, L, P, n_p, p, k)
    return f


def _repair_with(floor=True, diagonal=True, descending=False):
    def f(topp_mask, topk_idx):
        B, H, Nb, _ = topp_mask.shape
        mask = topp_mask.astype(np.uint8).copy()
        for b in range(B):
            for h in range(H):
                for i in range(Nb):
                    if floor:
                        mask[b, h, i, topk_idx[b, h, i]] = 1
                    if diagonal:
                        mask[b, h, i, i] = 1
        counts = mask.sum(axis=-1).astype(np.int32)
        idx = np.full((B, H, Nb, Nb), -1, dtype=np.int32)
        for b in range(B):
            for h in range(H):
                for i in range(Nb):
                    js = np.nonzero(mask[b, h, i])[0]
                    idx[b, h, i, :js.size] = js[::-1] if descending else js
        return OF.RepairResult(mask, counts, idx, counts.sum(-1).astype(np.int64), OF.lpt_worklist(counts))
    return f


def m_lpt_ties_high(counts):
    c = counts.reshape(-1).astype(np.int64)
    u = np.arange(c.size)
    return np.lexsort((-u, -c)).astype(np.int32)


def m_lpt_light_first(counts):
    c = counts.reshape(-1).astype(np.int64)
    u = np.arange(c.size)
    return np.lexsort((u, c)).astype(np.int32)


def _attention_items_with(scaled=True, keys_from_query=False, norm_axis=1):
    def f(qr_bits, kr_bits, vr_bits, counts, idx, S, items, scale=None):
        d = qr_bits.shape[-1]
        if scale is None:
            scale = 1.0 / np.sqrt(d) if scaled else 1.0
        out = {}
        for (b, h, i) in items:
            js = idx[b, h, i, :counts[b, h, i]]
            q = OF.bf16_bits_to_f64(qr_bits[b, h, i * S:(i + 1) * S])
            rows = np.concatenate([np.arange(j * S, (j + 1) * S) for j in js])
            krows = np.concatenate([np.arange(i * S, (i + 1) * S) for _ in js]) if keys_from_query else rows
            kk = OF.bf16_bits_to_f64(kr_bits[b, h, krows])
            vv = OF.bf16_bits_to_f64(vr_bits[b, h, rows])
            s = (q @ kk.T) * scale
            w = np.exp(s - s.max(axis=norm_axis, keepdims=True))
            w /= w.sum(axis=norm_axis, keepdims=True)
            out[(b, h, i)] = w @ vv
        return out
    return f


def m_dense_times_sqrt_d(q, k, v, scale=None):
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * math.sqrt(q.shape[-1])
    w = np.exp(s - s.max(axis=-1, keepdims=True))
    return np.matmul(w / w.sum(axis=-1, keepdims=True), v)


def m_dense_k_v_swapped(q, k, v, scale=None):
    s = np.matmul(q, np.swapaxes(v, -1, -2)) / math.sqrt(q.shape[-1])
    w = np.exp(s - s.max(axis=-1, keepdims=True))
    return np.matmul(w / w.sum(axis=-1, keepdims=True), k)


def _hilbert_with(gray=True, reverse_read=False):
    def f(c, bits):
        X = [int(v) for v in c]
        M = 1 << (bits - 1)
        Q = M
        while Q > 1:
            P = Q - 1
            for i in range(3):
                if X[i] & Q:
                    X[0] ^= P
                else:
                    t = (X[0] ^ X[i]) & P
                    X[0] ^= t
                    X[i] ^= t
            Q >>= 1
        if gray:
            for i in range(1, 3):
                X[i] ^= X[i - 1]
            t = 0
            Q = M
            while Q > 1:
                if X[2] & Q:
                    t ^= Q - 1
                Q >>= 1
            for i in range(3):
                X[i] ^= t
        h = 0
        for j in range(bits - 1, -1, -1):
            for i in (range(2, -1, -1) if reverse_read else range(3)):
                h = (h << 1) | ((X[i] >> j) & 1)
        return h
    return f


def m_tile_order_descending(g):
    """Tiles numbered from the far end of the curve."""
    o = _TILE_ORDER(g)
    return o[::-1].copy() if g.order == "hilbert" else o


def _sasa_with(rounding=math.floor, rem_to_last=False, wstar=max, interleaved=False):
    def f(prefix, head_work, num_ranks, alpha):
        B, H, Nb = prefix.shape
        hpr = H // num_ranks
        heads = [[h for h in range(H) if h % num_ranks == r] if interleaved else list(range(r * hpr, (r + 1) * hpr))
                 for r in range(num_ranks)]
        W = [int(head_work[:, hs].sum()) for hs in heads]
        Ws = wstar(W) if wstar is max else int(sum(W) / len(W))
        out = np.array(prefix, dtype=np.int64)
        for r in range(num_ranks):
            budget = max(0, int(rounding(alpha * float(Ws - W[r]))))
            n_rows = B * hpr * Nb
            q, rem = divmod(budget, n_rows)
            pos = 0
            for b in range(B):
                for h in heads[r]:
                    for i in range(Nb):
                        extra = (pos >= n_rows - rem) if rem_to_last else (pos < rem)
                        out[b, h, i] = min(Nb, int(prefix[b, h, i]) + q + (1 if extra else 0))
                        pos += 1
        return out
    return f


def m_ties_ignore_mass_below(rr, tol=1e-5):
    """T1 without the ranked prefix one short of the cut."""
    B, H, R, Nb = rr.L.shape
    t1 = np.zeros((B, H, R), dtype=bool)
    t2p = np.zeros_like(t1)
    t2k = np.zeros_like(t1)
    for b in range(B):
        for h in range(H):
            for i in range(R):
                order, C, n_p, kk = OF.topp_keep(rr.L[b, h, i], rr.P[b, h, i], rr.p, rr.k)
                Ls = rr.L[b, h, i, order]
                if rr.p < 1.0 and (abs(C[n_p - 1] - rr.p) <= tol or C[-1] < rr.p + tol):
                    t1[b, h, i] = True

                def close(n):
                    return n < Nb and abs(Ls[n - 1] - Ls[n]) <= tol * max(1.0, abs(Ls[n - 1]))
                t2p[b, h, i] = close(n_p)
                t2k[b, h, i] = close(kk)
    return t1, t2p, t2k


# (id, oracle function replaced, mutant, pin tests that must fail: (name, args))
MUTANTS = [
    ("tile-inner-xy-swapped", "tile_source_index", m_tile_within_xy_swapped,
     [("test_reorder_hand_fixtures", ()), ("test_reorder_blocks_are_tiles_bruteforce", ((4, 8, 8), (1, 8, 8)))]),
    ("tile-grid-column-major", "tile_source_index", m_tile_grid_column_major,
     [("test_reorder_hand_fixtures", ()), ("test_reorder_blocks_are_tiles_bruteforce", ((4, 16, 16), (2, 8, 8)))]),
    ("inverse-gathers", "inverse_reorder", m_inverse_gathers,
     [("test_reorder_roundtrip_identity", ())]),
    ("bf16-unshifted", "bf16_bits_to_f64", m_bf16_unshifted,
     [("test_bf16_bits_to_f64_matches_torch", ()), ("test_pool_hand_fixture", ())]),
    ("pool-sum", "pool_blocks", m_pool_sum,
     [("test_pool_hand_fixture", ()), ("test_pool_constant_tiles", ())]),
    ("pool-strided", "pool_blocks", m_pool_strided,
     [("test_pool_hand_fixture", ()), ("test_pool_constant_tiles", ())]),
    ("logits-unscaled", "block_logits", m_logits_unscaled, [("test_logits_and_softmax_against_torch", ())]),
    ("logits-over-d", "block_logits", m_logits_over_d, [("test_logits_and_softmax_against_torch", ())]),
    ("logits-transposed", "block_logits", m_logits_transposed, [("test_logits_and_softmax_against_torch", ())]),
    ("softmax-wrong-axis", "row_softmax", m_softmax_wrong_axis,
     [("test_logits_and_softmax_against_torch", ()), ("test_topp_bruteforce_small", (5,))]),
    ("softmax-unshifted", "row_softmax", m_softmax_unshifted, [("test_softmax_no_underflow_at_large_logits", ())]),
    ("rank-ties-high", "rank_order", m_rank_ties_high, [("test_topk_ties_prefer_lower_index", ())]),
    ("rank-ascending", "rank_order", m_rank_ascending,
     [("test_topp_hand_fixtures", ()), ("test_topp_bruteforce_small", (5,))]),
    ("cut-strict", "topp_keep", _topp_with(_cut_strict), [("test_topp_hand_fixtures", ())]),
    ("cut-one-short", "topp_keep", _topp_with(_cut_one_short),
     [("test_topp_hand_fixtures", ()), ("test_topp_bruteforce_small", (5,)), ("test_floor_and_diagonal_invariants", ())]),
    ("floor-from-the-tail", "route", _route_with(lambda order, kk: order[-kk:]),
     [("test_tiny_p_reduces_to_topk_union_diag", ())]),
    ("route-operands-swapped", "route", _route_with(rows="k", cols="q"), [("test_route_operand_order_hand_case", ())]),
    ("route-q-against-q", "route", _route_with(rows="q", cols="q"), [("test_route_operand_order_hand_case", ())]),
    ("route-k-against-k", "route", _route_with(rows="k", cols="k"), [("test_route_operand_order_hand_case", ())]),
    ("repair-drops-floor", "repair", _repair_with(floor=False),
     [("test_repair_compaction_and_head_work", ()), ("test_tiny_p_reduces_to_topk_union_diag", ())]),
    ("repair-drops-diagonal", "repair", _repair_with(diagonal=False),
     [("test_repair_compaction_and_head_work", ()), ("test_floor_and_diagonal_invariants", ())]),
    ("repair-descending-lists", "repair", _repair_with(descending=True),
     [("test_repair_compaction_and_head_work", ())]),
    ("lpt-ties-high", "lpt_worklist", m_lpt_ties_high, [("test_lpt_worklist_is_sorted_permutation", ())]),
    ("lpt-light-first", "lpt_worklist", m_lpt_light_first, [("test_lpt_worklist_is_sorted_permutation", ())]),
    ("attn-unscaled", "attention_items", _attention_items_with(scaled=False),
     [("test_masked_attention_all_blocks_equals_dense", ()), ("test_two_block_rows_match_sdpa_with_mask", ())]),
    ("attn-keys-from-query-block", "attention_items", _attention_items_with(keys_from_query=True),
     [("test_masked_attention_single_block_rows", ()), ("test_masked_attention_all_blocks_equals_dense", ())]),
    ("attn-normalised-over-queries", "attention_items", _attention_items_with(norm_axis=0),
     [("test_masked_attention_all_blocks_equals_dense", ())]),
    ("dense-times-sqrt-d", "dense_attention", m_dense_times_sqrt_d,
     [("test_dense_attention_matches_torch_sdpa", ()), ("test_attention_closed_form_two_keys", ())]),
    ("dense-k-v-swapped", "dense_attention", m_dense_k_v_swapped, [("test_dense_attention_matches_torch_sdpa", ())]),
    ("hilbert-no-gray", "hilbert_index_3d", _hilbert_with(gray=False),
     [("test_hilbert_2x2x2_matches_hand_derivation", ()), ("test_hilbert_cube_is_a_face_adjacent_path", (2,))]),
    ("hilbert-read-reversed", "hilbert_index_3d", _hilbert_with(reverse_read=True),
     [("test_hilbert_2x2x2_matches_hand_derivation", ())]),
    ("tile-order-descending", "tile_order", m_tile_order_descending,
     [("test_tile_order_2x2x2_grid_follows_the_hand_derived_curve", ())]),
    ("sasa-ceil", "sasa_extend", _sasa_with(rounding=math.ceil), [("test_sasa_hand_case", ())]),
    ("sasa-remainder-to-last", "sasa_extend", _sasa_with(rem_to_last=True), [("test_sasa_hand_case", ())]),
    ("sasa-mean-not-critical", "sasa_extend", _sasa_with(wstar=None), [("test_sasa_hand_case", ())]),
    ("sasa-ranks-interleaved", "sasa_extend", _sasa_with(interleaved=True), [("test_sasa_hand_case", ())]),
    ("ties-ignore-mass-below", "tie_flags", m_ties_ignore_mass_below, [("test_tie_flags_detect_constructed_ties", ())]),
]


@pytest.mark.parametrize("name,target,mutant,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(monkeypatch, name, target, mutant, catchers):
    assert hasattr(OF, target) and hasattr(O, target), target
    for pin, args in catchers:                 # every named pin passes on the real oracle
        getattr(pins, pin)(*args)
    monkeypatch.setattr(OF, target, mutant)    # calls inside the oracle module
    monkeypatch.setattr(O, target, mutant)     # calls through the package, as the pins make them
    survived = []
    for pin, args in catchers:
        try:
            with np.errstate(all="ignore"):
                getattr(pins, pin)(*args)
        except Exception:                      # an assertion, or the mutant breaking a shape
            continue
        survived.append(pin)
    assert not survived, f"mutant {name} passes {survived}"
