"""Pins for the CPU oracle: each check ties an oracle function to something other
than itself (hand-derived fixtures, brute force, library routines, closed forms,
invariants), so that a dropped term, a wrong sign, index or transposed operand
fails at least one of them.  CPU only."""
import dataclasses
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth
from conftest import GOLDEN


def _rand_bits(rng, shape, scale=1.0):
    return synth.bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


# ---------------------------------------------------------------- reorder ---------
def test_reorder_hand_fixtures():
    fx = json.load(open(os.path.join(GOLDEN, "reorder_fixtures.json")))
    for c in fx["cases"]:
        g = O.Geometry(1, 1, c["T"], c["Y"], c["X"], 2, c["tt"], c["ty"], c["tx"])
        assert O.tile_source_index(g).tolist() == c["src"]


@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (1, 8, 8)), ((4, 16, 16), (2, 8, 8)),
                                       ((3, 6, 10), (3, 2, 5)), ((2, 4, 6), (1, 1, 1))])
def test_reorder_blocks_are_tiles_bruteforce(grid, tile):
    T, Y, X = grid
    tt, ty, tx = tile
    g = O.Geometry(1, 1, T, Y, X, 2, tt, ty, tx)
    src = O.tile_source_index(g)
    assert sorted(src.tolist()) == list(range(g.N))          # a bijection
    # independent construction: walk tiles in raster order with nested loops
    expect = []
    for bt in range(T // tt):
        for by in range(Y // ty):
            for bx in range(X // tx):
                for lt in range(tt):
                    for ly in range(ty):
                        for lx in range(tx):
                            t, y, x = bt * tt + lt, by * ty + ly, bx * tx + lx
                            expect.append((t * Y + y) * X + x)
    assert src.tolist() == expect


def test_reorder_roundtrip_identity():
    rng = np.random.default_rng(1)
    g = O.Geometry(2, 3, 4, 8, 8, 16, 2, 4, 4)
    x = _rand_bits(rng, (2, 3, g.N, 16))
    xr = O.reorder(x, g)
    assert not np.array_equal(xr, x)
    assert np.array_equal(O.inverse_reorder(xr, g), x)
    assert np.array_equal(O.reorder(O.inverse_reorder(x, g), g), x)


def test_reorder_rejects_nondivisible():
    with pytest.raises(ValueError):
        O.tile_source_index(O.Geometry(1, 1, 4, 8, 9, 2, 1, 8, 8))


# ---------------------------------------------------------------- pooling ---------
def test_pool_hand_fixture():
    fx = json.load(open(os.path.join(GOLDEN, "pool_fixture.json")))
    x = synth.bf16_bits(np.array(fx["tokens"], dtype=np.float32))[None, None]
    got = O.pool_blocks(x, fx["S"])[0, 0]
    assert np.array_equal(got, np.array(fx["means"]))


def test_pool_constant_tiles():
    rng = np.random.default_rng(2)
    consts = rng.integers(-64, 64, size=(1, 2, 5, 8)).astype(np.float32) / 8.0
    x = np.repeat(consts, 7, axis=2)                     # 5 blocks of 7 identical tokens
    got = O.pool_blocks(synth.bf16_bits(x), 7)
    assert np.array_equal(got, consts.astype(np.float64))


def test_bf16_bits_to_f64_matches_torch():
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(1000) * 10).astype(np.float32)
    bits = synth.bf16_bits(f)
    want = torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_bits_to_f64(bits), want)


# ---------------------------------------------------------------- scores ----------
def test_logits_and_softmax_against_torch():
    rng = np.random.default_rng(4)
    qbar = rng.standard_normal((2, 3, 6, 16))
    kbar = rng.standard_normal((2, 3, 6, 16))
    L = O.block_logits(qbar, kbar)
    want = torch.einsum("bhid,bhjd->bhij", torch.from_numpy(qbar), torch.from_numpy(kbar)) / 4.0
    assert np.allclose(L, want.numpy(), rtol=1e-13, atol=1e-13)
    P = O.row_softmax(L)
    assert np.allclose(P.sum(-1), 1.0, atol=1e-12)
    assert np.allclose(P, torch.softmax(torch.from_numpy(L), dim=-1).numpy(), rtol=1e-12, atol=1e-15)
    # row i of L uses Qbar_i and key column j uses Kbar_j (not transposed)
    assert math.isclose(L[1, 2, 4, 1], float(qbar[1, 2, 4] @ kbar[1, 2, 1]) / 4.0, rel_tol=1e-13)


def test_softmax_no_underflow_at_large_logits():
    L = np.array([[1000.0, 999.0, -1000.0]])
    P = O.row_softmax(L)
    assert np.isfinite(P).all() and math.isclose(P.sum(), 1.0)


# ---------------------------------------------------------------- Top-p -----------
def test_topp_hand_fixtures():
    fx = json.load(open(os.path.join(GOLDEN, "topp_fixtures.json")))
    for c in fx["cases"]:
        P = np.array(c["P"])
        L = np.log(P)
        order, C, n_p, kk = O.topp_keep(L, P, c["p"], c["k"])
        assert n_p == c["n_p"], c
        assert sorted(order[:max(n_p, kk)].tolist()) == c["keep"], c


def _bruteforce_topp(P, p):
    """Minimum-cardinality subset with mass >= p; among those the largest mass."""
    Nb = P.size
    best = None
    for r in range(1, Nb + 1):
        for sub in itertools.combinations(range(Nb), r):
            m = P[list(sub)].sum()
            if m >= p and (best is None or m > best[1]):
                best = (set(sub), m)
        if best is not None:
            return best[0]
    return set(range(Nb))


@pytest.mark.parametrize("Nb", [2, 3, 5, 8])
def test_topp_bruteforce_small(Nb):
    rng = np.random.default_rng(10 + Nb)
    for trial in range(40):
        L = rng.standard_normal(Nb) * rng.uniform(0.3, 4.0)
        P = O.row_softmax(L[None])[0]
        for p in (0.3, 0.5, 0.8, 0.9, 0.99):
            order, C, n_p, kk = O.topp_keep(L, P, p, 1)
            assert set(order[:n_p].tolist()) == _bruteforce_topp(P, p)


def test_floor_and_diagonal_invariants():
    rng = np.random.default_rng(5)
    g = O.Geometry(2, 3, 2, 8, 16, 8, 1, 4, 4)
    q = _rand_bits(rng, (2, 3, g.N, 8), 3.0)
    k = _rand_bits(rng, (2, 3, g.N, 8), 3.0)
    for kfloor in (1, 3, 5):
        rr = O.route(q, k, g, 0.3, kfloor)
        rp = O.repair(rr.topp_mask, rr.topk_idx)
        assert (rp.counts >= min(kfloor, g.Nb)).all()
        ii = np.arange(g.Nb)
        assert (rp.mask[:, :, ii, ii] == 1).all()
        # the Top-p set of each row carries mass >= p
        mass = (rr.P * rr.topp_mask).sum(-1)
        assert (mass >= 0.3 - 1e-12).all()


def test_p_one_keeps_all_blocks():
    rng = np.random.default_rng(6)
    g = O.Geometry(1, 2, 2, 8, 8, 8, 1, 4, 4)
    q = _rand_bits(rng, (1, 2, g.N, 8), 4.0)
    k = _rand_bits(rng, (1, 2, g.N, 8), 4.0)
    rr = O.route(q, k, g, 1.0, 1)
    assert (rr.topp_mask == 1).all()


def test_tiny_p_reduces_to_topk_union_diag():
    rng = np.random.default_rng(7)
    g = O.Geometry(1, 2, 2, 8, 16, 8, 1, 4, 4)
    q = _rand_bits(rng, (1, 2, g.N, 8), 2.0)
    k = _rand_bits(rng, (1, 2, g.N, 8), 2.0)
    for kfloor in (1, 2, 4):
        rr = O.route(q, k, g, 1e-300, kfloor)
        rp = O.repair(rr.topp_mask, rr.topk_idx)
        top = torch.topk(torch.from_numpy(rr.L), kfloor, dim=-1).indices.numpy()
        for h in range(2):
            for i in range(g.Nb):
                want = set(top[0, h, i].tolist()) | {i}
                assert set(rp.idx[0, h, i, :rp.counts[0, h, i]].tolist()) == want


def test_topk_ties_prefer_lower_index():
    L = np.zeros(6)
    P = O.row_softmax(L[None])[0]
    order, C, n_p, kk = O.topp_keep(L, P, 1e-9, 3)
    assert order[:3].tolist() == [0, 1, 2]


def _f32_to_bf16_bits(a) -> np.ndarray:
    """Bit patterns of values that bfloat16 holds exactly (checked)."""
    f = np.asarray(a, dtype=np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), f)
    return bits


def test_route_operand_order_hand_case():
    """Pooled Q goes to the rows of the score matrix and pooled K to its columns: a
    hand-derived case with Qbar and Kbar deliberately different (a transposed or
    self-paired wiring keeps other sets)."""
    fx = json.load(open(os.path.join(GOLDEN, "route_operand_fixture.json")))
    gd = fx["geometry"]
    g = O.Geometry(gd["B"], gd["H"], gd["T"], gd["Y"], gd["X"], gd["d"], gd["tt"], gd["ty"], gd["tx"])
    q = _f32_to_bf16_bits(fx["q_tokens"])[None]
    k = _f32_to_bf16_bits(fx["k_tokens"])[None]
    rr = O.route(O.reorder(q, g), O.reorder(k, g), g, fx["p"], fx["k"])
    assert np.array_equal(rr.L[0], np.array(fx["L"], dtype=np.float64))
    assert rr.topp_mask[0].tolist() == fx["topp_mask"]
    assert rr.n_p[0].tolist() == fx["n_p"]
    assert rr.topk_idx[0].tolist() == fx["topk_idx"]
    rp = O.repair(rr.topp_mask, rr.topk_idx)
    assert rp.counts[0].tolist() == fx["repaired_counts"]


# ---------------------------------------------------------------- repair / LPT ----
def test_repair_compaction_and_head_work():
    rng = np.random.default_rng(8)
    B, H, Nb = 2, 3, 7
    m = (rng.random((B, H, Nb, Nb)) < 0.3).astype(np.uint8)
    tk = rng.integers(0, Nb, size=(B, H, Nb, 2)).astype(np.int32)
    rp = O.repair(m, tk)
    for b in range(B):
        for h in range(H):
            for i in range(Nb):
                want = set(np.nonzero(m[b, h, i])[0].tolist()) | set(tk[b, h, i].tolist()) | {i}
                got = rp.idx[b, h, i, :rp.counts[b, h, i]].tolist()
                assert got == sorted(want)
                assert (rp.idx[b, h, i, rp.counts[b, h, i]:] == -1).all()
    assert np.array_equal(rp.head_work, rp.mask.reshape(B, H, -1).sum(-1))


def test_lpt_worklist_is_sorted_permutation():
    rng = np.random.default_rng(9)
    counts = rng.integers(1, 6, size=(2, 3, 11)).astype(np.int32)
    wl = O.lpt_worklist(counts)
    flat = counts.reshape(-1)
    assert sorted(wl.tolist()) == list(range(flat.size))
    c = flat[wl]
    assert (np.diff(c) <= 0).all()
    for a, b in zip(wl[:-1], wl[1:]):                    # ties in ascending item id
        if flat[a] == flat[b]:
            assert a < b


# ---------------------------------------------------------------- attention -------
def _sdpa(q, k, v):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()


def test_dense_attention_matches_torch_sdpa():
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((2, 3, 40, 16)) for _ in range(3))
    assert np.allclose(O.dense_attention(q, k, v), _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


def test_attention_closed_form_two_keys():
    # one query, two keys, d=2: weights are a logistic of the score gap
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[1.0, 0.0], [0.0, 0.0]]]])
    v = np.array([[[[2.0, -1.0], [0.0, 3.0]]]])
    w1 = 1.0 / (1.0 + math.exp(-1.0 / math.sqrt(2.0)))
    want = w1 * v[0, 0, 0] + (1 - w1) * v[0, 0, 1]
    assert np.allclose(O.dense_attention(q, k, v)[0, 0, 0], want, rtol=1e-14)


def test_masked_attention_all_blocks_equals_dense():
    rng = np.random.default_rng(12)
    S, Nb, d = 8, 5, 16
    q, k, v = (_rand_bits(rng, (1, 2, S * Nb, d), 1.5) for _ in range(3))
    counts = np.full((1, 2, Nb), Nb, dtype=np.int32)
    idx = np.broadcast_to(np.arange(Nb, dtype=np.int32), (1, 2, Nb, Nb)).copy()
    got = O.attention(q, k, v, counts, idx, S)
    f = O.bf16_bits_to_f64
    assert np.allclose(got, _sdpa(f(q), f(k), f(v)), rtol=1e-12, atol=1e-12)


def test_masked_attention_single_block_rows():
    rng = np.random.default_rng(13)
    S, Nb, d = 8, 4, 16
    q, k, v = (_rand_bits(rng, (1, 1, S * Nb, d), 1.5) for _ in range(3))
    f = O.bf16_bits_to_f64
    for shift in (0, 1):                                  # diagonal, and "next block"
        counts = np.ones((1, 1, Nb), dtype=np.int32)
        idx = np.full((1, 1, Nb, Nb), -1, dtype=np.int32)
        idx[0, 0, :, 0] = (np.arange(Nb) + shift) % Nb
        got = O.attention(q, k, v, counts, idx, S)
        for i in range(Nb):
            j = (i + shift) % Nb
            want = _sdpa(f(q[:, :, i * S:(i + 1) * S]), f(k[:, :, j * S:(j + 1) * S]),
                         f(v[:, :, j * S:(j + 1) * S]))
            assert np.allclose(got[:, :, i * S:(i + 1) * S], want, rtol=1e-12, atol=1e-12)


def test_two_block_rows_match_sdpa_with_mask():
    rng = np.random.default_rng(14)
    S, Nb, d = 4, 6, 8
    q, k, v = (_rand_bits(rng, (1, 1, S * Nb, d), 2.0) for _ in range(3))
    f = O.bf16_bits_to_f64
    m = np.zeros((1, 1, Nb, Nb), dtype=np.uint8)
    for i in range(Nb):
        m[0, 0, i, i] = 1
        m[0, 0, i, (3 * i + 1) % Nb] = 1
    rp = O.repair(m, np.zeros((1, 1, Nb, 1), dtype=np.int32) + np.arange(Nb)[None, None, :, None])
    got = O.attention(q, k, v, rp.counts, rp.idx, S)
    tok_mask = np.kron(rp.mask[0, 0], np.ones((S, S))).astype(bool)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(f(q)), torch.from_numpy(f(k)), torch.from_numpy(f(v)),
        attn_mask=torch.from_numpy(tok_mask)).numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_pipeline_p1_equals_dense_in_natural_order():
    """reorder -> route(p=1) -> repair -> attention -> inverse == dense attention."""
    cfg = synth.CONFIGS["tiny"]
    g = O.Geometry.of(cfg)
    q, k, v = synth.make_qkv(cfg)
    qr, kr, vr = (O.reorder(t, g) for t in (q, k, v))
    rr = O.route(qr, kr, g, 1.0, cfg.k)
    rp = O.repair(rr.topp_mask, rr.topk_idx)
    out = O.inverse_reorder(O.attention(qr, kr, vr, rp.counts, rp.idx, g.S), g)
    f = O.bf16_bits_to_f64
    assert np.allclose(out, _sdpa(f(q), f(k), f(v)), rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- ties ------------
def _flags_for_row(L_row, p, k):
    L = np.asarray(L_row, dtype=np.float64)[None, None, None, :]
    P = O.row_softmax(L)
    Nb = L.shape[-1]
    rr = O.RouteResult(np.zeros((1, 1, 1, Nb), np.uint8), np.zeros((1, 1, 1, 1), np.int32),
                       L, P, np.zeros((1, 1, 1), np.int64), p=p, k=k)
    return [f[0, 0, 0] for f in O.tie_flags(rr)]


def test_tie_flags_detect_constructed_ties():
    # equal logits straddle the Top-p cut: masses ~ .783, .106, .106, .005
    assert _flags_for_row([3.0, 1.0, 1.0, -2.0], 0.85, 1) == [False, True, False]
    # equal logits straddle the floor boundary
    assert _flags_for_row([3.0, 1.0, 1.0, -2.0], 0.5, 2) == [False, False, True]
    # the cumulative mass lands exactly on p (dyadic masses .5, .25, ...)
    t1, t2p, t2k = _flags_for_row(np.log([0.5, 0.25, 0.125, 0.125]), 0.75, 1)
    assert t1 and not t2p and not t2k
    # the mass of the ranked prefix one short of the cut lies 1e-7 below p
    assert _flags_for_row(np.log([0.5, 0.2499999, 0.2, 0.0500001]), 0.75, 1) == [True, False, False]
    # a clean row raises no flag
    assert _flags_for_row([3.0, 1.0, 0.0, -2.0], 0.85, 1) == [False, False, False]


# ---------------------------------------------------------------- generator -------
def test_generator_deterministic_and_head_subset():
    cfg = synth.CONFIGS["tiny"].with_(H=3)
    a = synth.make_qkv(cfg)
    b = synth.make_qkv(cfg)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    sub = synth.make_qkv(cfg, heads=[2])
    for x, y in zip(a, sub):
        assert np.array_equal(x[:, 2:3], y)


def test_generator_bf16_rounding_matches_torch():
    rng = np.random.default_rng(15)
    f = (rng.standard_normal(4096) * 100).astype(np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_bits(f), want)


def test_generator_head_scales():
    cfg = synth.CONFIGS["stress720p"]
    a = synth.head_scales(cfg, np.zeros(cfg.H))
    assert (a[0::2] == 4.0).all() and (a[1::2] == 0.3).all()
    lu = synth.head_scales(synth.CONFIGS["wan480p"], np.linspace(0, 1, 40))
    assert math.isclose(lu[0], 0.5) and math.isclose(lu[-1], 4.0)


# ----------------------------------------------------------------- Hilbert tile numbering
def test_hilbert_2x2x2_matches_hand_derivation():
    fx = json.load(open(os.path.join(GOLDEN, "hilbert_fixture.json")))
    for h, c in enumerate(fx["cells_in_order"]):
        assert O.hilbert_index_3d(tuple(c), fx["bits"]) == h


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_hilbert_cube_is_a_face_adjacent_path(bits):
    side = 1 << bits
    idx = {}
    for c in itertools.product(range(side), repeat=3):
        idx[O.hilbert_index_3d(c, bits)] = c
    assert sorted(idx) == list(range(side ** 3))          # a bijection onto [0, side^3)
    assert idx[0] == (0, 0, 0)
    for h in range(1, side ** 3):                        # consecutive cells share a face
        a, b = idx[h - 1], idx[h]
        assert sum(abs(x - y) for x, y in zip(a, b)) == 1, (h, a, b)


def test_tile_order_raster_is_identity_and_hilbert_a_permutation():
    g = O.Geometry(1, 1, 20, 32, 48, 64, 2, 8, 8)
    assert np.array_equal(O.tile_order(g), np.arange(240))
    gh = dataclasses.replace(g, order="hilbert")
    o = O.tile_order(gh)
    assert sorted(o.tolist()) == list(range(240)) and not np.array_equal(o, np.arange(240))
    # a power-of-two grid: consecutive tiles are face neighbours
    g8 = O.Geometry(1, 1, 8, 32, 32, 64, 2, 8, 8, "hilbert")      # 4 x 4 x 4 tiles
    o8 = O.tile_order(g8)
    for a, b in zip(o8[:-1], o8[1:]):
        ca, cb = np.unravel_index(a, (4, 4, 4)), np.unravel_index(b, (4, 4, 4))
        assert sum(abs(int(x) - int(y)) for x, y in zip(ca, cb)) == 1


def test_tile_order_2x2x2_grid_follows_the_hand_derived_curve():
    # a 2 x 2 x 2 tile grid numbers its tiles along the hand-derived 2x2x2 curve; cell
    # (bt, by, bx) is raster tile (bt * 2 + by) * 2 + bx
    fx = json.load(open(os.path.join(GOLDEN, "hilbert_fixture.json")))
    g = O.Geometry(1, 1, 4, 16, 16, 64, 2, 8, 8, "hilbert")
    want = [(bt * 2 + by) * 2 + bx for bt, by, bx in fx["cells_in_order"]]
    assert O.tile_order(g).tolist() == want


def test_reorder_with_hilbert_numbering():
    g = O.Geometry(1, 2, 4, 16, 24, 64, 2, 8, 8, "hilbert")       # 2 x 2 x 3 tiles
    x = np.random.default_rng(5).integers(0, 1 << 16, size=(1, 2, g.N, 64), dtype=np.uint16)
    xr = O.reorder(x, g)
    assert np.array_equal(O.inverse_reorder(xr, g), x)
    src = O.tile_source_index(g)
    order = O.tile_order(g)
    nY, nX = g.Y // g.ty, g.X // g.tx
    for b in range(g.Nb):   # block b holds exactly the tokens of tile order[b], in raster order
        bt, rem = divmod(int(order[b]), nY * nX)
        by, bx = divmod(rem, nX)
        want = [((bt * g.tt + lt) * g.Y + by * g.ty + ly) * g.X + bx * g.tx + lx
                for lt in range(g.tt) for ly in range(g.ty) for lx in range(g.tx)]
        assert src[b * g.S:(b + 1) * g.S].tolist() == want


# ----------------------------------------------------------------- slack-aware augmentation
def _routed(cfg):
    og = O.Geometry.of(cfg)
    q, k, _ = synth.make_qkv(cfg)
    rr = O.route(O.reorder(q, og), O.reorder(k, og), og, cfg.p, cfg.k)
    rp = O.repair(rr.topp_mask, rr.topk_idx)
    prefix = np.maximum(rr.n_p, min(cfg.k, og.Nb))
    return og, rr, rp, prefix


def test_sasa_hand_case():
    # B = 1, H = 4 heads of Nb = 2 rows, every row keeping a ranked prefix of 1 block
    prefix = np.ones((1, 4, 2), dtype=np.int64)
    hw = np.array([[4, 3, 2, 1]])
    # 2 ranks {0, 1}, {2, 3}: W = 7, 3, W* = 7; alpha 0.5: B_1 = floor(0.5 * 4) = 2 over the
    # 4 rows of rank 1 in item order: q = 0, rem = 2, so rows (h2, i0), (h2, i1) get +1
    assert O.sasa_extend(prefix, hw, 2, 0.5).tolist() == [[[1, 1], [1, 1], [2, 2], [1, 1]]]
    # alpha 0.3: B_1 = floor(1.2) = 1, to the first row of rank 1 only
    assert O.sasa_extend(prefix, hw, 2, 0.3).tolist() == [[[1, 1], [1, 1], [2, 1], [1, 1]]]
    # alpha 1: B_1 = 4: q = 1 for every row of rank 1
    assert O.sasa_extend(prefix, hw, 2, 1.0).tolist() == [[[1, 1], [1, 1], [2, 2], [2, 2]]]
    # 4 ranks, alpha 1: W* = 4, budgets 0, 1, 2, 3 over 2 rows each: (h1, i0) +1; h2 +1, +1;
    # h3 +2 (capped at Nb = 2), +1
    assert O.sasa_extend(prefix, hw, 4, 1.0).tolist() == [[[1, 1], [2, 1], [2, 2], [2, 2]]]
    assert O.sasa_extend(prefix, hw, 4, 0.0).tolist() == prefix.tolist()


def test_sasa_invariants():
    cfg = synth.Config("sasa", B=1, H=4, d=64, T=4, Y=16, X=16, tt=1, ty=8, tx=8, p=0.9, k=2,
                       a_mode="alternating", a_lo=4.0, a_hi=0.5, noise_std=1.0, sigma=0.3, seed=3)
    og, rr, rp, prefix = _routed(cfg)
    for R in (1, 2, 4):
        for alpha in (0.0, 0.3, 1.0):
            au = O.sasa_augment(rr.L, prefix, rp.head_work, R, alpha)
            hpr = cfg.H // R
            W = [int(rp.head_work[:, r * hpr:(r + 1) * hpr].sum()) for r in range(R)]
            Wa = [int(au.head_work[:, r * hpr:(r + 1) * hpr].sum()) for r in range(R)]
            Ws = max(W)
            assert max(Wa) == Ws                                  # the critical path does not grow
            for r in range(R):
                assert Wa[r] - W[r] <= math.floor(alpha * (Ws - W[r]))   # within the rank's budget
                if W[r] == Ws:
                    assert Wa[r] == W[r]
            assert (au.mask >= rp.mask).all()                    # only additions
            if alpha == 0.0:
                assert np.array_equal(au.counts, rp.counts)
            for h in range(cfg.H):                               # kept minus diagonal = a ranked prefix
                for i in range(og.Nb):
                    order = O.rank_order(rr.L[0, h, i])
                    kept = au.mask[0, h, i].copy()
                    n = int(kept[order].cumprod().sum())
                    rest = kept.copy()
                    rest[order[:n]] = 0
                    rest[i] = 0
                    assert not rest.any()
