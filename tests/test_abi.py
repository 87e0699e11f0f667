"""Host-side checks of the C ABI: the library loads, exports every entry point the
header declares, and rejects bad arguments before touching the GPU.  CPU only."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_44_b200 as fva

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(fva_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"fva_reorder", "fva_inverse_reorder", "fva_route", "fva_repair", "fva_route_repair",
            "fva_block_sparse_attn"} <= names
    raw = ctypes.CDLL(fva.LIB_PATH)
    for n in sorted(names):
        assert hasattr(raw, n), n


def test_version_and_counters():
    assert fva.fva_version() >= 100
    assert fva.fva_launch_count() >= 0


def _g(**kw):
    base = dict(B=1, H=2, T=4, Y=8, X=8, d=64, tt=1, ty=8, tx=8)
    base.update(kw)
    return fva.Geom(**base)


def test_workspace_size_queries():
    g = _g()
    # pooled Q and K (float64), each 256-byte aligned, then the LPT sort's per-head
    # histograms over the counts 0..Nb (int32)
    nb = g.Nb
    rows = g.B * g.H * nb
    def al(x):
        return (x + 255) // 256 * 256
    lpt = al(g.B * g.H * (nb + 1) * 4)
    assert fva.fva_repair_workspace_size(g) == lpt
    assert fva.fva_route_workspace_size(g) == 2 * al(rows * g.d * 8) + lpt
    assert fva.fva_sasa_workspace_size(g) == al(2 * ((rows + 63) // 64 * 64) * 4) + lpt
    assert fva.fva_route_workspace_size(_g(X=9)) == 0          # invalid geometry
    assert fva.fva_repair_workspace_size(_g(X=9)) == 0


def _rc(fn, *args):
    return fn(*args)


def test_invalid_arguments_rejected_on_host():
    L = fva.lib
    g = _g().c()
    assert L.fva_reorder(None, None, g, None) == fva.FVA_ERR_INVALID_ARG
    assert b"null" in L.fva_last_error()
    bad = _g(X=9).c()
    assert L.fva_reorder(16, 32, bad, None) == fva.FVA_ERR_INVALID_ARG
    assert b"divisible" in L.fva_last_error()
    assert L.fva_reorder(16, 16, g, None) == fva.FVA_ERR_INVALID_ARG           # in place
    assert L.fva_reorder(17, 32, g, None) == fva.FVA_ERR_INVALID_ARG           # misaligned
    assert L.fva_reorder(16, 32, _g(d=96).c(), None) == fva.FVA_ERR_UNSUPPORTED
    assert L.fva_reorder(16, 32, _g(B=0).c(), None) == fva.FVA_ERR_INVALID_ARG
    # route: p and k ranges, workspace size and alignment
    args = lambda p, k, ws, wsb: (256, 512, g, p, k, 768, 1024, None, ws, wsb, None)
    need = fva.fva_route_workspace_size(_g())
    assert L.fva_route(*args(0.0, 1, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route(*args(1.5, 1, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route(*args(float("nan"), 1, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route(*args(0.9, 0, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route(*args(0.9, 1, 4096, need - 1)) == fva.FVA_ERR_INVALID_ARG
    assert b"workspace too small" in L.fva_last_error()
    assert L.fva_route(*args(0.9, 1, 4100, need)) == fva.FVA_ERR_INVALID_ARG  # not 256-aligned
    # fused route + repair: same argument rules
    fargs = lambda p, k, ws, wsb: (256, 512, g, p, k, None, None, 16, 32, 64, 128, ws, wsb, None)
    assert L.fva_route_repair(*fargs(0.0, 1, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair(*fargs(0.9, 0, 4096, need)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair(*fargs(0.9, 1, 4096, need - 1)) == fva.FVA_ERR_INVALID_ARG
    assert b"workspace too small" in L.fva_last_error()
    assert L.fva_route_repair(256, 512, g, 0.9, 1, None, None, None, 32, 64, 128, 4096, need, None) == \
        fva.FVA_ERR_INVALID_ARG
    assert b"null" in L.fva_last_error()
    # reorder with pooling, routing from pooled means
    assert L.fva_reorder_pool(16, 32, None, g, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_reorder_pool(16, 16, 64, g, None) == fva.FVA_ERR_INVALID_ARG            # in place
    assert L.fva_reorder_pool(16, 32, 68, g, None) == fva.FVA_ERR_INVALID_ARG            # pooled misaligned
    assert L.fva_reorder_pool(16, 32, 64, bad, None) == fva.FVA_ERR_INVALID_ARG
    rneed = fva.fva_repair_workspace_size(_g())
    assert rneed >= 4 * _g().B * _g().H * (_g().Nb + 1) and rneed % 256 == 0
    pargs = lambda p, k, ws=4096, wsb=rneed: (256, 512, g, p, k, None, None, 16, 32, 64, 128, ws, wsb, None)
    assert L.fva_route_repair_pooled(*pargs(0.0, 1)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_pooled(*pargs(0.9, 0)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_pooled(*pargs(0.9, 1, None)) == fva.FVA_ERR_INVALID_ARG       # no workspace
    assert L.fva_route_repair_pooled(*pargs(0.9, 1, 4096, rneed - 1)) == fva.FVA_ERR_INVALID_ARG
    assert b"workspace too small" in L.fva_last_error()
    assert L.fva_route_repair_pooled(*pargs(0.9, 1, 4100)) == fva.FVA_ERR_INVALID_ARG       # not 256-aligned
    assert L.fva_route_repair_pooled(None, 512, g, 0.9, 1, None, None, 16, 32, 64, 128, 4096, rneed, None) == \
        fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_pooled(264, 512, g, 0.9, 1, None, None, 16, 32, 64, 128, 4096, rneed, None) == \
        fva.FVA_ERR_INVALID_ARG                                                           # qbar misaligned
    # slack-aware augmentation: num_ranks must divide H, alpha in [0, 1], workspace size
    sneed = fva.fva_sasa_workspace_size(_g())
    sargs = lambda R, a, wsb: (256, 512, g, 0.9, 1, R, a, 16, 32, 64, 128, None, 4096, wsb, None)
    assert L.fva_route_repair_sasa(*sargs(3, 0.5, sneed)) == fva.FVA_ERR_INVALID_ARG     # H = 2
    assert L.fva_route_repair_sasa(*sargs(0, 0.5, sneed)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_sasa(*sargs(2, 1.5, sneed)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_sasa(*sargs(2, float("nan"), sneed)) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_route_repair_sasa(*sargs(2, 0.5, sneed - 1)) == fva.FVA_ERR_INVALID_ARG
    assert sneed >= 2 * 4 * _g().B * _g().H * _g().Nb
    # repair / attention: null pointers, k, unsupported tile for attention
    assert L.fva_repair(None, 16, g, 1, 16, 16, 16, 16, 4096, rneed, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_repair(16, 16, g, 0, 16, 16, 16, 16, 4096, rneed, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_repair(16, 16, g, 1, 16, 16, 16, 16, None, 0, None) == fva.FVA_ERR_INVALID_ARG  # no workspace
    assert L.fva_repair(16, 16, g, 1, 16, 16, 16, 16, 4096, rneed - 4, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_block_sparse_attn(16, 16, None, 16, 16, None, g, 0.0, 16, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_block_sparse_attn_natural(16, 16, 16, 16, 16, None, g, 0.0, None, None) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_block_sparse_attn_natural(16, 16, 16, 16, 16, None, _g(tt=1, ty=4, tx=8).c(), 0.0, 16, None) == \
        fva.FVA_ERR_UNSUPPORTED
    t32 = _g(tt=1, ty=4, tx=8).c()                                            # 32-token tiles
    assert L.fva_block_sparse_attn(16, 16, 16, 16, 16, None, t32, 0.0, 16, None) == fva.FVA_ERR_UNSUPPORTED
    assert L.fva_block_sparse_attn(16, 16, 16, 16, 16, None, g, float("inf"), 16, None) == fva.FVA_ERR_INVALID_ARG
    big = _g(T=64, Y=128, X=128, tt=1, ty=8, tx=8).c()                       # Nb = 16384 > 2048
    assert L.fva_route(256, 512, big, 0.9, 1, 768, 1024, None, 4096, 1 << 40, None) == fva.FVA_ERR_UNSUPPORTED


def test_python_wrapper_type_checks():
    import torch
    g = _g()
    x = torch.zeros((1, 2, 256, 64), dtype=torch.float32)
    with pytest.raises(TypeError):
        fva.fva_reorder(x, x, g)


def test_tile_order_table_matches_oracle():
    import numpy as np

    import oracle as O
    for (T, Y, X, tt, ty, tx) in [(20, 32, 48, 2, 8, 8), (20, 48, 80, 2, 8, 8), (3, 5, 7, 1, 1, 1),
                                  (8, 32, 32, 2, 8, 8), (1, 8, 8, 1, 8, 8), (6, 40, 24, 2, 8, 8)]:
        g = fva.Geom(1, 1, T, Y, X, 64, tt, ty, tx)
        want = O.tile_order(O.Geometry(1, 1, T, Y, X, 64, tt, ty, tx, "hilbert"))
        assert np.array_equal(fva.fva_tile_order(g, fva.FVA_TILES_HILBERT), want)
        assert np.array_equal(fva.fva_tile_order(g, fva.FVA_TILES_RASTER), np.arange(g.Nb))
    with pytest.raises(fva.FvaError):
        fva.fva_tile_order(_g(), 7)
    bad = _g().c()
    bad.tile_order = 18                                   # not 4-byte aligned
    assert fva.lib.fva_reorder(16, 32, bad, None) == fva.FVA_ERR_INVALID_ARG


def _declarations():
    """name -> parameter count of every function the header declares."""
    out = {}
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", f)).read(), flags=re.S)
        for m in re.finditer(r"\b(fva_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
            params = m.group(2).strip()
            out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_signatures_match_the_header():
    decl = _declarations()
    assert len(decl) >= 15
    for name, n in decl.items():
        f = getattr(fva.lib, name)
        assert f.argtypes is not None, f"{name}: no ctypes signature in the binding"
        assert len(f.argtypes) == n, f"{name}: header has {n} parameters, binding {len(f.argtypes)}"


def test_geometry_struct_layout():
    # 9 int32 sizes, then the tile-numbering pointer (8-byte aligned)
    assert ctypes.sizeof(fva._Geom) == 48
    assert fva._Geom.tile_order.offset == 40
