"""fva_route_static: routing for callers that cannot allocate device memory (a
plugin whose host framework owns every device allocation, a serving loop with a
fixed memory plan).  It must give the same results as fva_route with a caller
workspace, call after call, although every call reuses the library's one static
scratch array.  Collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import numpy as np
import pytest

import synth


def _geom(fva, cfg):
    return fva.Geom.of(cfg)


def test_oversized_geometry_is_rejected_without_gpu_work():
    import block_sparse_attention_44_b200 as fva
    g = _geom(fva, synth.CONFIGS["wan720p"].with_(tt=1))   # 64-token tiles: ~94 MiB of routing scratch
    assert fva.fva_route_workspace_size(g) > fva.ROUTE_STATIC_SCRATCH_BYTES
    rc = fva.lib.fva_route_static(256, 512, g.c(), 0.9, 4, 768, 1024, None, None)
    assert rc == fva.FVA_ERR_UNSUPPORTED
    assert b"static scratch" in fva.lib.fva_last_error()


@pytest.mark.gpu
def test_route_static_matches_route_on_consecutive_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_44_b200 as fva
    from gpu_util import to_dev

    # two different inputs, so the second call cannot pass on stale scratch contents
    cfg_a = synth.Config("noalloc_a", B=2, H=6, d=128, T=4, Y=16, X=48, tt=2, ty=8, tx=8, p=0.9, k=4, seed=11)
    cfg_b = cfg_a.with_(name="noalloc_b", p=0.8, k=2, seed=12)
    g = _geom(fva, cfg_a)
    assert fva.fva_route_workspace_size(g) <= fva.ROUTE_STATIC_SCRATCH_BYTES

    def inputs(cfg):
        q, k, _ = synth.make_qkv(cfg)
        shp = (g.B, g.H, g.N, g.d)
        qr, kr = (torch.empty(shp, dtype=torch.bfloat16, device="cuda") for _ in range(2))
        fva.fva_reorder(to_dev(q), qr, g)
        fva.fva_reorder(to_dev(k), kr, g)
        return qr, kr

    def outputs(kk):
        return (torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.uint8, device="cuda"),
                torch.empty((g.B, g.H, g.Nb, min(kk, g.Nb)), dtype=torch.int32, device="cuda"),
                torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.float64, device="cuda"))

    ws = torch.empty((fva.fva_route_workspace_size(g),), dtype=torch.uint8, device="cuda")
    for cfg in (cfg_a, cfg_b):                        # two calls in a row
        qr, kr = inputs(cfg)
        m_ref, t_ref, l_ref = outputs(cfg.k)
        fva.fva_route(qr, kr, g, cfg.p, cfg.k, m_ref, t_ref, ws, logits_out=l_ref)
        m, t, l = outputs(cfg.k)
        fva.fva_route_static(qr, kr, g, cfg.p, cfg.k, m, t, logits_out=l)
        torch.cuda.synchronize()
        assert fva.fva_get_device_error() == 0
        # routing is exact integer work on float64 logits: the tolerance is equality
        assert torch.equal(m, m_ref)
        assert torch.equal(t, t_ref)
        assert np.array_equal(l.cpu().numpy(), l_ref.cpu().numpy())
