"""Thin Python binding of libfva.so (the C ABI in include/fva.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  Importing fails loudly if
the library has not been built (``python -m block_sparse_attention_44_b200.build``);
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

__all__ = [
    "FvaError", "Geom", "lib", "fva_reorder", "fva_inverse_reorder", "fva_route_workspace_size", "fva_route",
    "fva_route_static", "fva_repair_workspace_size", "fva_repair", "fva_block_sparse_attn", "fva_get_device_error", "fva_last_error",
    "fva_launch_count", "fva_version", "RouteOutputs", "RepairOutputs", "SparseAttention", "HostPipeline",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfva.so")

FVA_OK, FVA_ERR_INVALID_ARG, FVA_ERR_UNSUPPORTED, FVA_ERR_CUDA, FVA_ERR_TIMEOUT = range(5)
_CODES = {1: "FVA_ERR_INVALID_ARG", 2: "FVA_ERR_UNSUPPORTED", 3: "FVA_ERR_CUDA", 4: "FVA_ERR_TIMEOUT"}


class FvaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_CODES.get(code, code)}: {msg}")
        self.code = code


class _Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "H", "T", "Y", "X", "d", "tt", "ty", "tx")] + \
               [("tile_order", ctypes.c_void_p)]


FVA_TILES_RASTER, FVA_TILES_HILBERT = 0, 1


@dataclasses.dataclass(frozen=True)
class Geom:
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
    tile_order: Optional[torch.Tensor] = dataclasses.field(default=None, compare=False)  # device int32 [Nb]

    @property
    def N(self) -> int:
        return self.T * self.Y * self.X

    @property
    def S(self) -> int:
        return self.tt * self.ty * self.tx

    @property
    def Nb(self) -> int:
        return self.N // self.S

    def c(self) -> _Geom:
        order = None if self.tile_order is None else self.tile_order.data_ptr()
        return _Geom(self.B, self.H, self.T, self.Y, self.X, self.d, self.tt, self.ty, self.tx, order)

    @staticmethod
    def of(cfg) -> "Geom":
        return Geom(cfg.B, cfg.H, cfg.T, cfg.Y, cfg.X, cfg.d, cfg.tt, cfg.ty, cfg.tx)

    def with_tiles(self, kind: int, device="cuda") -> "Geom":
        """This geometry with the tile numbering `kind` (FVA_TILES_RASTER / _HILBERT) as a device table."""
        table = fva_tile_order(self, kind)
        return dataclasses.replace(self, tile_order=torch.from_numpy(table).to(device))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_44_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, i64, f32, f64 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.c_float, ctypes.c_double)
    sig = {
        "fva_reorder": ([vp, vp, _Geom, vp], ctypes.c_int),
        "fva_tile_order": ([_Geom, i32, vp], ctypes.c_int),
        "fva_inverse_reorder": ([vp, vp, _Geom, vp], ctypes.c_int),
        "fva_route_workspace_size": ([_Geom], sz),
        "fva_route": ([vp, vp, _Geom, f64, i32, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "fva_route_static": ([vp, vp, _Geom, f64, i32, vp, vp, vp, vp], ctypes.c_int),
        "fva_route_repair": ([vp, vp, _Geom, f64, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "fva_reorder_pool": ([vp, vp, vp, _Geom, vp], ctypes.c_int),
        "fva_sasa_workspace_size": ([_Geom], sz),
        "fva_route_repair_sasa": ([vp, vp, _Geom, f64, i32, i32, f64, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "fva_route_repair_pooled": ([vp, vp, _Geom, f64, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "fva_repair_workspace_size": ([_Geom], sz),
        "fva_repair": ([vp, vp, _Geom, i32, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "fva_block_sparse_attn": ([vp, vp, vp, vp, vp, vp, _Geom, f32, vp, vp], ctypes.c_int),
        "fva_block_sparse_attn_natural": ([vp, vp, vp, vp, vp, vp, _Geom, f32, vp, vp], ctypes.c_int),
        "fva_get_device_error": ([vp, ctypes.POINTER(i32)], ctypes.c_int),
        "fva_debug_set_wait_limit": ([i64], ctypes.c_int),
        "fva_last_error": ([], ctypes.c_char_p),
        "fva_launch_count": ([], i64),
        "fva_version": ([], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int) -> None:
    if rc != FVA_OK:
        raise FvaError(rc, lib.fva_last_error().decode())


def _need(t: torch.Tensor, dtype: torch.dtype, shape, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")


# ------------------------------------------------------------------ 1:1 wrappers ----
def fva_tile_order(g: Geom, kind: int):
    """Host table of a tile numbering: order[b] = raster index of the tile numbered b."""
    import numpy as np
    out = np.empty(g.Nb, dtype=np.int32)
    _check(lib.fva_tile_order(dataclasses.replace(g, tile_order=None).c(), int(kind),
                              out.ctypes.data_as(ctypes.c_void_p)))
    return out


def fva_reorder(x: torch.Tensor, xr: torch.Tensor, g: Geom, stream=None) -> None:
    shp = (g.B, g.H, g.N, g.d)
    _need(x, torch.bfloat16, shp, "x")
    _need(xr, torch.bfloat16, shp, "xr")
    _check(lib.fva_reorder(_ptr(x), _ptr(xr), g.c(), _stream(stream)))


def fva_inverse_reorder(xr: torch.Tensor, x: torch.Tensor, g: Geom, stream=None) -> None:
    shp = (g.B, g.H, g.N, g.d)
    _need(xr, torch.bfloat16, shp, "xr")
    _need(x, torch.bfloat16, shp, "x")
    _check(lib.fva_inverse_reorder(_ptr(xr), _ptr(x), g.c(), _stream(stream)))


def fva_reorder_pool(x: torch.Tensor, xr: torch.Tensor, pooled: torch.Tensor, g: Geom, stream=None) -> None:
    """fva_reorder that also writes the float64 tile means (routing's pooled Q or K)."""
    shp = (g.B, g.H, g.N, g.d)
    _need(x, torch.bfloat16, shp, "x")
    _need(xr, torch.bfloat16, shp, "xr")
    _need(pooled, torch.float64, (g.B, g.H, g.Nb, g.d), "pooled")
    _check(lib.fva_reorder_pool(_ptr(x), _ptr(xr), _ptr(pooled), g.c(), _stream(stream)))


def fva_route_workspace_size(g: Geom) -> int:
    return int(lib.fva_route_workspace_size(g.c()))


def fva_route(qr, kr, g: Geom, p: float, k: int, topp_mask, topk_idx, workspace, logits_out=None, stream=None):
    shp = (g.B, g.H, g.N, g.d)
    _need(qr, torch.bfloat16, shp, "qr")
    _need(kr, torch.bfloat16, shp, "kr")
    _need(topp_mask, torch.uint8, (g.B, g.H, g.Nb, g.Nb), "topp_mask")
    _need(topk_idx, torch.int32, (g.B, g.H, g.Nb, min(k, g.Nb)), "topk_idx")
    if logits_out is not None:
        _need(logits_out, torch.float64, (g.B, g.H, g.Nb, g.Nb), "logits_out")
    _check(lib.fva_route(_ptr(qr), _ptr(kr), g.c(), float(p), int(k), _ptr(topp_mask), _ptr(topk_idx),
                         _ptr(logits_out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                         _stream(stream)))


ROUTE_STATIC_SCRATCH_BYTES = 64 << 20


def fva_route_static(qr, kr, g: Geom, p: float, k: int, topp_mask, topk_idx, logits_out=None, stream=None):
    """fva_route without a workspace, for callers that cannot allocate device memory
    (e.g. a plugin whose host framework owns all device allocations, or a serving loop
    with a fixed memory plan).  The routing scratch is a 64 MiB device array inside the
    library, shared by every call on a device: calls that overlap on the GPU race.
    Larger geometries raise FvaError(FVA_ERR_UNSUPPORTED)."""
    shp = (g.B, g.H, g.N, g.d)
    _need(qr, torch.bfloat16, shp, "qr")
    _need(kr, torch.bfloat16, shp, "kr")
    _need(topp_mask, torch.uint8, (g.B, g.H, g.Nb, g.Nb), "topp_mask")
    _need(topk_idx, torch.int32, (g.B, g.H, g.Nb, min(k, g.Nb)), "topk_idx")
    if logits_out is not None:
        _need(logits_out, torch.float64, (g.B, g.H, g.Nb, g.Nb), "logits_out")
    _check(lib.fva_route_static(_ptr(qr), _ptr(kr), g.c(), float(p), int(k), _ptr(topp_mask), _ptr(topk_idx),
                                _ptr(logits_out), _stream(stream)))


def fva_route_repair(qr, kr, g: Geom, p: float, k: int, counts, idx, head_work, worklist, workspace,
                     topp_mask=None, topk_idx=None, stream=None):
    """fva_route followed by fva_repair in one persistent kernel plus the LPT launch;
    the Top-p mask and Top-k ids are written only when their tensors are given."""
    shp = (g.B, g.H, g.N, g.d)
    _need(qr, torch.bfloat16, shp, "qr")
    _need(kr, torch.bfloat16, shp, "kr")
    if topp_mask is not None:
        _need(topp_mask, torch.uint8, (g.B, g.H, g.Nb, g.Nb), "topp_mask")
    if topk_idx is not None:
        _need(topk_idx, torch.int32, (g.B, g.H, g.Nb, min(k, g.Nb)), "topk_idx")
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    _need(head_work, torch.int64, (g.B, g.H), "head_work")
    _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    _check(lib.fva_route_repair(_ptr(qr), _ptr(kr), g.c(), float(p), int(k), _ptr(topp_mask), _ptr(topk_idx),
                                _ptr(counts), _ptr(idx), _ptr(head_work), _ptr(worklist), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream)))


def _workspace(workspace, nbytes: int, like: torch.Tensor) -> torch.Tensor:
    """The caller's workspace, or a fresh device buffer of nbytes (PyTorch allocates it)."""
    if workspace is not None:
        return workspace
    return torch.empty((max(int(nbytes), 256),), dtype=torch.uint8, device=like.device)


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def fva_route_repair_pooled(qbar, kbar, g: Geom, p: float, k: int, counts, idx, head_work, worklist,
                            topp_mask=None, topk_idx=None, workspace=None, stream=None):
    """fva_route_repair from block means already computed (fva_reorder_pool).  workspace:
    fva_repair_workspace_size(g) bytes (allocated here when not given)."""
    _need(qbar, torch.float64, (g.B, g.H, g.Nb, g.d), "qbar")
    _need(kbar, torch.float64, (g.B, g.H, g.Nb, g.d), "kbar")
    if topp_mask is not None:
        _need(topp_mask, torch.uint8, (g.B, g.H, g.Nb, g.Nb), "topp_mask")
    if topk_idx is not None:
        _need(topk_idx, torch.int32, (g.B, g.H, g.Nb, min(k, g.Nb)), "topk_idx")
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    _need(head_work, torch.int64, (g.B, g.H), "head_work")
    _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    ws = _workspace(workspace, fva_repair_workspace_size(g), counts)
    _check(lib.fva_route_repair_pooled(_ptr(qbar), _ptr(kbar), g.c(), float(p), int(k), _ptr(topp_mask),
                                       _ptr(topk_idx), _ptr(counts), _ptr(idx), _ptr(head_work), _ptr(worklist),
                                       _ptr(ws), _nbytes(ws), _stream(stream)))


def fva_sasa_workspace_size(g: Geom) -> int:
    return int(lib.fva_sasa_workspace_size(g.c()))


def fva_route_repair_sasa(qbar, kbar, g: Geom, p: float, k: int, num_ranks: int, alpha: float, counts, idx,
                          head_work, worklist, workspace, extra=None, stream=None):
    """fva_route_repair_pooled with slack-aware augmentation over num_ranks virtual ranks."""
    _need(qbar, torch.float64, (g.B, g.H, g.Nb, g.d), "qbar")
    _need(kbar, torch.float64, (g.B, g.H, g.Nb, g.d), "kbar")
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    _need(head_work, torch.int64, (g.B, g.H), "head_work")
    _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    if extra is not None:
        _need(extra, torch.int32, (g.B, g.H, g.Nb), "extra")
    _check(lib.fva_route_repair_sasa(_ptr(qbar), _ptr(kbar), g.c(), float(p), int(k), int(num_ranks), float(alpha),
                                     _ptr(counts), _ptr(idx), _ptr(head_work), _ptr(worklist), _ptr(extra),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def fva_repair_workspace_size(g: Geom) -> int:
    return int(lib.fva_repair_workspace_size(g.c()))


def fva_repair(topp_mask, topk_idx, g: Geom, k: int, counts, idx, head_work, worklist, workspace=None, stream=None):
    _need(topp_mask, torch.uint8, (g.B, g.H, g.Nb, g.Nb), "topp_mask")
    _need(topk_idx, torch.int32, (g.B, g.H, g.Nb, min(k, g.Nb)), "topk_idx")
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    _need(head_work, torch.int64, (g.B, g.H), "head_work")
    _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    ws = _workspace(workspace, fva_repair_workspace_size(g), counts)
    _check(lib.fva_repair(_ptr(topp_mask), _ptr(topk_idx), g.c(), int(k), _ptr(counts), _ptr(idx), _ptr(head_work),
                          _ptr(worklist), _ptr(ws), _nbytes(ws), _stream(stream)))


def fva_block_sparse_attn(qr, kr, vr, counts, idx, worklist, g: Geom, softmax_scale: float, out_r, stream=None):
    shp = (g.B, g.H, g.N, g.d)
    for t, n in ((qr, "qr"), (kr, "kr"), (vr, "vr"), (out_r, "out_r")):
        _need(t, torch.bfloat16, shp, n)
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    if worklist is not None:
        _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    _check(lib.fva_block_sparse_attn(_ptr(qr), _ptr(kr), _ptr(vr), _ptr(counts), _ptr(idx), _ptr(worklist), g.c(),
                                     float(softmax_scale), _ptr(out_r), _stream(stream)))


def fva_block_sparse_attn_natural(qr, kr, vr, counts, idx, worklist, g: Geom, softmax_scale: float, out,
                                  stream=None):
    """fva_block_sparse_attn writing the output in natural token order (inverse reorder fused)."""
    shp = (g.B, g.H, g.N, g.d)
    for t, n in ((qr, "qr"), (kr, "kr"), (vr, "vr"), (out, "out")):
        _need(t, torch.bfloat16, shp, n)
    _need(counts, torch.int32, (g.B, g.H, g.Nb), "counts")
    _need(idx, torch.int32, (g.B, g.H, g.Nb, g.Nb), "idx")
    if worklist is not None:
        _need(worklist, torch.int32, (g.B * g.H * g.Nb,), "worklist")
    _check(lib.fva_block_sparse_attn_natural(_ptr(qr), _ptr(kr), _ptr(vr), _ptr(counts), _ptr(idx), _ptr(worklist),
                                             g.c(), float(softmax_scale), _ptr(out), _stream(stream)))


def fva_get_device_error(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device error word, 0 if none."""
    code = ctypes.c_int32(0)
    rc = lib.fva_get_device_error(_stream(stream), ctypes.byref(code))
    if rc == FVA_ERR_CUDA:
        raise FvaError(rc, lib.fva_last_error().decode())
    return int(code.value)


def fva_debug_set_wait_limit(cycles: int) -> None:
    """Test only: pipeline wait limit (SM cycles) of the attention launches that follow;
    0 restores the default."""
    _check(lib.fva_debug_set_wait_limit(int(cycles)))


def fva_last_error() -> str:
    return lib.fva_last_error().decode()


def fva_launch_count() -> int:
    return int(lib.fva_launch_count())


def fva_version() -> int:
    return int(lib.fva_version())


# ------------------------------------------------------------------ the whole path ---
@dataclasses.dataclass
class RouteOutputs:
    topp_mask: torch.Tensor
    topk_idx: torch.Tensor


@dataclasses.dataclass
class RepairOutputs:
    counts: torch.Tensor
    idx: torch.Tensor
    head_work: torch.Tensor
    worklist: torch.Tensor


class SparseAttention:
    """The whole path on one device with buffers held across calls:
    reorder(Q, K, V) -> route -> repair -> block-sparse attention -> inverse reorder.

    Buffers are allocated once through PyTorch for a geometry; `__call__` only
    enqueues library kernels on the current (or given) stream.  With fused=True
    (default) Q and K are pooled by their reorder pass (fva_reorder_pool), routing and
    repair run as fva_route_repair_pooled and the Top-p mask / Top-k ids are not
    materialised; fused=False runs fva_reorder, fva_route, then fva_repair.
    """

    def __init__(self, g: Geom, p: float, k: int, device="cuda", use_lpt: bool = True,
                 softmax_scale: float = 0.0, fused: bool = True):
        self.g, self.p, self.k, self.use_lpt, self.scale = g, p, k, use_lpt, softmax_scale
        self.fused = fused
        dev = torch.device(device)
        shp = (g.B, g.H, g.N, g.d)
        self.qr, self.kr, self.vr, self.outr = (torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(4))
        kk = min(k, g.Nb)
        self.route = RouteOutputs(torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.uint8, device=dev),
                                  torch.empty((g.B, g.H, g.Nb, kk), dtype=torch.int32, device=dev))
        self.rep = RepairOutputs(torch.empty((g.B, g.H, g.Nb), dtype=torch.int32, device=dev),
                                 torch.empty((g.B, g.H, g.Nb, g.Nb), dtype=torch.int32, device=dev),
                                 torch.empty((g.B, g.H), dtype=torch.int64, device=dev),
                                 torch.empty((g.B * g.H * g.Nb,), dtype=torch.int32, device=dev))
        self.ws = torch.empty((max(fva_route_workspace_size(g), 256),), dtype=torch.uint8, device=dev)
        self.rws = torch.empty((max(fva_repair_workspace_size(g), 256),), dtype=torch.uint8, device=dev)
        self.qbar, self.kbar = (torch.empty((g.B, g.H, g.Nb, g.d), dtype=torch.float64, device=dev)
                                for _ in range(2))

    def routing(self, stream=None) -> None:
        g = self.g
        if self.fused:   # the means come from the reorder pass (reorder_qk)
            fva_route_repair_pooled(self.qbar, self.kbar, g, self.p, self.k, self.rep.counts, self.rep.idx,
                                    self.rep.head_work, self.rep.worklist, workspace=self.rws, stream=stream)
            return
        fva_route(self.qr, self.kr, g, self.p, self.k, self.route.topp_mask, self.route.topk_idx, self.ws,
                  stream=stream)
        fva_repair(self.route.topp_mask, self.route.topk_idx, g, self.k, self.rep.counts, self.rep.idx,
                   self.rep.head_work, self.rep.worklist, workspace=self.rws, stream=stream)

    def attention(self, stream=None) -> None:
        """Tile-major output into self.outr."""
        fva_block_sparse_attn(self.qr, self.kr, self.vr, self.rep.counts, self.rep.idx,
                              self.rep.worklist if self.use_lpt else None, self.g, self.scale, self.outr,
                              stream=stream)

    def attention_natural(self, out, stream=None) -> None:
        """Natural-order output into `out` (the inverse reorder fused into the epilogue)."""
        fva_block_sparse_attn_natural(self.qr, self.kr, self.vr, self.rep.counts, self.rep.idx,
                                      self.rep.worklist if self.use_lpt else None, self.g, self.scale, out,
                                      stream=stream)

    def reorder_qkv(self, q, k, v, stream=None) -> None:
        g = self.g
        if self.fused:
            fva_reorder_pool(q, self.qr, self.qbar, g, stream)
            fva_reorder_pool(k, self.kr, self.kbar, g, stream)
        else:
            fva_reorder(q, self.qr, g, stream)
            fva_reorder(k, self.kr, g, stream)
        fva_reorder(v, self.vr, g, stream)

    def __call__(self, q, k, v, out, stream=None) -> torch.Tensor:
        g = self.g
        self.reorder_qkv(q, k, v, stream)
        self.routing(stream)
        if self.fused:
            self.attention_natural(out, stream)
        else:
            self.attention(stream)
            fva_inverse_reorder(self.outr, out, g, stream)
        return out


class HostPipeline:
    """The whole path over batches held in pinned host memory, with the copies hidden
    under the kernels: the host->device copy of batch s+1 and the device->host copy of
    batch s-1 run while batch s computes.

    Two device input sets and two device outputs alternate between batches, on three
    streams: copy-in, compute (the path's kernels in order) and copy-out.  Only the
    reorder pass reads an input set (everything after it reads the tile-major copies),
    so a set may be overwritten once its reorder has run; an output may be overwritten
    once its copy-out has run.  Events carry exactly those two hazards plus the two
    data dependencies (copy-in before reorder, attention before copy-out).

    `submit` enqueues one batch and returns an event recorded after its copy-out; the
    host tensors must stay alive and unmodified until that event completes.
    """

    def __init__(self, path: SparseAttention, compute_stream=None):
        g = path.g
        dev = path.qr.device
        shp = (g.B, g.H, g.N, g.d)
        self.path = path
        self.compute = compute_stream if compute_stream is not None else torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.inputs = [tuple(torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(3)) for _ in range(2)]
        self.outputs = [torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.in_free = [None, None]    # reorder of the set's last batch has run
        self.out_free = [None, None]   # copy-out of the output's last batch has run
        self.count = 0

    def submit(self, qh: torch.Tensor, kh: torch.Tensor, vh: torch.Tensor, outh: torch.Tensor) -> torch.cuda.Event:
        j = self.count % 2
        ins, out = self.inputs[j], self.outputs[j]
        for h, name in ((qh, "q"), (kh, "k"), (vh, "v"), (outh, "out")):
            if h.dtype != torch.bfloat16 or tuple(h.shape) != tuple(out.shape):
                raise ValueError(f"{name}: expected bf16 of shape {tuple(out.shape)}, got {h.dtype} {tuple(h.shape)}")
            if h.is_cuda or not h.is_pinned() or not h.is_contiguous():
                raise ValueError(f"{name}: must be a contiguous pinned host tensor")
        if self.in_free[j] is not None:
            self.copy_in.wait_event(self.in_free[j])
        with torch.cuda.stream(self.copy_in):
            for d, h in zip(ins, (qh, kh, vh)):
                d.copy_(h, non_blocking=True)
        in_ready = torch.cuda.Event()
        in_ready.record(self.copy_in)

        self.compute.wait_event(in_ready)
        self.path.reorder_qkv(*ins, self.compute)
        self.in_free[j] = torch.cuda.Event()
        self.in_free[j].record(self.compute)
        self.path.routing(self.compute)
        if self.out_free[j] is not None:
            self.compute.wait_event(self.out_free[j])
        self.path.attention_natural(out, self.compute)
        out_ready = torch.cuda.Event()
        out_ready.record(self.compute)

        self.copy_out.wait_event(out_ready)
        with torch.cuda.stream(self.copy_out):
            outh.copy_(out, non_blocking=True)
        self.out_free[j] = torch.cuda.Event()
        self.out_free[j].record(self.copy_out)
        self.count += 1
        return self.out_free[j]

    def join(self, stream=None) -> None:
        """Make `stream` (default: the compute stream) wait for every enqueued copy-out."""
        s = self.compute if stream is None else stream
        for e in self.out_free:
            if e is not None:
                s.wait_event(e)
