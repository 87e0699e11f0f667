"""Benchmark of the adaptive block-sparse attention path on B200.

One step = one pass of the whole path over one Wan-like attention layer held in
HBM: reorder(Q, K with pooling; V) -> route + repair from the pooled means ->
block-sparse attention writing the output in natural order (6 launches).  `value`
is the step's throughput in actual (sparse) attention TFLOP/s; the JSON line also
carries the dense-equivalent rate, the routing GB/s (standalone and together with
the reorder), the attention kernel's roofline fraction, an end-to-end figure through
host buffers (HostPipeline, the copies overlapped with the kernels; the serial
copy-compute-copy figure beside it), the clocks seen while timing, and the CPU oracle
timed on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan720p] [--impl reference]
                    [--tile-order raster|hilbert] [--static-order] [--no-side-configs]
                    [--report stress|sweep|sasa|route [--tile64]]

At the default wan720p layer (1 GPU) the line also carries `side_configs`: the
head-heterogeneity stress layer and the same layer with 64-token tiles, measured
briefly after the headline timing.

Multi-GPU (torchrun): every rank runs its own replica of the layer (weak scaling,
no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_CONFIG = "wan720p"
# value = actual (kept-pair) attention TFLOP/s of the whole path; the dense-equivalent
# rate, the fraction of the bf16 peak and the routing GB/s are further keys of the line
METRIC = "block-sparse attn TFLOPS (actual & dense-equiv) + % bf16 peak; routing GB/s, 1\u00d7B200"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--impl", default="fva", choices=["fva", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tile-order", choices=("raster", "hilbert"), default="raster",
                    help="tile numbering: raster, or along the 3D Hilbert curve")
    ap.add_argument("--static-order", action="store_true", help="item-id order instead of the LPT work list")
    ap.add_argument("--tile64", action="store_true",
                    help="the --config layer with 1x8x8 tiles (64-token blocks), for the headline line or --report route")
    ap.add_argument("--no-side-configs", action="store_true",
                    help="skip the stress720p and 64-token-tile keys of the headline line")
    ap.add_argument("--report", choices=["stress", "sweep", "sasa", "route"], default=None,
                    help="instead of the headline line: head-heterogeneity stress (LPT vs item-id order) or the "
                         "p x tile sweep at 720p scale, one JSON line per measurement")
    return ap.parse_args(argv)


def workload_desc(cfg) -> dict:
    return {
        "workload": f"{cfg.name}: single attention layer, B={cfg.B}, H={cfg.H}, head_dim={cfg.d}, "
                    f"latent {cfg.T}x{cfg.Y}x{cfg.X}={cfg.N} tokens, tiles {cfg.tt}x{cfg.ty}x{cfg.tx}={cfg.S} "
                    f"({cfg.Nb} blocks), p={cfg.p}, k={cfg.k}",
        "B": cfg.B, "H": cfg.H, "head_dim": cfg.d, "tokens": cfg.N, "tile": cfg.S, "blocks": cfg.Nb,
        "p": cfg.p, "k": cfg.k, "generator": f"random Fourier features sigma={cfg.sigma}, a_h {cfg.a_mode} "
                                             f"[{cfg.a_lo}, {cfg.a_hi}], noise std {cfg.noise_std:.3g}, seed {cfg.seed}",
        "l2": f"inputs larger than L2 ({cfg.B * cfg.H * cfg.N * cfg.d * 2 / 1e6:.0f} MB per Q/K/V tensor)",
    }


DATA = "synthetic (seeded random-Fourier-feature Q/K, Gaussian V; stands in for Wan2.2 latents)"


def arm_config(cfg, args, world: int) -> dict:
    """The `config` object of the JSON line, the same for the GPU arm and the reference arm."""
    return dict(workload_desc(cfg), parallelism=f"replicas x{world} (no data-path collective)",
                order="static" if args.static_order else "lpt", tiles=args.tile_order)


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def attn_source_hash() -> str:
    """Hash of the attention kernel's code (attn.cu + fva_common.cuh) with // comments and
    blank lines removed, so that only a change of the code itself invalidates a capture."""
    h = hashlib.sha256()
    for f in ("attn.cu", "fva_common.cuh"):
        text = open(os.path.join(ROOT, "block_sparse_attention_44_b200", "csrc", f), encoding="utf-8").read()
        for line in text.splitlines():
            code = re.sub(r"//.*$", "", line).rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:12]


def attn_traffic(cfg_name: str, launches_units: float):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the
    current attention source; scaled by processed block pairs when captured on a smaller case."""
    p = os.path.join(ROOT, "profiles", "attn_dram_traffic.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"source_hash:\s*([0-9a-f]+)", txt)
    b = re.search(r"dram_bytes_per_block_pair:\s*([0-9.eE+]+)", txt)
    if not m or not b or m.group(1) != attn_source_hash():
        return None
    return float(b.group(1)) * launches_units


# ------------------------------------------------------------------ clocks ---------
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 10 ms while active."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []
        self.stop = threading.Event()
        self.nv = None

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.nv = None
        return self

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), int(get_reasons(self.h))))
            except Exception:
                pass
            self.stop.wait(0.01)

    def __exit__(self, *a):
        self.stop.set()
        if self.nv is not None:
            self.t.join(timeout=2)
            try:
                self.nv.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if self.nv is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for name, attr in self.REASONS.items():
                if r & getattr(self.nv, attr, 0):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "NVML, 10 ms period"}


# ------------------------------------------------------------------ CPU oracle ---------
def oracle_sample(cfg, qkv, budget_s: float = 10.0):
    """The oracle, as it stands, on a bounded sample of the workload: heads in order, each
    reordered, routed and repaired, then masked float64 attention query block by query
    block, until the time budget is spent.  Returns (TFLOP/s, seconds, description)."""
    import oracle as O
    og = O.Geometry.of(cfg.with_(H=1))
    q, k, v = qkv
    flops = 0.0
    heads = items = 0
    t0 = time.perf_counter()
    for h in range(cfg.H):
        qr, kr, vr = (O.reorder(t[:1, h:h + 1], og) for t in (q, k, v))
        rr = O.route(qr, kr, og, cfg.p, cfg.k)
        rp = O.repair(rr.topp_mask, rr.topk_idx)
        heads += 1
        for i in range(og.Nb):
            O.attention_items(qr, kr, vr, rp.counts, rp.idx, og.S, [(0, 0, i)])
            flops += 4.0 * og.S * og.S * og.d * float(rp.counts[0, 0, i])
            items += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"{cfg.name} batch 0: {heads} of {cfg.H} heads reordered, routed and repaired by the oracle, then "
            f"float64 masked attention for {items} query blocks ({og.Nb} per head) in head order; throughput = "
            f"sparse attention FLOPs executed / wall time")
    return flops / dt / 1e12, dt, desc


def cpu_cores() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def arm_cfg(args):
    """The --config layer, with 1x8x8 tiles when --tile64 is given."""
    cfg = synth.CONFIGS[args.config]
    return cfg.with_(name=cfg.name + "_tile64", tt=1) if args.tile64 else cfg


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    cfg = arm_cfg(args)
    qkv = synth.make_qkv(cfg)
    vals, secs = [], []
    desc = ""
    for s in range(args.warmup + args.steps):
        v, dt, desc = oracle_sample(cfg, qkv, budget_s=1.5)
        if s >= args.warmup:
            vals.append(v)
            secs.append(dt)
    value = statistics.median(vals)
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": DATA, "config": arm_config(cfg, args, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks ------------
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (every rank calls it; world 1: x itself).
    Multi-rank times are taken this way: the job takes as long as its slowest rank."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Aggregate throughput of `world` replicas that each process units_per_rank in `ms`
    (the max over ranks): weak scaling, units per second over the whole job."""
    return world * units_per_rank / (ms * 1e-3)


# ------------------------------------------------------------------ GPU arm ----------
def run_gpu(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    import block_sparse_attention_44_b200 as fva

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = arm_cfg(args)
    g = fva.Geom.of(cfg)
    if args.tile_order == "hilbert":
        g = g.with_tiles(fva.FVA_TILES_HILBERT, device=dev)
    peaks = load_peaks()

    q, k, v = synth.make_qkv(cfg)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cv, dt, desc = oracle_sample(cfg, (q, k, v), budget_s=10.0)
        cpu = {"value": cv, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc,
               "seconds": round(dt, 2)}
    def host_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    qh, kh, vh = (host_bf16(a).pin_memory() for a in (q, k, v))
    del q, k, v
    qd, kd, vd = (t.to(dev) for t in (qh, kh, vh))
    out = torch.empty_like(qd)
    outh = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    path = fva.SparseAttention(g, cfg.p, cfg.k, device=dev, use_lpt=not args.static_order)
    stream = torch.cuda.current_stream(dev)

    def step():
        path(qd, kd, vd, out, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert fva.fva_get_device_error(stream) == 0

    counts = path.rep.counts
    pairs = int(counts.sum().item())
    flops_actual = 4.0 * g.S * g.S * g.d * pairs
    flops_dense = 4.0 * g.B * g.H * float(g.N) ** 2 * g.d
    density = pairs / float(g.B * g.H * g.Nb * g.Nb)

    # --- timed region: K whole steps; per-stage events on the launching stream
    K = args.steps
    E = lambda: torch.cuda.Event(enable_timing=True)
    ev = [[E() for _ in range(4)] for _ in range(K)]
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = fva.fva_launch_count()
    with ClockSampler(gpu_id) as clk:
        start, stop = E(), E()
        start.record(stream)
        for s in range(K):
            e = ev[s]
            e[0].record(stream)
            path.reorder_qkv(qd, kd, vd, stream)  # Q and K pooled by their reorder pass
            e[1].record(stream)
            path.routing(stream)                  # fva_route_repair_pooled: select + repair + LPT list
            e[2].record(stream)
            path.attention_natural(out, stream)   # attention, output written in natural order
            e[3].record(stream)
        stop.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    launches = fva.fva_launch_count() - launches0
    assert fva.fva_get_device_error(stream) == 0
    total_ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    ms = total_ms / K
    stage = np.array([[ev[s][i].elapsed_time(ev[s][i + 1]) for i in range(3)] for s in range(K)])
    st_mean = stage.mean(axis=0)            # reorder x3 (+ pooling), routing from the means, attention (ms)
    attn_ms = float(st_mean[2])
    route_ms = float(st_mean[1])

    # routing as one call from reordered Q and K (pooling included): fva_route_repair
    fused_route_ms = _time_ms(lambda: fva.fva_route_repair(path.qr, path.kr, g, cfg.p, cfg.k, path.rep.counts,
                                                           path.rep.idx, path.rep.head_work, path.rep.worklist,
                                                           path.ws, stream=stream), stream, 10)
    # the unfused entry points, timed apart (same inputs): fva_route, then fva_repair
    sep_route_ms = _time_ms(lambda: fva.fva_route(path.qr, path.kr, g, cfg.p, cfg.k, path.route.topp_mask,
                                                  path.route.topk_idx, path.ws, stream=stream), stream, 10)
    sep_repair_ms = _time_ms(lambda: fva.fva_repair(path.route.topp_mask, path.route.topk_idx, g, cfg.k,
                                                    path.rep.counts, path.rep.idx, path.rep.head_work,
                                                    path.rep.worklist, workspace=path.rws, stream=stream),
                             stream, 10)
    path.routing(stream)

    # --- end to end through host buffers: every step copies its Q/K/V in from pinned host
    # memory and its O back out.  HostPipeline (the package's host-batch API) runs batch
    # s+1's copy-in and batch s-1's copy-out under batch s's kernels; the serial loop
    # (copy in, compute, copy out, one after another) is timed beside it.
    h2d = 3 * qh.numel() * 2
    d2h = outh.numel() * 2
    outh2 = [outh, torch.empty_like(outh).pin_memory()]
    pipe = fva.HostPipeline(path, stream)
    for i in range(2):
        pipe.submit(qh, kh, vh, outh2[i % 2])
    pipe.join()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    s0, s1 = E(), E()
    s0.record(stream)
    pipe.copy_in.wait_stream(stream)
    for i in range(K):
        pipe.submit(qh, kh, vh, outh2[i % 2])
    pipe.join()
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / K, world, dev)
    assert fva.fva_get_device_error(stream) == 0
    # the pipelined result is the device-resident step's result, bit for bit
    e2e_same = bool(torch.equal(outh2[(K - 1) % 2].view(torch.int16), out.cpu().view(torch.int16)))

    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    s0, s1 = E(), E()
    s0.record(stream)
    for _ in range(K):
        qd.copy_(qh, non_blocking=True)
        kd.copy_(kh, non_blocking=True)
        vd.copy_(vh, non_blocking=True)
        step()
        outh.copy_(out, non_blocking=True)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    serial_ms = max_over_ranks(s0.elapsed_time(s1) / K, world, dev)

    if rank != 0:
        return
    bytes_route = 2.0 * g.B * g.H * g.N * g.d * 2          # Qr and Kr read once (pooling)
    bytes_reorder = 3 * 2.0 * g.B * g.H * g.N * g.d * 2    # Q, K, V read + write
    achieved = flops_actual / (attn_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]          # burst: the kernel runs for tens of ms per step
    traffic = attn_traffic(cfg.name, pairs)
    value = whole_job_rate(world, flops_actual, ms) / 1e12
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": DATA,
        "config": arm_config(cfg, args, world),
        "dense_equiv_tflops": whole_job_rate(world, flops_dense, ms) / 1e12,
        "attn_pct_bf16_peak": 100.0 * achieved / peak,
        "attn_pct_bf16_peak_sustained": 100.0 * achieved / peaks["bf16_tflops_sustained"],
        "attn_kernel_tflops": achieved,
        "attn_kernel_dense_equiv_tflops": flops_dense / (attn_ms * 1e-3) / 1e12,
        "density": density,
        "routing_gbs": bytes_route / (fused_route_ms * 1e-3) / 1e9,
        "routing_frac_hbm": bytes_route / (fused_route_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "reorder_routing_gbs": (bytes_reorder + 4 * g.B * g.H * g.Nb * g.d * 8) / ((st_mean[0] + route_ms) * 1e-3) / 1e9,
        "reorder_routing_frac_hbm": (bytes_reorder + 4 * g.B * g.H * g.Nb * g.d * 8) / ((st_mean[0] + route_ms) * 1e-3)
                                    / 1e9 / peaks["hbm_gbs"],
        "reorder_gbs": bytes_reorder / (st_mean[0] * 1e-3) / 1e9,
        "routing_overhead_pct": 100.0 * route_ms / attn_ms,
        "stage_ms": {"reorder_qkv_pool": st_mean[0], "route_repair_from_pooled": st_mean[1],
                     "attention_natural_out": st_mean[2], "route_repair_fused": fused_route_ms,
                     "route_unfused": sep_route_ms, "repair_unfused": sep_repair_ms},
        "routing_unfused_gbs": bytes_route / ((sep_route_ms + sep_repair_ms) * 1e-3) / 1e9,
        "roofline": {"bound": "tensor", "kernel": "attn_kernel (fva_block_sparse_attn)", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_src": f"{peaks['src']} bf16 burst (cuBLAS 8192^3, best of 10)",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "attn_ms_per_launch": attn_ms,
                     "traffic": traffic,
                     "algorithmic_units": f"{pairs} kept block pairs x {4 * g.S * g.S * g.d} FLOP"},
        "routing_roofline": {"bound": "hbm", "call": "fva_route_repair (pool + select + LPT)",
                             "achieved": bytes_route / (fused_route_ms * 1e-3) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": bytes_route / (fused_route_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "e2e": {"value": whole_job_rate(world, flops_actual, e2e_ms) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "api": "HostPipeline (copies overlapped)",
                "matches_device_result": e2e_same, "serial_ms_per_step": serial_ms,
                "serial_value": whole_job_rate(world, flops_actual, serial_ms) / 1e12},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if not args.no_side_configs and world == 1 and cfg.name == "wan720p":
        line["side_configs"] = side_configs(path, qd, kd, vd, dev, stream, peaks)
    print(json.dumps(line), flush=True)


def side_configs(path, qd, kd, vd, dev, stream, peaks, reps=3):
    """Compact measurements of the two other 720p-scale layers, on the same device
    buffers after the headline timing: the head-heterogeneity stress layer (LPT work
    list against item-id order, lambda_SM) and the wan720p layer with 64-token tiles
    (attention and routing rates).  CUDA events, `reps` launches each after one warm-up."""
    import torch
    import block_sparse_attention_44_b200 as fva
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {}

    def layer(cfg, p_obj, extra):
        g = p_obj.g
        p_obj(qd, kd, vd, torch.empty_like(qd), stream)
        torch.cuda.synchronize(dev)
        assert fva.fva_get_device_error(stream) == 0
        counts = p_obj.rep.counts.cpu().numpy().reshape(-1)
        pairs = int(counts.sum())
        flops = 4.0 * g.S * g.S * g.d * pairs
        attn_ms = _time_ms(lambda: p_obj.attention(stream), stream, reps)
        route_ms = _time_ms(lambda: fva.fva_route_repair(p_obj.qr, p_obj.kr, g, cfg.p, cfg.k, p_obj.rep.counts,
                                                         p_obj.rep.idx, p_obj.rep.head_work, p_obj.rep.worklist,
                                                         p_obj.ws, stream=stream), stream, reps)
        rbytes = 2.0 * g.B * g.H * g.N * g.d * 2
        d = {"workload": workload_desc(cfg)["workload"], "density": pairs / float(g.B * g.H * g.Nb * g.Nb),
             "attn_ms": attn_ms, "attn_tflops": flops / (attn_ms * 1e-3) / 1e12,
             "attn_frac_bf16_burst": flops / (attn_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
             "attn_dense_equiv_tflops": 4.0 * g.B * g.H * float(g.N) ** 2 * g.d / (attn_ms * 1e-3) / 1e12,
             "route_repair_ms": route_ms, "routing_gbs": rbytes / (route_ms * 1e-3) / 1e9,
             "routing_frac_hbm": rbytes / (route_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        d.update(extra(p_obj, counts, attn_ms))
        return d

    # head-heterogeneity stress: same grid, alternating sharp / diffuse heads, p = 0.95
    cfg = synth.CONFIGS["stress720p"]
    q, k, v = synth.make_qkv(cfg)
    for dst, a in ((qd, q), (kd, k), (vd, v)):
        dst.copy_(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
    del q, k, v
    sp = fva.SparseAttention(fva.Geom.of(cfg), cfg.p, cfg.k, device=dev)

    def stress_extra(p_obj, counts, lpt_ms):
        wl = p_obj.rep.worklist.cpu().numpy()
        hw = p_obj.rep.head_work.cpu().numpy().reshape(-1)
        g = p_obj.g
        p_obj.use_lpt = False
        static_ms = _time_ms(lambda: p_obj.attention(stream), stream, reps)
        p_obj.use_lpt = True
        return {"static_order_attn_ms": static_ms, "lpt_speedup": static_ms / lpt_ms,
                "lambda_sm_lpt": cta_imbalance(counts, wl, n_sm),
                "lambda_sm_static": cta_imbalance(counts, np.arange(counts.size), n_sm),
                "head_density_even": float(hw[0::2].mean() / (g.Nb * g.Nb)),
                "head_density_odd": float(hw[1::2].mean() / (g.Nb * g.Nb))}
    out["stress720p"] = layer(cfg, sp, stress_extra)
    del sp
    # the wan720p layer again (same generator and seed) with 64-token tiles: 1200 blocks
    cfg = synth.CONFIGS["wan720p"]
    q, k, v = synth.make_qkv(cfg)
    for dst, a in ((qd, q), (kd, k), (vd, v)):
        dst.copy_(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
    del q, k, v
    cfg64 = cfg.with_(name="wan720p_tile64", tt=1)
    tp = fva.SparseAttention(fva.Geom.of(cfg64), cfg64.p, cfg64.k, device=dev)
    out["wan720p_tile64"] = layer(cfg64, tp, lambda *a: {})
    del tp
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ reports ----------
def _time_ms(fn, stream, reps):
    import torch
    E = lambda: torch.cuda.Event(enable_timing=True)
    a, b = E(), E()
    fn()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def cta_imbalance(counts, order, n_cta):
    """lambda_SM = max / mean kept block pairs per CTA when CTAs stride through `order`."""
    per = np.zeros(n_cta)
    for pos, u in enumerate(order):
        per[pos % n_cta] += counts[u]
    return float(per.max() / per.mean())


def run_sasa_report(args):
    """Slack-aware augmentation at 480p: 8 virtual ranks of 5 heads, alpha 0 .. 1."""
    import torch
    import block_sparse_attention_44_b200 as fva
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    cfg = synth.CONFIGS["wan480p"]
    g = fva.Geom.of(cfg)
    q, k, v = synth.make_qkv(cfg)
    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    path = fva.SparseAttention(g, cfg.p, cfg.k, device=dev)
    out = torch.empty_like(qd)
    path(qd, kd, vd, out, stream)
    ws = torch.empty((fva.fva_sasa_workspace_size(g),), dtype=torch.uint8, device=dev)
    ranks = 8
    hpr = g.H // ranks
    base_hw = path.rep.head_work.clone()
    W0 = [int(base_hw[:, r * hpr:(r + 1) * hpr].sum()) for r in range(ranks)]
    for alpha in (0.0, 0.25, 0.5, 1.0):
        run = lambda: fva.fva_route_repair_sasa(path.qbar, path.kbar, g, cfg.p, cfg.k, ranks, alpha, path.rep.counts,
                                                path.rep.idx, path.rep.head_work, path.rep.worklist, ws,
                                                stream=stream)
        route_ms = _time_ms(run, stream, 5)
        torch.cuda.synchronize()
        assert fva.fva_get_device_error(stream) == 0
        pairs = int(path.rep.counts.sum().item())
        W1 = [int(path.rep.head_work[:, r * hpr:(r + 1) * hpr].sum()) for r in range(ranks)]
        attn_ms = _time_ms(lambda: path.attention_natural(out, stream), stream, 3)
        line = {"report": "sasa", "workload": cfg.name, "virtual_ranks": ranks, "alpha": alpha,
                "density": pairs / float(g.B * g.H * g.Nb * g.Nb), "pairs_added": pairs - sum(W0),
                "rank_work_max_over_mean_before": max(W0) / (sum(W0) / ranks),
                "rank_work_max_over_mean_after": max(W1) / (sum(W1) / ranks),
                "critical_rank_work": [max(W0), max(W1)],
                "route_sasa_ms": route_ms, "attn_ms": attn_ms,
                "attn_tflops": 4.0 * g.S * g.S * g.d * pairs / (attn_ms * 1e-3) / 1e12}
        print(json.dumps(line), flush=True)


def run_route_report(args, reps=5):
    """Routing calls alone at --config (tile 1x8x8 when the name ends in _tile64): the
    standalone fva_route_repair from reordered Q and K, its unfused pair and the routing
    from pooled means, each timed with CUDA events over `reps` calls after one warm-up."""
    import torch
    import block_sparse_attention_44_b200 as fva
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()
    name = args.config
    cfg = synth.CONFIGS[name]
    if getattr(args, "tile64", False):
        cfg = cfg.with_(name=name + "_tile64", tt=1)
    g = fva.Geom.of(cfg)
    q, k, v = synth.make_qkv(cfg)
    del v
    qd, kd = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (q, k))
    del q, k
    path = fva.SparseAttention(g, cfg.p, cfg.k, device=dev)
    fva.fva_reorder_pool(qd, path.qr, path.qbar, g, stream)
    fva.fva_reorder_pool(kd, path.kr, path.kbar, g, stream)
    torch.cuda.synchronize()
    rbytes = 2.0 * g.B * g.H * g.N * g.d * 2
    calls = {
        "route_repair": lambda: fva.fva_route_repair(path.qr, path.kr, g, cfg.p, cfg.k, path.rep.counts, path.rep.idx,
                                                     path.rep.head_work, path.rep.worklist, path.ws, stream=stream),
        "route": lambda: fva.fva_route(path.qr, path.kr, g, cfg.p, cfg.k, path.route.topp_mask, path.route.topk_idx,
                                       path.ws, stream=stream),
        "repair": lambda: fva.fva_repair(path.route.topp_mask, path.route.topk_idx, g, cfg.k, path.rep.counts,
                                         path.rep.idx, path.rep.head_work, path.rep.worklist, workspace=path.rws,
                                         stream=stream),
        "route_repair_pooled": lambda: path.routing(stream),
    }
    line = {"report": "route", "workload": workload_desc(cfg)["workload"], "reps": reps}
    for key, fn in calls.items():
        line[key + "_ms"] = _time_ms(fn, stream, reps)
    assert fva.fva_get_device_error(stream) == 0
    line["routing_gbs"] = rbytes / (line["route_repair_ms"] * 1e-3) / 1e9
    line["routing_frac_hbm"] = line["routing_gbs"] / peaks["hbm_gbs"]
    line["density"] = float(path.rep.counts.sum().item()) / (g.B * g.H * g.Nb * g.Nb)
    print(json.dumps(line), flush=True)


def run_report(args):
    import torch
    import block_sparse_attention_44_b200 as fva
    if args.report == "sasa":
        run_sasa_report(args)
        return
    if args.report == "route":
        run_route_report(args)
        return
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks = load_peaks()
    base = synth.CONFIGS["stress720p" if args.report == "stress" else "wan720p"]
    q, k, v = synth.make_qkv(base)
    def host_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    qd, kd, vd = host_bf16(q), host_bf16(k), host_bf16(v)
    del q, k, v
    if args.report == "stress":
        cases = [base]
    else:
        cases = [c for c in synth.sweep_configs()]
    for cfg in cases:
        g = fva.Geom.of(cfg)
        path = fva.SparseAttention(g, cfg.p, cfg.k, device=dev)
        out = torch.empty_like(qd)
        path(qd, kd, vd, out, stream)
        torch.cuda.synchronize()
        assert fva.fva_get_device_error(stream) == 0
        counts = path.rep.counts.cpu().numpy().reshape(-1)
        pairs = int(counts.sum())
        flops = 4.0 * g.S * g.S * g.d * pairs
        dense = 4.0 * g.B * g.H * float(g.N) ** 2 * g.d
        route_ms = _time_ms(lambda: fva.fva_route_repair(path.qr, path.kr, g, cfg.p, cfg.k, path.rep.counts,
                                                         path.rep.idx, path.rep.head_work, path.rep.worklist,
                                                         path.ws, stream=stream), stream, 5)
        path.use_lpt = True
        lpt_ms = _time_ms(lambda: path.attention(stream), stream, 5)
        line = {"report": args.report, "workload": cfg.name, "tile": g.S, "blocks": g.Nb, "p": cfg.p, "k": cfg.k,
                "density": pairs / float(g.B * g.H * g.Nb * g.Nb),
                "attn_ms": lpt_ms, "attn_tflops": flops / (lpt_ms * 1e-3) / 1e12,
                "attn_dense_equiv_tflops": dense / (lpt_ms * 1e-3) / 1e12,
                "attn_frac_bf16_burst": flops / (lpt_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "route_repair_ms": route_ms, "routing_gbs": 2.0 * g.B * g.H * g.N * g.d * 2 / (route_ms * 1e-3) / 1e9,
                "routing_overhead_pct": 100.0 * route_ms / lpt_ms}
        if args.report == "stress":
            wl = path.rep.worklist.cpu().numpy()
            hw = path.rep.head_work.cpu().numpy().reshape(-1)
            path.use_lpt = False
            static_ms = _time_ms(lambda: path.attention(stream), stream, 5)
            path.use_lpt = True
            line.update({"static_order_attn_ms": static_ms, "lpt_speedup": static_ms / lpt_ms,
                         "lambda_sm_lpt": cta_imbalance(counts, wl, n_sm),
                         "lambda_sm_static": cta_imbalance(counts, np.arange(counts.size), n_sm),
                         "head_density_even": float(hw[0::2].mean() / (g.Nb * g.Nb)),
                         "head_density_odd": float(hw[1::2].mean() / (g.Nb * g.Nb))})
        print(json.dumps(line), flush=True)
        del path, out
        torch.cuda.empty_cache()


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.report:
        run_report(args)
        return
    import torch
    import torch.distributed as dist
    import datetime
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
