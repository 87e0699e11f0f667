"""The multi-rank host logic of bench.py on CPU, world size 2: the max-over-ranks time
reduction and whole-job rate over gloo, and the reference arm under torchrun (rank 0
alone works and prints one JSON line, the other rank exits 0 without work).  The GPU
replicas share no data, so these are the only cross-rank steps."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world)     # ranks took 10 ms and 15 ms
        rate = bench.whole_job_rate(world, 1.0e6, slowest)
        dist.barrier()
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; the rate counts both ranks' units over it
    assert [g[1] for g in got] == [15.0, 15.0]
    assert all(abs(g[2] - 2 * 1.0e6 / 15.0e-3) < 1e-3 for g in got)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.whole_job_rate(1, 100.0, 2.0) == 100.0 / 2.0e-3


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 1 and d["warmup"] == 1 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["cores"] >= 1
    # the same metric, unit, direction, data and config object as the GPU arm prints
    sys.path.insert(0, ROOT)
    import bench
    args = bench.parse(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "1"])
    cfg = bench.synth.CONFIGS[args.config]
    assert d["config"] == json.loads(json.dumps(bench.arm_config(cfg, args, 2)))
    assert (d["metric"], d["unit"], d["higher_is_better"], d["data"]) == (bench.METRIC, "TFLOP/s", True, bench.DATA)
