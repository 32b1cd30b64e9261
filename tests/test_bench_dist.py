"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on
the slowest rank's time and on the whole-job value, and the reference arm
runs on rank 0 only (the other ranks exit 0 without output)."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 1.0 + rank * 0.5          # rank 1 is the slow one
        ms = bench.max_over_ranks(my_ms)  # CPU tensor for gloo
        dist.barrier()
        q.put((rank, ms, bench.whole_job_tops(2.0e12, world, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 1.5                              # max over ranks
        assert abs(value - 2 * 2.0e12 / 1.5e-3 / 1e12) < 1e-9  # both batches / slowest time


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_tops(1e12, 1, 1.0) == 1000.0


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line_on_rank_zero():
    """The reference arm (the oracle on the host cores) prints exactly one JSON
    line with the keys the bench contract asks of it."""
    import json
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--ref-rows", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_profiled_traffic_only_for_unchanged_kernel_sources():
    import hashlib
    import bench
    root = os.path.dirname(os.path.abspath(bench.__file__))
    h = hashlib.sha256()
    for f in bench.TC2_TRAFFIC["sources"]:
        with open(os.path.join(root, f), "rb") as fh:
            h.update(fh.read())
    current = dict(bench.TC2_TRAFFIC, sources_sha256=h.hexdigest())
    assert bench.profiled_traffic(current) == current["bytes"]
    stale = dict(current, sources_sha256="0" * 64)
    assert bench.profiled_traffic(stale) is None
    missing = dict(current, sources=["no/such/file.cu"])
    assert bench.profiled_traffic(missing) is None
