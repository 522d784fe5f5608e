"""The multi-process path of bench.py on CPU: two gloo ranks run the rank setup,
barrier and aggregation the benchmark uses for N GPU replicas (total tokens over
ranks / slowest rank's time)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "FT_BENCH_BACKEND": "gloo"})
    import bench
    import torch.distributed as dist
    r, w, lr = bench.dist_setup(world)
    bench.barrier()
    tokens, secs = bench.aggregate(100 * (r + 1), 0.5 + r, None)
    # the host-memory decision is taken by all ranks together: one short rank stops both
    stop = bench.agree_any(r == 1, None)
    go = bench.agree_any(False, None)
    q.put((r, w, lr, tokens, secs, stop, go))
    dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, local, tokens, secs, stop, go) in enumerate(res):
        assert (rank, world, local) == (r, 2, r)
        assert tokens == 300.0 and secs == 1.5      # sum of tokens, max of times
        assert stop is True and go is False


def test_host_memory_guard_for_replicas():
    # N replicas on a node pin N copies of the expert pool; the bench stops before
    # allocating when the node's available memory cannot hold them
    sys.path.insert(0, ROOT)
    import bench
    with open("/proc/meminfo") as f:
        avail = next(int(l.split()[1]) * 1024 for l in f if l.startswith("MemAvailable:"))
    assert bench.host_memory_short(1 << 20, 2) is None
    why = bench.host_memory_short(avail, 2)
    assert why is not None and "2 replicas" in why
    assert bench.agree_any(True) is True and bench.agree_any(False) is False


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(7, 2.5) == (7, 2.5)


def test_reference_arm_json_line():
    # the reference arm times the CPU oracle and prints the contract's JSON line (no GPU)
    import json
    import subprocess
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--reference-budget-s", "5"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # the same config dict as the GPU arm's line, so the two lines describe one workload
    sys.path.insert(0, ROOT)
    import bench
    assert line["config"] == bench.headline_config(1)
    # a rank other than 0 exits at once without a line
    env1 = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3"], cwd=ROOT, env=env1, capture_output=True, text=True, timeout=120)
    assert out1.returncode == 0 and out1.stdout.strip() == ""


def test_traffic_ratio_only_while_the_sources_hash_the_same(tmp_path):
    # the bench reports an ncu traffic figure for a kernel only while its sources hash to the
    # value recorded with the capture; any edit turns it into null with the current hash
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    rel = os.path.relpath(str(src), ROOT)
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    bench.TRAFFIC["_probe"] = {"sources": [rel], "sha256": sha, "ratio": 1.25, "capture": "probe capture"}
    try:
        assert bench.kernel_traffic("_probe", 100.0) == (125.0, "probe capture")
        src.write_text("kernel v2\n")
        traffic, why = bench.kernel_traffic("_probe", 100.0)
        assert traffic is None and hashlib.sha256(src.read_bytes()).hexdigest()[:12] in why
    finally:
        del bench.TRAFFIC["_probe"]
    for key in bench.TRAFFIC:      # every recorded figure names its capture and its sources exist
        t = bench.TRAFFIC[key]
        assert t["capture"] and all(os.path.exists(os.path.join(ROOT, r)) for r in t["sources"])
