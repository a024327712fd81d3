"""The benchmark's multi-process plumbing on CPU: two gloo ranks run the same
barrier and max-over-ranks steps that bench.py runs under torchrun with NCCL,
and the whole-job value is the work of every rank over the slowest rank's
time.  The path has no data-path collective (independent replicas), so these
two calls are all that crosses ranks."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(backend="gloo", timeout_s=60)
    try:
        d.barrier()
        my_ms = 10.0 + 5.0 * rank                 # rank 1 is the slowest
        worst = d.max(my_ms)
        value = bench.whole_job_tflops(2.0e12, 4, d.world, worst)
        q.put((rank, d.world, worst, value))
        d.barrier()
    finally:
        d.close()


def test_two_gloo_ranks_time_by_the_slowest_rank():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, worst, value in out:
        assert world == 2
        assert worst == 15.0                       # the max over ranks, seen by every rank
        # 2 ranks x 4 steps x 2 TFLOP over 15 ms
        assert value == pytest.approx(2 * 4 * 2.0 / 15e-3)


def test_reference_arm_only_rank0_works():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference on rank 0 of a single-process run prints one
    JSON line with the arm's keys: the oracle timed on the host cores, with
    its own cpu_baseline and an e2e entry that moves no bytes."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert d["steps"] == 1 and d["warmup"] == 0 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["ms_per_step"] > 0
    assert d["config"]["workload"] and d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
