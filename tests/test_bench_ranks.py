"""Multi-rank bookkeeping of bench.py on CPU: two gloo ranks.

The hot path shards by independent sequences (replicas, no data-path
collective), so what a multi-GPU run adds is the timing reduction: every rank
times its own replica, the job takes as long as the slowest rank, and the
whole-job throughput counts every rank's tokens.  These tests run that
reduction over a real process group (gloo, world size 2) without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [12.5, 20.0][rank]  # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, world, "cpu")
        e2e = bench.max_over_ranks([40.0, 30.0][rank], world, "cpu")
        value = bench.job_throughput(65536, ms, world)
        results[rank] = (ms, e2e, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    for rank in range(world):
        ms, e2e, value = got[rank]
        assert ms == 20.0 and e2e == 40.0  # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 65536 / 0.020)  # both replicas' tokens


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.job_throughput(100, 10.0, 1) == pytest.approx(10000.0)


def _bench(args, env_extra):
    import json
    import subprocess

    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_line_on_the_host():
    """--impl reference times the oracle on the host cores (no GPU needed) and
    prints one line with the arm's own metric, cpu_baseline and e2e."""
    args = ["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    (line,) = _bench(args, {"RANK": "0", "WORLD_SIZE": "1"})
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    assert line["higher_is_better"] is True and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # under torchrun only rank 0 runs it: another rank prints nothing and exits 0
    assert _bench(args, {"RANK": "1", "WORLD_SIZE": "2"}) == []
