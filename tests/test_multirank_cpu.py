"""The N>1 path of the benchmark on CPU: two ``gloo`` ranks.

Every rank runs an independent replica of the layer (no exchange between
GPUs), the timed region is bracketed by a barrier, and the reported time is
the maximum over ranks.  These tests run that plumbing as two real processes
on the host: the max-over-ranks reduction, the whole-job throughput it feeds,
per-rank synthetic inputs, and the reference arm under torchrun (rank 0
prints one JSON line, every other rank exits 0 without work).
"""

from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank elapsed times: rank 1 is the slow one
        mine = [3.25, 7.5][rank]
        dist.barrier()
        slowest = bench.max_over_ranks(mine, world, torch.device("cpu"))
        rate = bench.whole_job_rate(bench.weight_bytes(17408, 5120), world, 10, slowest)
        # each rank draws its own activations from the seeded generator
        bits, _, _ = synth.activations(1, 256, synth.rng_for(1, rank, "act"), 3)
        digest = int(torch.as_tensor(bits.astype("int64")).sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "rate": rate, "digests": gathered}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_whole_job_rate(tmp_path):
    import torch.multiprocessing as mp

    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn",
                       join=True)
    import bench
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r in res:
        assert r["slowest"] == 7.5
        # two replicas, 10 steps each, timed by the slower rank
        expect = 2 * bench.weight_bytes(17408, 5120) * 10 / 7.5e-3 / 1e9
        assert r["rate"] == pytest.approx(expect, rel=1e-12)
    # both ranks see the same gathered list, and the replicas' inputs differ
    assert res[0]["digests"] == res[1]["digests"]
    assert res[0]["digests"][0] != res[0]["digests"][1]


def test_max_over_ranks_alone_is_identity():
    import bench
    assert bench.max_over_ranks(4.5, 1, None) == 4.5
    assert bench.whole_job_rate(1e9, 1, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--ref-seconds", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 2 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
