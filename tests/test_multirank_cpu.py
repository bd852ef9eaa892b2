"""World-size-2 checks of the benchmark's multi-rank host logic on CPU (gloo):
max-over-ranks timing, the barrier, and that the reference arm runs on rank 0
only.  No GPU, no collective on any data path."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        bench.barrier(world)
        t = bench.max_over_ranks(1.5 + rank, world)  # rank 1 is the slow one
        # the same collective sequence on every rank, twice
        t2 = bench.max_over_ranks(10.0 - rank, world)
        results[rank] = (t, t2)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    port = free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: (2.5, 10.0), 1: (2.5, 10.0)}


def _reference_worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import contextlib
    import io
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
                    "--reference-seconds", "2", "--gpus", str(world)])
    results[rank] = buf.getvalue()


def test_reference_arm_prints_on_rank0_only():
    world = 2
    port = free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_reference_worker, args=(world, port, results), nprocs=world, join=True)
        import json
        line = json.loads(results[0].strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
        assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
        assert line["e2e"]["h2d_bytes_per_step"] == 0
        assert results[1] == ""


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)


def test_bench_launches_its_own_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself
    (torch.distributed.run on 127.0.0.1); here through the reference arm, which
    needs no GPU: rank 0 prints the one JSON line, with n_gpus = 2."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3", "--reference-seconds", "2"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["impl"] == "reference"


def test_bench_rejects_a_world_size_that_differs_from_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--workload", "tiny", "--gpus", "4"])
