"""bench.py's multi-process path on the CPU (world size 2, gloo): the
barrier / max-over-ranks helpers every rank's timing goes through, and the
reference arm under torchrun (rank 0 alone runs and prints one line)."""
import json
import os
import random
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.dist_helpers(world, torch.device("cpu"))
        barrier()
        got = max_over_ranks(0.25 + rank)  # each rank's own "time"
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr(got))
        barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    port = random.randint(20000, 40000)
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert float(open(tmp_path / f"rank{r}.txt").read()) == 1.25


def test_single_rank_helpers_are_no_ops():
    barrier, max_over_ranks = bench.dist_helpers(1, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.5) == 3.5


def test_reference_arm_under_torchrun_two_ranks():
    port = random.randint(20000, 40000)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2
    assert out["config"] == bench.step_config(out["config"]["workload"], 2)
    assert out["value"] > 0 and out["e2e"]["value"] == out["value"]
    assert out["cpu_baseline"]["kind"] == "oracle"
