"""bench.py's multi-rank plumbing on CPU: two gloo ranks, no GPU.

One process per GPU is the launch model (torchrun); with no GPU the same helpers
fall back to gloo, so the barrier, the max-over-ranks timing reduction and the
rank-0-only reporting of the reference arm are exercised here.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.dist_init(world)
    assert dist.get_backend() == "gloo"
    bench.barrier(world)
    slowest = bench.max_over_ranks(1.5 + rank, world)       # each rank's "device time"
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": slowest}, f)
    bench.barrier(world)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_barrier_gloo(tmp_path):
    world = 2
    torch.multiprocessing.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                                          start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json"))["max"] for r in range(world)]
    assert got == [2.5, 2.5]


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.dist_init(1) is None


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_two_ranks():
    # rank 0 alone times the oracle and prints one JSON line; rank 1 exits 0 without work
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
