"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): process-group setup, the
barrier, the max-over-ranks timing, and the reference arm, which rank 0 alone runs and prints.

bench.py runs one independent replica per GPU (the hot path does not shard): its only
cross-rank steps are these, so they are what a CPU test can check without a GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    world, r, local = bench.dist_setup(None)
    assert (world, r, local) == (2, rank, rank)
    bench.barrier(world)
    m = bench.max_over_ranks(10.0 * (rank + 1), world, "cpu")
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(m))
    bench.barrier(world)
    dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo(tmp_path):
    mp.start_processes(_rank_main, args=(free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    got = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(2)]
    assert got == [20.0, 20.0]


def test_reference_arm_two_ranks_prints_one_line():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--gpus", "2",
           "--impl", "reference", "--workload", "tiny_f32", "--steps", "1", "--warmup", "0", "--ref-budget", "0.2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
