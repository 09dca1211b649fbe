"""The multi-process path of bench.py on the CPU (gloo, world size 2): the
barrier and the max-over-ranks reduction that the timing uses, and the
reference arm launched as the driver launches it (torchrun, one process per
rank), where rank 0 alone runs and prints one JSON line and the other ranks
exit 0 without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(w, "gloo")
    bench.barrier(dist)
    # Each rank's "step time" differs; every rank must see the maximum.
    m = bench.max_over_ranks(dist, 1.5 + 2.0 * rank, torch.device("cpu"))
    bench.barrier(dist)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(m))


def test_barrier_and_max_over_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, free_port(), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        assert float((tmp_path / f"rank{r}.txt").read_text()) == 3.5


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    assert bench.init_dist(1, "gloo") is None
    bench.barrier(None)
    assert bench.max_over_ranks(None, 0.25, torch.device("cpu")) == 0.25


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "2", "--warmup", "3"]
    proc = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=280)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, proc.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2
    assert res["steps"] == 2 and res["warmup"] == 3
    assert res["value"] > 0 and res["unit"] == "GB/s"
    assert res["e2e"]["h2d_bytes_per_step"] == 0
    assert res["cpu_baseline"]["kind"] == "oracle"
