"""The bench's multi-process plumbing (one process per GPU, replicas only) run as two
gloo ranks on CPU: barrier, max-over-ranks device time, whole-job aggregate, and the
reference arm printing on rank 0 only."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "CUDA_VISIBLE_DEVICES": ""})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    assert (w, r) == (world, rank) and bench.dist_backend() == "gloo"
    bench.barrier(w)
    ms = [1.5, 4.0][rank]                     # each rank's own device time
    mx = bench.max_over_ranks(ms, w)
    rate = bench.aggregate_rate(w, 1e9, mx)   # 1e9 units per rank per step
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": mx, "rate": rate}, f)
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_aggregate(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 4.0                   # the slowest rank sets the job's step time
        assert r["rate"] == pytest.approx(2 * 1e9 / 4.0e-3)  # both ranks' units over that time


def test_reference_arm_prints_on_rank0_only(tmp_path):
    """Under torchrun the reference arm runs on rank 0 and the other ranks exit 0 silently."""
    import subprocess
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "dense_512", "--oracle-gflop", "0.02"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0 and p.stdout.strip() == ""
    env["RANK"], env["LOCAL_RANK"] = "0", "0"
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "dense_512", "--oracle-gflop", "0.02"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["cpu_baseline"]["kind"] == "oracle"
