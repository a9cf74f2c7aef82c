"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

The step partitions into independent parameter groups, so N ranks run N
independent replicas (weak scaling) and the only collectives are the barrier
around the timed region and the max-over-ranks reduction of the timings.
These tests run that plumbing with world_size 2 over gloo, and the reference
arm under torchrun (rank 0 alone works and prints one line).
"""
import json
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


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench.dist_env()
        cpu = torch.device("cpu")
        bench.barrier(ws, cpu)
        # each rank reports its own time; everyone gets the slowest
        mx = bench.max_over_ranks(10.0 + 5.0 * rank, ws, cpu)
        bench.barrier(ws, cpu)
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"ws": ws, "rank": r, "local": local, "max": mx}, f)
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(2)]
    for r, g in enumerate(got):
        assert g == {"ws": 2, "rank": r, "local": r, "max": 15.0}


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    """bench.py --impl reference with two ranks: rank 0 times the oracle and
    prints the one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-sample", "4096"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["steps"] == 1
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


@pytest.mark.parametrize("ws,n,steps,ms", [(1, 1000, 10, 2.0), (4, 6738415616, 50, 1103.0)])
def test_weak_scaling_value_is_whole_job_throughput(ws, n, steps, ms):
    sys.path.insert(0, ROOT)
    import bench
    v = bench.throughput_gparams(ws, n, steps, ms)
    assert abs(v - ws * n * steps / (ms * 1e-3) / 1e9) <= 1e-12 * v
