"""Multi-rank plumbing of bench.py, on CPU with the gloo backend (world size 2).

The ISA forward shards by (b, h) with no exchange step, so the multi-GPU
path is one replica of the workload per rank plus the timing reduction.
These tests cover that host logic without a GPU: the max-over-ranks
reduction every rank takes part in, the per-rank replica inputs, the
report's parallelism field, and the reference arm's rank-0-only output."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from workloads import CONFIGS, make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        local_ms = 1.5 + rank  # rank 1 is the slow one
        got = bench.max_over_ranks(local_ms, "cpu")
        cfg = CONFIGS["tiny"]
        q_bits = make_inputs(cfg, seed=bench.replica_seed(rank))[0]
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"env": [w, r, lr], "max": got, "q_head": q_bits.reshape(-1)[:64].tolist(),
                       "parallelism": bench.config_dict(cfg, w)["parallelism"]}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_timing_and_run_own_replicas(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["env"] == [world, r, r]
        assert d["max"] == pytest.approx(2.5)  # every rank reports the slowest rank's time
        assert d["parallelism"] == "replicas x2"
    assert not np.array_equal(res[0]["q_head"], res[1]["q_head"])  # each replica draws its own inputs


def test_max_over_ranks_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(3.25, "cpu") == 3.25


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "0", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert p.returncode == 0, p.stderr
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    if rank != 0:
        assert lines == []
    else:
        assert len(lines) == 1
        rec = json.loads(lines[0])
        assert rec["impl"] == "reference" and rec["unit"] == "ms" and rec["value"] > 0
        assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
