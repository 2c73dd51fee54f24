"""Multi-rank plumbing of bench.py and of the head sharding, on CPU with the
gloo backend (world size 2).

The ISA forward shards by (b, h) with no exchange step, so the multi-GPU
path is one replica of the workload per rank (or one problem's heads split
over the ranks) plus the timing reduction, and, for callers that want the
whole output everywhere, one all-gather of the output heads.  These tests
cover that host logic without a GPU: the max-over-ranks reduction every
rank takes part in, the per-rank replica inputs, the head partition and
its gather, the report's parallelism field, and the reference arm's
rank-0-only output."""
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


def _shard_worker(rank, world, port, out_dir, H=4):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from sparse_attention_context_b200.sharding import gather_heads, shard_heads
    from workloads import CONFIGS, make_inputs, to_torch_bf16

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CONFIGS["tiny"].replace(H=H, N_src=96, N_ctx=64)
        h0, h1 = shard_heads(cfg.H, world, rank)
        local = to_torch_bf16(make_inputs(cfg, seed=0, heads=range(h0, h1))[0])
        full = gather_heads(local)  # stands in for the output slices of the per-rank forwards
        torch.save(full, os.path.join(out_dir, f"full{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H,world", [(4, 2), (7, 3)])
def test_head_shards_gather_to_the_whole_problem(tmp_path, H, world):
    """Each rank draws only its heads of one seeded problem; the gathered
    slices equal the whole problem drawn in one process, on every rank.
    7 heads over 3 ranks gives slices of 3, 2 and 2 heads."""
    import torch

    from workloads import CONFIGS, make_inputs, to_torch_bf16

    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path), H), nprocs=world, join=True,
                       start_method="spawn")
    cfg = CONFIGS["tiny"].replace(H=H, N_src=96, N_ctx=64)
    whole = to_torch_bf16(make_inputs(cfg, seed=0)[0])
    for r in range(world):
        got = torch.load(tmp_path / f"full{r}.pt")
        assert got.shape == whole.shape
        assert torch.equal(got.view(torch.int16), whole.view(torch.int16))


@pytest.mark.parametrize("H,world", [(24, 1), (24, 2), (24, 8), (40, 8), (7, 3), (3, 4)])
def test_shard_heads_partition(H, world):
    from sparse_attention_context_b200.sharding import shard_heads

    ranges = [shard_heads(H, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))  # contiguous, no overlap
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_config_names_the_parallelism():
    import bench
    from workloads import CONFIGS

    cfg = CONFIGS["480p"]
    assert bench.config_dict(cfg, 1)["parallelism"] == "single GPU"
    assert bench.config_dict(cfg, 4)["parallelism"] == "replicas x4"
    assert bench.config_dict(cfg, 4, "heads")["parallelism"] == "heads sharded x4"


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
