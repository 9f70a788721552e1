"""The multi-rank (N > 1) host path of bench.py on the CPU: two gloo ranks, as
torchrun would start them, one process each.  Every rank draws its own batch
(independent problems, weak scaling), the job's time is the slowest rank's, and
the whole-job throughput counts every rank's work.  Sharding the batch across
ranks gives, rank by rank, exactly the per-batch results of the whole batch
(no communication across the batch dimension), checked with the fp64 oracle."""
import contextlib
import io
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from causal_self_attention_gptattn_b200.workloads import WORKLOADS, make_inputs

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import oracle
    g = bench.init_ranks(WORLD, backend="gloo")
    try:
        # the slowest rank sets the job's time
        assert bench.max_over_ranks(g, 1.5 + rank, "cpu") == 2.5
        # each rank's own batch of the small workload (fp32, B=2 per rank)
        w = WORKLOADS[1]
        qkv, dy = make_inputs(w.B, w.T, w.n_head, w.hs, dtype=torch.float32, seed=bench.rank_seed(w, rank))
        y, lse = oracle.forward(qkv, w.n_head)
        shards = [torch.zeros_like(qkv) for _ in range(WORLD)]
        dist.all_gather(shards, qkv)
        ys = [torch.zeros(y.shape, dtype=torch.float64) for _ in range(WORLD)]
        dist.all_gather(ys, torch.from_numpy(y))
        if rank == 0:
            assert not torch.equal(shards[0], shards[1]), "ranks must draw different batches"
            whole_y, _ = oracle.forward(torch.cat(shards, dim=0), w.n_head)
            assert np.array_equal(whole_y, torch.cat(ys, dim=0).numpy())
        dist.barrier()
        open(os.path.join(out_dir, f"rank{rank}.ok"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    assert sorted(os.listdir(tmp_path)) == ["rank0.ok", "rank1.ok"]


def test_whole_job_throughput_counts_every_rank():
    # 2 ranks x 10 steps x 1 TFLOP in 1 s (the slowest rank) = 20 TFLOP/s
    assert bench.aggregate_tflops(2, 10, 1e12, 1000.0) == pytest.approx(20.0)
    assert bench.aggregate_tflops(1, 10, 1e12, 500.0) == pytest.approx(20.0)
    assert bench.max_over_ranks(None, 3.0) == 3.0
    assert bench.init_ranks(1) is None
    w = WORKLOADS[3]
    assert len({bench.rank_seed(w, r) for r in range(8)}) == 8


def test_reference_arm_prints_only_on_rank_0():
    args = types.SimpleNamespace(warmup=0, steps=1, gpus=2)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS[1], rank=1)
    assert buf.getvalue() == ""
