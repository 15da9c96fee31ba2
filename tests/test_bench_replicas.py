"""The N-GPU path of bench.py, on CPU with two gloo ranks: every rank runs its
own batch of the same shape (replicas, weak scaling), the job's time is the
slowest rank's (max over ranks), and the whole-job value counts every rank's
tokens.  The reference arm runs on rank 0 only."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import argparse
    import contextlib
    import io
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank device time: rank 1 is slower
        mine = 10.0 + 5.0 * rank
        out[rank] = bench.reduce_max(mine, "cpu")
        # every rank's batch has the same shape and its own adapters
        wl = workloads.make("decode_q_proj", seed=rank)
        out[world + rank] = float(wl.T)
        out[2 * world + rank] = float(int(wl.adapter_ids.astype(np.int64).sum()))
        # the reference arm prints its line on rank 0 only
        args = argparse.Namespace(workload="tiny", steps=1, warmup=1, cpu_budget=0.05, ref_budget=0.2, weights="bf16")
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args, rank, world, 0)
        out[3 * world + rank] = float(len(buf.getvalue().strip().splitlines()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    """Max over ranks on every rank, same shape and different draws per rank, all
    ranks' tokens over the slowest time, reference line from rank 0 only."""
    world = 2
    out = torch.zeros(4 * world, dtype=torch.float64).share_memory_()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 15.0
    assert out[2] == out[3]
    assert out[4] != out[5]
    assert out[6] == 1.0 and out[7] == 0.0
    v = bench.job_value(world, 32, 100, float(out[0]))
    assert v == pytest.approx(2 * 32 * 100 / 15e-3)


def test_reduce_max_without_process_group_is_identity():
    assert not dist.is_initialized()
    assert bench.reduce_max(3.5, "cpu") == 3.5
