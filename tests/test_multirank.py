"""The N > 1 path of the benchmark on CPU: two gloo ranks each time their own
batch; the job's step time is the max over ranks and the throughput counts the
units of every rank (weak scaling, no collective on the data path)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from diffusion_transformer_video_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + 5.0 * rank, 30.0 - rank]          # this rank's (step ms, e2e ms)
        step_ms, e2e_ms = bench.max_over_ranks(local, dist, "cpu")
        w = wl.get_workload("tiny")
        x = wl.make_inputs(w, bench.rank_seed(0, rank), which=("x",))["x"]
        q.put((rank, step_ms, e2e_ms, int(x.astype(np.int64).sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_max_and_draw_their_own_batch():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]   # max(10, 15)
    assert [r[2] for r in res] == [30.0, 30.0]   # max(30, 29)
    assert res[0][3] != res[1][3]                # different batches per rank


def test_job_throughput_counts_every_rank():
    w = wl.get_workload("480p")
    one = bench.job_throughput(w.attn_flops(), 1, 20.0)
    eight = bench.job_throughput(w.attn_flops(), 8, 20.0)
    assert eight == pytest.approx(8 * one)
    assert one == pytest.approx(w.attn_flops() / 0.020 / 1e12)
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]
