"""Host logic of the multi-GPU bench path on CPU ranks (gloo, world size 2): each rank streams
its own independent sequence batch (no collective on the data path), the step time is the
maximum over ranks and the job throughput counts every rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 180.0][rank]
        total = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_throughput(world, total, steps=3)
        dist.barrier()
        q.put((rank, total, value))
    finally:
        dist.destroy_process_group()


def test_step_time_is_max_over_ranks_and_value_counts_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, value in res:
        assert total == 180.0
        assert value == pytest.approx(2 * bench.WL.batch * bench.TOK_PER_STEP / (60.0 / 1e3))


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1, None) == 7.5


def test_ranks_stream_independent_sequences():
    k0, v0, q0 = bench.workload_inputs(seq=0)
    k1, v1, q1 = bench.workload_inputs(seq=1)
    assert k0.shape == k1.shape and q0.shape == q1.shape
    assert not np.array_equal(k0, k1) and not np.array_equal(q0, q1)
