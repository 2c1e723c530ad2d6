"""The multi-GPU bench path runs independent replicas; its only cross-rank
step is the timing reduction.  Two gloo ranks on CPU check that reduction
and the whole-job throughput formula."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = [0.75, 0.8125][rank]                      # the slower rank sets the job time
        ms = bench.max_over_ranks(local_ms)
        out[rank] = ms
        out[2 + rank] = bench.job_tokens_per_s(256, world, ms)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replica_ranks_report_the_slowest():
    world = 2
    out = mp.get_context("spawn").Manager().list([0.0] * 4)
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 0.8125
    assert out[2] == out[3] == pytest.approx(256 * 2 / 0.8125e-3)


def test_single_process_is_a_no_op():
    import bench
    assert bench.max_over_ranks(1.25) == 1.25
    assert bench.job_tokens_per_s(256, 1, 0.5) == pytest.approx(512000.0)
