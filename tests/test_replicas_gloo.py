"""The multi-GPU bench path is replicas only (the decode, quantize and
scoring work has no exchange step): every rank runs its own copy and the
job's time is the slowest rank's.  The host logic of that path runs here as
two gloo ranks on the CPU."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took 10 + 3 r ms for a step of 2 GB
        t = bench.max_over_ranks(dist, 10.0 + 3.0 * rank, "cpu")
        out[rank] = (t, bench.whole_job_gbs(world, 2e9, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork of this process
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1]
    t, v = out[0]
    assert t == 13.0
    assert abs(v - 2 * 2e9 / 13e-3 / 1e9) < 1e-9


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 7.5, "cpu") == 7.5
    assert abs(bench.whole_job_gbs(1, 1e9, 1.0) - 1000.0) < 1e-9
