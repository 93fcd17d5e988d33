"""The multi-GPU layout of bench.py on CPU: N independent replicas (one per
rank, no collective on the data path), the step time taken as the maximum
over ranks and the job's throughput counting every rank's units. Run as two
gloo ranks over 127.0.0.1 (no GPU needed)."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = [2.0, 5.0][rank]          # ranks finish at different times
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        out[rank] = (ms, bench.job_throughput(1000, world, ms))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, val = res[0]
    assert ms == 5.0
    assert val == pytest.approx(2 * 1000 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    assert bench.job_throughput(6_291_456, 1, 0.1) == pytest.approx(62.91456)
