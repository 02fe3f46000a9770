"""The replicas-only multi-GPU path on the host: world-size-2 gloo ranks on CPU.

Every (batch, head, query tile) is independent, so ranks run independent
copies of the workload; the only cross-rank step is the MAX of the timed
region, from which rank 0 reports whole-job throughput (weak scaling).
"""
import os
import socket

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
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [100.0, 250.0][rank]                 # rank 1 is the slow one
    tops, ms = bench.job_throughput(local_ms, 1e12, 10, dist, "cpu")
    out[rank] = (tops, ms)
    dist.barrier()
    dist.destroy_process_group()


def test_job_throughput_takes_the_slowest_rank_and_counts_all_ranks():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for r in (0, 1):
        tops, ms = out[r]
        assert ms == 250.0
        assert tops == pytest.approx(2 * 1e12 * 10 / 0.25 / 1e12)


def test_job_throughput_single_process():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    tops, ms = bench.job_throughput(200.0, 2e12, 5)
    assert ms == 200.0 and tops == pytest.approx(2e12 * 5 / 0.2 / 1e12)
