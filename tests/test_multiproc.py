"""Host logic of the multi-GPU bench path on CPU: two gloo ranks (replicas) must
agree on the max of their per-rank times, as bench.py does over NCCL on GPUs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier()
        results[rank] = bench.aggregate_max(values[rank], "cpu")
        bench.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("values", [(3.5, 1.25), (0.5, 7.0)])
def test_max_over_ranks_two_gloo_ranks(values):
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, list(values), results), nprocs=2, join=True,
                       start_method="spawn")
    assert results[0] == results[1] == max(values)


def test_aggregate_without_process_group_is_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.aggregate_max(2.5, "cpu") == 2.5
