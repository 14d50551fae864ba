"""The benchmark's multi-rank host logic on CPU: two gloo ranks run the same
max-over-ranks aggregation bench.py uses under torchrun (each rank times an
independent replica; whole-job throughput = bytes of all ranks / the slowest
rank's time).  No GPU: the device tensors of the collectives live on the CPU."""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, loc = bench.dist_setup()
        assert (w, r, loc) == (world, rank, rank)
        # rank r took (10 + 5 r) ms for 4 steps of (1 + r) GB each
        value, total_ms, all_bytes = bench.aggregate_over_ranks(10.0 + 5.0 * rank, (1 + rank) * 1e9, 4,
                                                               torch.device("cpu"), world)
        results[rank] = (value, total_ms, all_bytes)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_aggregation_gloo(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    slowest = 10.0 + 5.0 * (world - 1)
    total_bytes = sum((1 + r) * 1e9 for r in range(world)) * 4
    for r in range(world):
        value, total_ms, all_bytes = results[r]
        assert total_ms == slowest               # every rank reports the slowest rank's time
        assert all_bytes == total_bytes          # bytes of all ranks
        assert abs(value - total_bytes / (slowest / 1e3) / 1e9) < 1e-9


def test_single_rank_aggregation_needs_no_process_group():
    import bench
    value, total_ms, all_bytes = bench.aggregate_over_ranks(8.0, 2e9, 4, torch.device("cpu"), 1)
    assert total_ms == 8.0 and all_bytes == 8e9 and abs(value - 1000.0) < 1e-9
