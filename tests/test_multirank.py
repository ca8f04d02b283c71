"""Host logic of the multi-GPU benchmark path on CPU: two gloo ranks agree on
the slowest replica's time and report the whole-job throughput. The path has
no data exchange (replicas only), so this is the only cross-rank step."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = [10.0, 12.5][rank]
    ms = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
    value = bench.aggregate_value(step_bytes=1_000_000_000, steps=4, total_ms_max=ms, world=world)
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 12.5
        # 2 replicas x 4 steps x 1 GB in 12.5 ms
        assert value == pytest.approx(2 * 4 * 1.0 / 12.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, torch.device("cpu"), 1) == 3.0
    assert bench.aggregate_value(10**9, 10, 1000.0, 1) == pytest.approx(10.0)
