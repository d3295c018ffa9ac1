"""Multi-rank host logic on CPU (gloo, world size 2, 127.0.0.1).

The path shards by replica: every rank runs the whole workload on its own
input (weak scaling) with no data-path collective; the only collectives are the
benchmark's barrier and the max over ranks of the step time.  These tests run
that logic as gloo ranks, including a rank that fails before the collective
(the survivor must get an error from a short process-group timeout, not hang).
"""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port, timeout_s=60):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _worker_max(rank, world, port, out):
    import torch.distributed as dist
    import bench
    import workloads as W
    _init(rank, world, port)
    bench.barrier(world)
    my_ms = 100.0 + 7.0 * rank
    mx = bench.max_over_ranks(my_ms, world)
    seed = bench.replica_seed(W.VIDEO, rank)
    value = bench.job_throughput(1e12, world, 10, mx)
    out[rank] = (mx, seed, value)
    bench.barrier(world)
    dist.destroy_process_group()


def test_replicas_take_the_max_over_ranks_and_distinct_seeds():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker_max, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0] == 107.0
    assert out[0][1] != out[1][1]
    # two replicas of 1 TFLOP per step, 10 steps in 107 ms
    assert abs(out[0][2] - 2 * 1e12 * 10 / 0.107 / 1e12) < 1e-9


def _worker_fail(rank, world, port, out):
    import torch.distributed as dist
    import bench
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        out[rank] = "left"
        return                              # leaves between steps, no collective in flight
    try:
        bench.max_over_ranks(1.0, world)
        out[rank] = "returned"
    except Exception as e:                  # the short timeout ends the collective with an error
        out[rank] = "error:" + type(e).__name__
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.timeout(120)
def test_a_missing_rank_ends_the_collective_with_an_error():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.start_processes(_worker_fail, args=(world, port, out), nprocs=world, start_method="spawn", join=False)
    while not ctx.join(timeout=60):
        pass
    assert out[1] == "left"
    assert out[0].startswith("error:")
