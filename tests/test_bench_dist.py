"""The multi-GPU plumbing of bench.py (replicas only: barrier, max-over-ranks
timing, weak-scaling aggregation), exercised as two gloo ranks on CPU."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    ws, r = bench.init_dist("gloo")
    assert (ws, r) == (world, rank)
    bench.barrier()
    t = bench.max_over_ranks(1.5 + rank)  # rank 1 is the slow one
    v = bench.aggregate_throughput(32768, 10, ws, t)
    q.put((rank, t, v))
    dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, v in res:
        assert t == 2.5                         # every rank reports the slowest rank's time
        assert v == 32768 * 10 * 2 / 2.5        # rows of all ranks / max time


def test_single_process_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.aggregate_throughput(100, 4, 1, 2.0) == 200.0


def test_attention_flops_count_documents_only():
    import h3_inputs as hi
    dims, lay = hi.workload("t2va_32k_pad168")
    f = bench.attention_flops(dims, lay)
    assert f == 4.0 * 56 * 128 * (32600 ** 2 + 168 ** 2)
    assert torch.tensor(f) > 0
