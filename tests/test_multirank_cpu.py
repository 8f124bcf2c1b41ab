"""Multi-rank host logic of bench.py on CPU: two gloo ranks agree on the max
event time and on the whole-job throughput (weak scaling: every rank runs its
own replica of the workload)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        r, w, lr = bench.dist_info()
        assert (r, w, lr) == (rank, world, rank)
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        bench.barrier()
        results[rank] = bench.reduce_max(local_ms)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert results[0] == results[1] == 15.0


def test_reduce_max_is_identity_without_a_process_group():
    import bench
    assert not dist.is_initialized()
    assert bench.reduce_max(3.25) == 3.25


def test_bench_cli_defaults():
    import bench
    args = bench.parse_args([])
    assert args.gpus == 1 and args.config == "decode_m1" and args.impl == "ours"
    assert args.warmup >= 3
