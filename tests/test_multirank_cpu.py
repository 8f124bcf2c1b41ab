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
    # The default workload is the largest single-GPU one (prefill M=8192).
    assert args.gpus == 1 and args.config == "prefill_m8192" and args.impl == "ours"
    assert args.warmup >= 3


def test_ncu_traffic_is_dropped_once_the_kernel_sources_change(monkeypatch):
    import bench
    key = ("prefill_m8192", "tcgen05")
    bytes_, _ = bench.NCU_TRAFFIC_BYTES[key]
    monkeypatch.setitem(bench.NCU_TRAFFIC_BYTES, key, (bytes_, bench.kernel_source_hash("tcgen05")))
    assert bench.ncu_traffic(*key) == bytes_
    monkeypatch.setitem(bench.NCU_TRAFFIC_BYTES, key, (bytes_, "000000000000"))
    assert bench.ncu_traffic(*key) is None


def _sharded_worker(rank, world, port, mode, results):
    """One rank: its partial forward from the oracle (no GPU here), then the
    package's all-reduce of ``out`` over gloo."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    import numpy as np
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import oracle as orc
        from nvfp4_weight_quantized_moe_b200 import all_reduce_out, expert_owner_range
        from workloads import make_problem
        from workloads.generators import MoEConfig
        cfg = MoEConfig("shard", hidden=64, inter=64, experts=6, topk=2, tokens=5,
                        router="uniform", seed=41)
        inter = cfg.inter
        if mode == "ep":
            lo, hi = expert_owner_range(cfg.experts, world, rank)
            prob = make_problem(cfg, null_experts=[e for e in range(cfg.experts) if not lo <= e < hi])
            fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (0, 1, 2)]
        else:
            prob = make_problem(cfg)
            inter = cfg.inter // world

            def fn(m):
                kind = "row" if m == 2 else "column"

                def get(e):
                    p, s, s2 = prob.expert_weight(m, e)
                    return (*orc.shard_nvfp4(p, s, kind, rank, world), s2)
                return get
            fns = [fn(m) for m in (0, 1, 2)]
        part = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *fns,
                               hidden=cfg.hidden, inter=inter)["out"]
        out = torch.from_numpy(part.copy())
        all_reduce_out(out)
        full_prob = make_problem(cfg)
        full = orc.moe_forward(full_prob.x_bf16, full_prob.topk_ids, full_prob.topk_weights,
                               cfg.experts, *[lambda e, m=m: full_prob.expert_weight(m, e)
                                              for m in (0, 1, 2)],
                               hidden=cfg.hidden, inter=cfg.inter)["out"]
        results[rank] = float(np.max(np.abs(out.numpy() - full)) / np.max(np.abs(full)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["ep", "tp"])
def test_sharded_partial_outputs_all_reduce_to_the_full_output(mode):
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, mode, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        assert results[0] < 1e-12 and results[1] < 1e-12


def test_bench_routes_every_load_time_op():
    # Each --op other than the layer forward goes to the load-time runner.
    import bench
    seen = []
    orig_load, orig_ours = bench.run_load_op, bench.run_ours
    bench.run_load_op = lambda args, *a: seen.append(("load", args.op))
    bench.run_ours = lambda args, *a: seen.append(("layer", args.op))
    try:
        for op in ("check_scales", "shard", "twins", "layer"):
            bench.main(["--op", op])
    finally:
        bench.run_load_op, bench.run_ours = orig_load, orig_ours
    assert seen == [("load", "check_scales"), ("load", "shard"), ("load", "twins"), ("layer", "layer")]
