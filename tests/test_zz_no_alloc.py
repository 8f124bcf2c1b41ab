"""The allocation-free gate+up entry point (nvfp4_moe_gate_up_silu_noalloc).

It is for callers that cannot give the library a workspace (their device memory
belongs to another allocator or a fixed budget, or they must not call
cudaMalloc).  It must give the same act as the workspace call on the same
inputs, call after call, and refuse requests larger than its fixed scratch.
This file runs last so that, if it fails, a stop-at-first-failure run has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
from workloads import make_problem
from workloads.generators import MoEConfig

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS_FRAC = 4e-3


def _close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got))
    assert orc.relative_l2(got, ref) <= REL_L2
    assert float(np.max(np.abs(got - ref))) <= MAX_ABS_FRAC * float(np.max(np.abs(ref)))


def test_no_alloc_gate_up_matches_the_workspace_call_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_weight_quantized_moe_b200 as nvm
    from nvfp4_weight_quantized_moe_b200 import _binding as B
    from workloads.device import upload_inputs, upload_layer

    cfg = MoEConfig("noalloc", hidden=1024, inter=512, experts=16, topk=4, tokens=24,
                    router="zipf", seed=31)
    prob = make_problem(cfg)
    layer = upload_layer(prob)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(cfg.tokens)
    nvm.route_sort(ids, cfg.experts, bufs.expert_offsets, bufs.sorted_pair_ids, bufs.pair_pos,
                   bufs.active_experts, bufs.active_count, bufs.status)
    cap = nvm.active_cap(cfg.experts, cfg.pairs)
    kept = int(bufs.expert_offsets[-1].item())

    # Reference: the existing workspace entry point on the same (tcgen05) path.
    ws = layer.workspace(cfg.tokens)
    nvm.gate_up_silu_ws(x, layer.gate.tables, layer.up.tables, bufs.act, bufs.expert_offsets,
                        bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count, cfg.inter,
                        cfg.hidden, cap, cfg.tokens, cfg.topk, cfg.experts, ws, path=2)
    torch.cuda.synchronize()
    ref = bufs.act[:kept].cpu().numpy().copy()

    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        bufs.act.fill_(float("nan"))
        status = B._lib.nvfp4_moe_gate_up_silu_noalloc(
            x.data_ptr(), layer.gate.tables, layer.up.tables, bufs.act.data_ptr(),
            bufs.expert_offsets.data_ptr(), bufs.sorted_pair_ids.data_ptr(),
            bufs.active_experts.data_ptr(), bufs.active_count.data_ptr(), cfg.inter, cfg.hidden,
            cap, cfg.tokens, cfg.topk, cfg.experts, stream)
        torch.cuda.synchronize()
        assert status == 0
        assert nvm.device_error() == 0
        _close(bufs.act[:kept].cpu().numpy(), ref)


def test_no_alloc_refuses_requests_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_weight_quantized_moe_b200 import _binding as B
    t = B.ExpertTables(8, 8, 8)
    p = ctypes.c_void_p(8)
    # 8192 tokens x 4 pairs x 1024 hidden x 2 bytes = 64 MiB of packed rows: over the limit.
    status = B._lib.nvfp4_moe_gate_up_silu_noalloc(p, t, t, p, p, p, p, p, 512, 1024, 16, 8192, 4,
                                                   16, None)
    assert status == 2
