"""The allocation-free gate+up entry point (nvfp4_moe_gate_up_silu_noalloc).

It is for callers that cannot give the library a workspace: their device
memory belongs to another allocator or to a fixed budget, or they must not
call cudaMalloc.  Its act must match the fp64 oracle within the forward's
tolerance, and agree with the workspace call on the same inputs, call after
call.  Requests larger than its fixed scratch must be refused.  Two shapes are
run: a few rows per expert (16-row token passes) and more than 16 rows per
expert (128-row token passes, about 4 MiB of packed rows in the scratch).
This file runs last so that, if it fails, a stop-at-first-failure run has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
from workloads import make_problem
from workloads.generators import MATRIX_GATE, MATRIX_UP, MoEConfig

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS_FRAC = 4e-3


def _close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), what
    rel = orc.relative_l2(got, ref)
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e}"
    err = float(np.max(np.abs(got - ref)))
    assert err <= MAX_ABS_FRAC * float(np.max(np.abs(ref))), f"{what}: max abs {err:.3e}"


CASES = [
    # 96 pairs over 16 experts: at most 16 rows per expert (16-row passes)
    MoEConfig("noalloc16", hidden=1024, inter=512, experts=16, topk=4, tokens=24,
              router="zipf", seed=31),
    # 2048 pairs over 16 experts, ~128 rows each (128-row passes, ragged groups)
    MoEConfig("noalloc128", hidden=1024, inter=512, experts=16, topk=4, tokens=512,
              router="uniform", seed=32),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_no_alloc_gate_up_matches_the_oracle_twice(cfg):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nvfp4_weight_quantized_moe_b200 as nvm
    from nvfp4_weight_quantized_moe_b200 import _binding as B
    from workloads.device import upload_inputs, upload_layer

    prob = make_problem(cfg)
    layer = upload_layer(prob)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(cfg.tokens)
    nvm.route_sort(ids, cfg.experts, bufs.expert_offsets, bufs.sorted_pair_ids, bufs.pair_pos,
                   bufs.active_experts, bufs.active_count, bufs.status)
    cap = nvm.active_cap(cfg.experts, cfg.pairs)

    # The oracle's act by sorted position.
    rs = orc.route_sort(prob.topk_ids, cfg.experts)
    kept = int(rs.expert_offsets[-1])
    ref = orc.gate_up_silu(prob.x_bf16, cfg.topk, rs,
                           lambda e: prob.expert_weight(MATRIX_GATE, e),
                           lambda e: prob.expert_weight(MATRIX_UP, e), cfg.inter)[:kept]

    # The existing workspace entry point on the same (tcgen05) path.
    ws = layer.workspace(cfg.tokens)
    nvm.gate_up_silu_ws(x, layer.gate.tables, layer.up.tables, bufs.act, bufs.expert_offsets,
                        bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count, cfg.inter,
                        cfg.hidden, cap, cfg.tokens, cfg.topk, cfg.experts, ws, path=2)
    torch.cuda.synchronize()
    act_ws = bufs.act[:kept].cpu().numpy().copy()
    _close(act_ws, ref, "workspace call vs oracle")

    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        bufs.act.fill_(float("nan"))
        status = B._lib.nvfp4_moe_gate_up_silu_noalloc(
            x.data_ptr(), layer.gate.tables, layer.up.tables, bufs.act.data_ptr(),
            bufs.expert_offsets.data_ptr(), bufs.sorted_pair_ids.data_ptr(),
            bufs.active_experts.data_ptr(), bufs.active_count.data_ptr(), cfg.inter, cfg.hidden,
            cap, cfg.tokens, cfg.topk, cfg.experts, stream)
        torch.cuda.synchronize()
        assert status == 0
        assert nvm.device_error() == 0
        got = bufs.act[:kept].cpu().numpy()
        _close(got, ref, f"no-alloc call {call} vs oracle")
        _close(got, act_ws, f"no-alloc call {call} vs workspace call")


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
