"""Put a seeded problem on the GPU as the library's device containers.

Plumbing for tests and the benchmark: it copies the generator's bytes to the
device and builds the pointer tables; it computes nothing of the forward.
"""

from __future__ import annotations

import numpy as np
import torch

from .generators import MATRIX_DOWN, MATRIX_GATE, MATRIX_UP, MoEProblem, draw_expert_weight, matrix_shape


def upload_projection(prob: MoEProblem, matrix: int, device="cuda"):
    """NVFP4Projection of one matrix for all experts, drawn expert by expert."""
    from nvfp4_weight_quantized_moe_b200 import NVFP4Projection

    cfg = prob.cfg
    n, k = matrix_shape(cfg, matrix)
    packed = torch.zeros((cfg.experts, n, k // 2), dtype=torch.uint8, device=device)
    scale = torch.zeros((cfg.experts, n, k // 16), dtype=torch.uint8, device=device)
    for e in range(cfg.experts):
        if e in prob.null_experts:
            continue
        p, s = draw_expert_weight(cfg, matrix, e)
        packed[e].copy_(torch.from_numpy(p))
        scale[e].copy_(torch.from_numpy(s))
    scale2 = torch.from_numpy(prob.scale2[matrix].copy()).to(device)
    return NVFP4Projection(packed, scale, scale2, null_experts=prob.null_experts)


def upload_shared(prob: MoEProblem, device="cuda"):
    """The shared expert's three projections, each an NVFP4Projection of one expert."""
    from nvfp4_weight_quantized_moe_b200 import NVFP4Projection

    out = []
    for matrix in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN):
        p, s, s2 = prob.shared_weight(matrix)
        out.append(NVFP4Projection(torch.from_numpy(p[None]).to(device),
                                   torch.from_numpy(s[None]).to(device),
                                   torch.tensor([float(s2)], dtype=torch.float32, device=device)))
    return tuple(out)


def upload_layer(prob: MoEProblem, device="cuda", shared: bool = False, shared_rows: int = 0,
                 activation=None):
    """The problem's layer on the device; ``activation`` given: a non-gated layer
    (up and down only) with that activation."""
    from nvfp4_weight_quantized_moe_b200 import NVFP4MoE

    gate = None if activation is not None else upload_projection(prob, MATRIX_GATE, device)
    return NVFP4MoE(gate, upload_projection(prob, MATRIX_UP, device),
                    upload_projection(prob, MATRIX_DOWN, device), prob.cfg.topk,
                    shared=upload_shared(prob, device) if shared else None,
                    shared_rows=shared_rows, activation=activation)


def upload_inputs(prob: MoEProblem, device="cuda"):
    """x (bf16), topk_ids (i32), topk_weights (f32) on the device."""
    x = torch.from_numpy(prob.x_bf16.view(np.int16)).view(torch.bfloat16).to(device)
    ids = torch.from_numpy(np.ascontiguousarray(prob.topk_ids)).to(device)
    w = torch.from_numpy(np.ascontiguousarray(prob.topk_weights)).to(device)
    return x, ids, w
