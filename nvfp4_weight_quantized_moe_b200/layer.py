"""Device-side containers for one NVFP4 MoE layer and its four-call forward.

PyTorch here only owns device memory and supplies the stream; every step of
the forward is one call into the C ABI (``_binding``).
"""

from __future__ import annotations

from typing import Iterable, Optional

import torch

from . import _binding as B


class NVFP4Projection:
    """One NVFP4 projection for every expert, resident on the device.

    packed  u8  [E, N, K/2]  packed E2M1 codes, low nibble = even k
    scale   u8  [E, N, K/16] E4M3 block scales
    scale2  f32 [E]          weight_scale_2 per expert
    Experts listed in ``null_experts`` get NULL table entries (skipped).
    """

    def __init__(self, packed: torch.Tensor, scale: torch.Tensor, scale2: torch.Tensor,
                 null_experts: Iterable[int] = ()):
        if packed.dtype != torch.uint8 or scale.dtype != torch.uint8:
            raise TypeError("packed and scale must be uint8")
        if packed.device.type != "cuda":
            raise ValueError("weights must be on a CUDA device")
        e, n, half_k = packed.shape
        if tuple(scale.shape) != (e, n, half_k * 2 // 16):
            raise ValueError("scale shape must be [E, N, K/16]")
        self.packed = packed.contiguous()
        self.scale = scale.contiguous()
        self.scale2 = scale2.to(device=packed.device, dtype=torch.float32).contiguous()
        self.num_experts, self.n, self.k = e, n, half_k * 2
        null = set(int(i) for i in null_experts)
        pp = [0 if i in null else self.packed.data_ptr() + i * self.packed.stride(0) for i in range(e)]
        sp = [0 if i in null else self.scale.data_ptr() + i * self.scale.stride(0) for i in range(e)]
        self.packed_ptrs = torch.tensor(pp, dtype=torch.int64, device=packed.device)
        self.scale_ptrs = torch.tensor(sp, dtype=torch.int64, device=packed.device)
        self.tables = B.ExpertTables(self.packed_ptrs.data_ptr(), self.scale_ptrs.data_ptr(),
                                     self.scale2.data_ptr())

    @property
    def nbytes_per_expert(self) -> int:
        """Packed nibbles + block scales of one expert (the bytes a pass must read)."""
        return self.n * self.k // 2 + self.n * self.k // 16


class MoEBuffers:
    """Outputs and intermediates of one forward, for M tokens."""

    def __init__(self, num_tokens: int, topk: int, num_experts: int, hidden: int, inter: int,
                 device, out_bf16: bool = False):
        p = num_tokens * topk
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.num_tokens, self.topk = num_tokens, topk
        self.expert_offsets = torch.empty(num_experts + 1, **i32)
        self.sorted_pair_ids = torch.empty(max(p, 1), **i32)
        self.pair_pos = torch.empty(max(p, 1), **i32)
        self.active_experts = torch.empty(num_experts, **i32)
        self.active_count = torch.empty(1, **i32)
        self.status = torch.empty(1, **i32)
        self.act = torch.empty(max(p, 1), inter, **f32)
        self.y = torch.empty(max(p, 1), hidden, **f32)
        self.out = torch.empty(max(num_tokens, 1), hidden, **f32)
        self.out_bf16 = (torch.empty(max(num_tokens, 1), hidden, dtype=torch.bfloat16, device=device)
                         if out_bf16 else None)
        # The same pointers as one nvfp4_moe_buffers, for the one-call forward.
        self.c_buffers = B.Buffers(
            self.expert_offsets.data_ptr(), self.sorted_pair_ids.data_ptr(), self.pair_pos.data_ptr(),
            self.active_experts.data_ptr(), self.active_count.data_ptr(), self.status.data_ptr(),
            self.act.data_ptr(), self.y.data_ptr(), self.out.data_ptr(),
            self.out_bf16.data_ptr() if self.out_bf16 is not None else None)


class NVFP4MoE:
    """The grouped NVFP4 expert forward of one layer."""

    def __init__(self, gate: NVFP4Projection, up: NVFP4Projection, down: NVFP4Projection, topk: int):
        if not (gate.num_experts == up.num_experts == down.num_experts):
            raise ValueError("expert counts differ")
        if gate.n != up.n or gate.k != up.k or down.n != gate.k or down.k != gate.n:
            raise ValueError("gate/up must be [I, H] and down [H, I]")
        self.gate, self.up, self.down = gate, up, down
        self.num_experts = gate.num_experts
        self.hidden, self.inter = gate.k, gate.n
        self.topk = topk

    def buffers(self, num_tokens: int, out_bf16: bool = False) -> MoEBuffers:
        return MoEBuffers(num_tokens, self.topk, self.num_experts, self.hidden, self.inter,
                          self.gate.packed.device, out_bf16)

    def workspace(self, num_tokens: int) -> torch.Tensor:
        """Device workspace of the tcgen05 path for batches of up to num_tokens."""
        n = B.workspace_bytes(num_tokens, self.topk, self.hidden, self.inter)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.gate.packed.device)

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                bufs: Optional[MoEBuffers] = None, path: int = 0, split: int = 0,
                tiles: int = 0, depth: int = 0, workspace: Optional[torch.Tensor] = None,
                stream=None, steps: bool = False) -> MoEBuffers:
        """Run the four steps on ``stream``; results land in ``bufs`` (returned).
        One library call (nvfp4_moe_forward) by default; ``steps=True`` makes the
        four single-step calls instead (same kernels, same results).

        path / split / tiles / depth are the launch options of the two
        projections (0 = chosen from the shape); see nvfp4_moe_launch_opts.
        With a ``workspace`` (see :meth:`workspace`) the projections may take
        the tcgen05 path."""
        m = x.shape[0]
        if bufs is None:
            bufs = self.buffers(m)
        if m > bufs.num_tokens:
            raise ValueError("buffers were sized for fewer tokens")
        if not steps:
            B.forward(x, topk_ids, topk_weights, self.gate.tables, self.up.tables, self.down.tables,
                      bufs.c_buffers, self.num_experts, self.hidden, self.inter, workspace=workspace,
                      path=path, split=split, tiles=tiles, depth=depth, stream=stream)
            return bufs
        p = m * self.topk
        cap = B.active_cap(self.num_experts, p)
        B.route_sort(topk_ids, self.num_experts, bufs.expert_offsets, bufs.sorted_pair_ids,
                     bufs.pair_pos, bufs.active_experts, bufs.active_count, bufs.status,
                     stream=stream)
        opts = dict(path=path, split=split, tiles=tiles, depth=depth, stream=stream)
        if workspace is None:
            B.gate_up_silu(x, self.gate.tables, self.up.tables, bufs.act, bufs.expert_offsets,
                           bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count,
                           self.inter, self.hidden, cap, m, self.topk, **opts)
            B.down(bufs.act, self.down.tables, bufs.y, bufs.expert_offsets, bufs.active_experts,
                   bufs.active_count, self.hidden, self.inter, cap, m, self.topk, **opts)
        else:
            B.gate_up_silu_ws(x, self.gate.tables, self.up.tables, bufs.act, bufs.expert_offsets,
                              bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count,
                              self.inter, self.hidden, cap, m, self.topk, self.num_experts,
                              workspace, **opts)
            B.down_ws(bufs.act, self.down.tables, bufs.y, bufs.expert_offsets,
                      bufs.active_experts, bufs.active_count, self.hidden, self.inter, cap, m,
                      self.topk, self.num_experts, workspace, **opts)
        B.blend(bufs.y, topk_weights, bufs.pair_pos, bufs.out, bufs.out_bf16, stream=stream)
        return bufs
