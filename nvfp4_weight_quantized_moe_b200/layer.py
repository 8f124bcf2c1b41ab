"""Device-side containers for one NVFP4 MoE layer and its four-call forward.

PyTorch here only owns device memory and supplies the stream; every step of
the forward is one call into the C ABI (``_binding``).  Sharding across ranks
is set up here too: tensor-parallel shards of the weights (one library call
per projection) and expert-parallel blocks (NULL table entries for the experts
a rank does not hold); either way a rank's ``out`` is a partial sum that one
all-reduce completes (:func:`all_reduce_out`).
"""

from __future__ import annotations

from typing import Iterable, Optional

import torch

from . import _binding as B


def expert_owner_range(num_experts: int, world: int, rank: int):
    """[lo, hi): the block of consecutive experts rank holds under expert
    parallelism; block sizes differ by at most one (lo = rank * E // world)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * num_experts // world, (rank + 1) * num_experts // world


def all_reduce_out(out: torch.Tensor, group=None) -> torch.Tensor:
    """Sum a rank's partial ``out`` over the process group (in place).

    Expert- and tensor-parallel ranks each produce a partial sum of the layer
    output; one all-reduce (NCCL on GPUs) completes it on every rank."""
    import torch.distributed as dist
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


class NVFP4Projection:
    """One NVFP4 projection for every expert, resident on the device.

    packed  u8  [B, N, K/2]  packed E2M1 codes, low nibble = even k
    scale   u8  [B, N, K/16] E4M3 block scales
    scale2  f32 [B]          weight_scale_2 per expert
    The tables list ``num_experts`` experts (default B); expert e in
    [first_expert, first_expert + B) is packed[e - first_expert], every other
    one, and those in ``null_experts``, a NULL entry (skipped by the forward).
    """

    def __init__(self, packed: torch.Tensor, scale: torch.Tensor, scale2: torch.Tensor,
                 null_experts: Iterable[int] = (), first_expert: int = 0,
                 num_experts: Optional[int] = None):
        if packed.dtype != torch.uint8 or scale.dtype != torch.uint8:
            raise TypeError("packed and scale must be uint8")
        if packed.device.type != "cuda":
            raise ValueError("weights must be on a CUDA device")
        e, n, half_k = packed.shape
        if tuple(scale.shape) != (e, n, half_k * 2 // 16):
            raise ValueError("scale shape must be [E, N, K/16]")
        total = e if num_experts is None else int(num_experts)
        if first_expert < 0 or first_expert + e > total:
            raise ValueError("expert block outside the table")
        self.packed = packed.contiguous()
        self.scale = scale.contiguous()
        s2 = scale2.to(device=packed.device, dtype=torch.float32).reshape(-1)
        if s2.numel() != e:
            raise ValueError("scale2 must hold one value per expert of the block")
        self.first_expert = first_expert
        self.num_experts, self.n, self.k = total, n, half_k * 2
        null = set(int(i) for i in null_experts)
        held = lambda i: first_expert <= i < first_expert + e and i not in null
        pp = [self.packed.data_ptr() + (i - first_expert) * self.packed.stride(0) if held(i) else 0
              for i in range(total)]
        sp = [self.scale.data_ptr() + (i - first_expert) * self.scale.stride(0) if held(i) else 0
              for i in range(total)]
        s2_full = torch.zeros(total, dtype=torch.float32, device=packed.device)
        s2_full[first_expert:first_expert + e] = s2
        self.scale2 = s2_full
        self.packed_ptrs = torch.tensor(pp, dtype=torch.int64, device=packed.device)
        self.scale_ptrs = torch.tensor(sp, dtype=torch.int64, device=packed.device)
        self.tables = B.ExpertTables(self.packed_ptrs.data_ptr(), self.scale_ptrs.data_ptr(),
                                     self.scale2.data_ptr())

    @property
    def nbytes_per_expert(self) -> int:
        """Packed nibbles + block scales of one expert (the bytes a pass must read)."""
        return self.n * self.k // 2 + self.n * self.k // 16

    def expert_block(self, lo: int, hi: int) -> "NVFP4Projection":
        """A projection holding copies of experts [lo, hi) only, the others NULL
        (what an expert-parallel rank keeps resident)."""
        f = self.first_expert
        if not f <= lo <= hi <= f + self.packed.shape[0]:
            raise ValueError("experts not held by this projection")
        return NVFP4Projection(self.packed[lo - f:hi - f].clone(), self.scale[lo - f:hi - f].clone(),
                               self.scale2[lo:hi].clone(), first_expert=lo,
                               num_experts=self.num_experts)

    def shard(self, kind: int, rank: int, tp: int) -> "NVFP4Projection":
        """This tensor-parallel rank's shard (``B.SHARD_COLUMN``: N / tp rows;
        ``B.SHARD_ROW``: K / tp of every row), in one library call."""
        if self.first_expert != 0 or self.packed.shape[0] != self.num_experts:
            raise ValueError("shard a projection that holds every expert")
        packed, scale = B.shard_nvfp4(self.packed, self.scale, kind, rank, tp)
        null = (self.packed_ptrs == 0).nonzero().flatten().tolist()
        return NVFP4Projection(packed, scale, self.scale2.clone(), null_experts=null)


class MoEBuffers:
    """Outputs and intermediates of one forward, for M tokens.

    With a shared expert, ``topk`` and ``num_experts`` count its slot and
    table entries, and ``topk_ids`` / ``topk_weights`` hold the appended
    routing [M, topk] that nvfp4_moe_append_shared writes.
    """

    def __init__(self, num_tokens: int, topk: int, num_experts: int, hidden: int, inter: int,
                 device, out_bf16: bool = False, shared: bool = False):
        p = num_tokens * topk
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.num_tokens, self.topk = num_tokens, topk
        self.topk_ids = torch.empty(max(num_tokens, 1), topk, **i32) if shared else None
        self.topk_weights = torch.empty(max(num_tokens, 1), topk, **f32) if shared else None
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


class _Tables:
    """Expert tables of one projection with the shared expert's entries appended."""

    def __init__(self, routed: NVFP4Projection, shared: NVFP4Projection, slots: int):
        dev = routed.packed.device
        sp, ss = shared.packed_ptrs[:1], shared.scale_ptrs[:1]
        self.packed_ptrs = torch.cat([routed.packed_ptrs, sp.expand(slots)]).contiguous()
        self.scale_ptrs = torch.cat([routed.scale_ptrs, ss.expand(slots)]).contiguous()
        self.scale2 = torch.cat([routed.scale2, shared.scale2[:1].expand(slots)]).to(dev).contiguous()
        self.tables = B.ExpertTables(self.packed_ptrs.data_ptr(), self.scale_ptrs.data_ptr(),
                                     self.scale2.data_ptr())


class NVFP4MoE:
    """The grouped NVFP4 expert forward of one layer, optionally with a shared expert.

    ``gate=None`` makes a layer of non-gated experts (up and down only, as the
    experts whose twins ``prepare_prefill_weights`` builds in
    nemotron_moe/prefill_weights.rs): act = f(x Wu^T) with f = ``activation``
    ("relu2" or "silu"), then down and blend as usual.

    ``shared`` = (gate, up, down) projections of one expert (E = 1) with the
    routed experts' shapes: every token also runs it, in the same gate+up and
    down launches (nvfp4_moe_append_shared), and ``out`` adds its output times
    the per-token ``shared_weights`` given to :meth:`forward` (1 by default).
    ``shared_rows`` tokens share one table entry of the shared expert, and so
    one group of CTAs; by default about the routed rows per expert.
    """

    def __init__(self, gate: Optional[NVFP4Projection], up: NVFP4Projection, down: NVFP4Projection,
                 topk: int, shared=None, shared_rows: int = 0, activation: Optional[str] = None):
        if gate is None:
            if activation not in B.ACTIVATIONS:
                raise ValueError(f"a non-gated layer needs activation in {sorted(B.ACTIVATIONS)}")
            if shared is not None:
                raise ValueError("the shared expert is built for gated layers only")
        elif activation is not None:
            raise ValueError("activation applies to non-gated layers (gate=None)")
        ref = gate if gate is not None else up
        if not (ref.num_experts == up.num_experts == down.num_experts):
            raise ValueError("expert counts differ")
        if ref.n != up.n or ref.k != up.k or down.n != up.k or down.k != up.n:
            raise ValueError("gate/up must be [I, H] and down [H, I]")
        self.gate, self.up, self.down = gate, up, down
        self.activation = activation
        self.num_experts = up.num_experts
        self.hidden, self.inter = up.k, up.n
        self.topk = topk
        self.shared = None
        self.shared_rows = int(shared_rows)
        if shared is not None:
            sg, su, sd = shared
            for sp, rp in ((sg, gate), (su, up), (sd, down)):
                if sp.num_experts != 1 or (sp.n, sp.k) != (rp.n, rp.k):
                    raise ValueError("the shared expert is one expert with the routed shapes")
            self.shared = (sg, su, sd)
        self._ext = {}

    # -- sharding across ranks ---------------------------------------------------
    def tensor_parallel(self, rank: int, tp: int) -> "NVFP4MoE":
        """This rank's layer under tensor parallelism: gate and up keep I / tp rows
        (column-parallel), down I / tp of its K (row-parallel), as
        shard_quantized_nvfp4 in quant_shard.rs; the shared expert likewise.  The
        rank's ``out`` is a partial sum (see :func:`all_reduce_out`)."""
        col, row = B.SHARD_COLUMN, B.SHARD_ROW
        shared = None
        if self.shared is not None:
            sg, su, sd = self.shared
            shared = (sg.shard(col, rank, tp), su.shard(col, rank, tp), sd.shard(row, rank, tp))
        gate = self.gate.shard(col, rank, tp) if self.gate is not None else None
        return NVFP4MoE(gate, self.up.shard(col, rank, tp), self.down.shard(row, rank, tp),
                        self.topk, shared=shared, shared_rows=self.shared_rows,
                        activation=self.activation)

    def expert_parallel(self, rank: int, world: int) -> "NVFP4MoE":
        """This rank's layer under expert parallelism: copies of its block of
        experts (:func:`expert_owner_range`), NULL entries for the rest.  The
        shared expert, if any, runs on rank 0 only.  The rank's ``out`` is a
        partial sum (see :func:`all_reduce_out`)."""
        lo, hi = expert_owner_range(self.num_experts, world, rank)
        projs = [p.expert_block(lo, hi) if p is not None else None
                 for p in (self.gate, self.up, self.down)]
        shared = self.shared if rank == 0 else None
        return NVFP4MoE(*projs, self.topk, shared=shared, shared_rows=self.shared_rows,
                        activation=self.activation)

    # -- shared expert bookkeeping ------------------------------------------------
    def rows_per_shared_slot(self, num_tokens: int) -> int:
        """Tokens per shared table entry for a batch of num_tokens."""
        if self.shared_rows:
            rows = self.shared_rows
        else:
            mean = -(-num_tokens * self.topk // self.num_experts)
            rows = max(16, -(-mean // 16) * 16)
        room = 1024 - self.num_experts
        if room < 1:
            raise ValueError("no table entries left for the shared expert")
        return max(rows, -(-num_tokens // room))

    def _ext_tables(self, slots: int):
        if slots not in self._ext:
            self._ext[slots] = tuple(_Tables(r, s, slots)
                                     for r, s in zip((self.gate, self.up, self.down), self.shared))
        return self._ext[slots]

    def _route_shape(self, num_tokens: int):
        """(slots per token, table entries) of a batch."""
        if self.shared is None:
            return self.topk, self.num_experts
        slots = B.shared_slots(num_tokens, self.rows_per_shared_slot(num_tokens))
        return self.topk + 1, self.num_experts + slots

    def buffers(self, num_tokens: int, out_bf16: bool = False) -> MoEBuffers:
        k, e = self._route_shape(num_tokens)
        if self.shared is not None:
            e = 1024  # the library's largest table: enough entries for any batch size
        return MoEBuffers(num_tokens, k, e, self.hidden, self.inter, self.up.packed.device,
                          out_bf16, shared=self.shared is not None)

    def workspace(self, num_tokens: int) -> torch.Tensor:
        """Device workspace of the tcgen05 path for batches of up to num_tokens."""
        k, _ = self._route_shape(num_tokens)
        n = B.workspace_bytes(num_tokens, k, self.hidden, self.inter)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=self.up.packed.device)

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                bufs: Optional[MoEBuffers] = None, path: int = 0, split: int = 0,
                tiles: int = 0, depth: int = 0, workspace: Optional[torch.Tensor] = None,
                stream=None, steps: bool = False, staging: int = 0,
                shared_weights: Optional[torch.Tensor] = None) -> MoEBuffers:
        """Run the four steps on ``stream``; results land in ``bufs`` (returned).
        One library call (nvfp4_moe_forward) by default; ``steps=True`` makes the
        four single-step calls instead (same kernels, same results).

        path / split / tiles / depth / staging are the launch options of the two
        projections (0 = chosen from the shape); see nvfp4_moe_launch_opts.
        With a ``workspace`` (see :meth:`workspace`) the projections may take
        the tcgen05 path.  With a shared expert, the routing is first extended
        by one slot per token (one more library call) and ``shared_weights``
        (f32 [M] or None for 1) weighs its output."""
        m = x.shape[0]
        if bufs is None:
            bufs = self.buffers(m)
        if m > bufs.num_tokens:
            raise ValueError("buffers were sized for fewer tokens")
        if self.gate is None:
            return self._forward_nongated(x, topk_ids, topk_weights, bufs, path, split, tiles,
                                          depth, staging, workspace, stream, steps, shared_weights)
        gate_t, up_t, down_t = self.gate.tables, self.up.tables, self.down.tables
        topk, num_experts = self.topk, self.num_experts
        if self.shared is not None:
            rows = self.rows_per_shared_slot(m)
            slots = B.shared_slots(m, rows)
            if num_experts + slots > bufs.active_experts.numel():
                raise ValueError("buffers hold too few expert entries for this batch")
            ids, ws = bufs.topk_ids[:m], bufs.topk_weights[:m]
            B.append_shared(topk_ids, topk_weights, num_experts, rows, ids, ws,
                            shared_weights=shared_weights, stream=stream)
            topk_ids, topk_weights = ids, ws
            gate_t, up_t, down_t = (t.tables for t in self._ext_tables(slots))
            topk, num_experts = topk + 1, num_experts + slots
        elif shared_weights is not None:
            raise ValueError("shared_weights given to a layer without a shared expert")
        if not steps:
            B.forward(x, topk_ids, topk_weights, gate_t, up_t, down_t, bufs.c_buffers, num_experts,
                      self.hidden, self.inter, workspace=workspace, path=path, split=split,
                      tiles=tiles, depth=depth, staging=staging, stream=stream)
            return bufs
        p = m * topk
        cap = B.active_cap(num_experts, p)
        B.route_sort(topk_ids, num_experts, bufs.expert_offsets[:num_experts + 1],
                     bufs.sorted_pair_ids, bufs.pair_pos, bufs.active_experts[:num_experts],
                     bufs.active_count, bufs.status, stream=stream)
        opts = dict(path=path, split=split, tiles=tiles, depth=depth, staging=staging, stream=stream)
        if workspace is None:
            B.gate_up_silu(x, gate_t, up_t, bufs.act, bufs.expert_offsets, bufs.sorted_pair_ids,
                           bufs.active_experts, bufs.active_count, self.inter, self.hidden, cap, m,
                           topk, **opts)
            B.down(bufs.act, down_t, bufs.y, bufs.expert_offsets, bufs.active_experts,
                   bufs.active_count, self.hidden, self.inter, cap, m, topk, **opts)
        else:
            B.gate_up_silu_ws(x, gate_t, up_t, bufs.act, bufs.expert_offsets,
                              bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count,
                              self.inter, self.hidden, cap, m, topk, num_experts, workspace, **opts)
            B.down_ws(bufs.act, down_t, bufs.y, bufs.expert_offsets, bufs.active_experts,
                      bufs.active_count, self.hidden, self.inter, cap, m, topk, num_experts,
                      workspace, **opts)
        B.blend(bufs.y, topk_weights, bufs.pair_pos, bufs.out, bufs.out_bf16, stream=stream)
        return bufs

    def _forward_nongated(self, x, topk_ids, topk_weights, bufs, path, split, tiles, depth,
                          staging, workspace, stream, steps, shared_weights) -> MoEBuffers:
        if shared_weights is not None:
            raise ValueError("shared_weights given to a layer without a shared expert")
        opts = dict(path=path, split=split, tiles=tiles, depth=depth, staging=staging,
                    stream=stream)
        if not steps:
            B.forward_nongated(x, topk_ids, topk_weights, self.up.tables, self.down.tables,
                               bufs.c_buffers, self.num_experts, self.hidden, self.inter,
                               self.activation, workspace=workspace, **opts)
            return bufs
        m, topk, e = x.shape[0], self.topk, self.num_experts
        cap = B.active_cap(e, m * topk)
        B.route_sort(topk_ids, e, bufs.expert_offsets[:e + 1], bufs.sorted_pair_ids,
                     bufs.pair_pos, bufs.active_experts[:e], bufs.active_count, bufs.status,
                     stream=stream)
        if workspace is None:
            B.up_act(x, self.up.tables, bufs.act, bufs.expert_offsets, bufs.sorted_pair_ids,
                     bufs.active_experts, bufs.active_count, self.inter, self.hidden, cap, m, topk,
                     self.activation, **opts)
            B.down(bufs.act, self.down.tables, bufs.y, bufs.expert_offsets, bufs.active_experts,
                   bufs.active_count, self.hidden, self.inter, cap, m, topk, **opts)
        else:
            B.up_act_ws(x, self.up.tables, bufs.act, bufs.expert_offsets, bufs.sorted_pair_ids,
                        bufs.active_experts, bufs.active_count, self.inter, self.hidden, cap, m,
                        topk, e, self.activation, workspace, **opts)
            B.down_ws(bufs.act, self.down.tables, bufs.y, bufs.expert_offsets, bufs.active_experts,
                      bufs.active_count, self.hidden, self.inter, cap, m, topk, e, workspace, **opts)
        B.blend(bufs.y, topk_weights, bufs.pair_pos, bufs.out, bufs.out_bf16, stream=stream)
        return bufs

    def shared_rows_of(self, bufs: MoEBuffers, m: int):
        """(sh_act [M, I], sh_out [M, H]) views of the last forward's shared rows.

        They start at sorted position expert_offsets[E] (read from the device,
        which synchronises): the kept routed pairs all sort before them.
        """
        if self.shared is None:
            raise ValueError("no shared expert")
        lo = int(bufs.expert_offsets[self.num_experts].item())
        return bufs.act[lo:lo + m], bufs.y[lo:lo + m]
