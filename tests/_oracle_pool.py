"""The oracle's full forward at the large workload sizes, spread over host processes.

Test helper.  The oracle's grouped forward visits the active experts one at
a time, and the rows of a NULL expert are zero.  So the oracle run with every
expert outside a block set to NULL yields exactly that block's rows of act and
y, by sorted position.  Each worker process runs the oracle's own
``route_sort``, ``gate_up_silu`` and ``down_proj`` for one block of experts.
The parent copies the rows of each block into place and finishes with the
oracle's ``blend``.  No arithmetic of the forward is written here.

The workers are started with 'spawn', which is safe after the parent has
initialised CUDA.  Each one limits its BLAS to one thread.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from typing import Dict, Optional, Sequence

import numpy as np

import oracle as orc
from workloads import make_problem
from workloads.generators import MATRIX_DOWN, MATRIX_GATE, MATRIX_UP, MoEConfig

_PROBLEM: Dict[MoEConfig, object] = {}


def _problem(cfg: MoEConfig):
    if cfg not in _PROBLEM:
        _PROBLEM.clear()
        _PROBLEM[cfg] = make_problem(cfg)
    return _PROBLEM[cfg]


def _init_worker():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _block_rows(args):
    """(lo, hi, act rows, y rows) of every expert of one block, by the oracle."""
    cfg, block = args
    prob = _problem(cfg)
    own = frozenset(block)
    gate, up, down = (
        (lambda e, m=m: prob.expert_weight(m, e) if e in own else None)
        for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN))
    rs = orc.route_sort(prob.topk_ids, cfg.experts)
    # np.zeros maps its pages lazily: only this block's rows take memory.
    act = orc.gate_up_silu(prob.x_bf16, cfg.topk, rs, gate, up, cfg.inter)
    y = orc.down_proj(act, rs, down, cfg.hidden)
    rows = []
    for e in block:
        lo, hi = int(rs.expert_offsets[e]), int(rs.expert_offsets[e + 1])
        rows.append((lo, hi, act[lo:hi].copy(), y[lo:hi].copy()))
    return rows


def moe_forward_pooled(cfg: MoEConfig, workers: Optional[int] = None,
                       block: int = 4) -> Dict[str, object]:
    """The result of ``orc.moe_forward`` on ``make_problem(cfg)`` (sort, act, y, out)."""
    prob = _problem(cfg)
    rs = orc.route_sort(prob.topk_ids, cfg.experts)
    active = [int(e) for e in rs.active_experts[: rs.active_count]]
    blocks: Sequence[Sequence[int]] = [active[i:i + block] for i in range(0, len(active), block)]
    p = cfg.pairs
    act = np.zeros((p, cfg.inter), dtype=np.float64)
    y = np.zeros((p, cfg.hidden), dtype=np.float64)
    if workers is None:
        workers = max(1, min(len(os.sched_getaffinity(0)), 16, len(blocks)))
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers, initializer=_init_worker) as pool:
        for part in pool.imap_unordered(_block_rows, [(cfg, b) for b in blocks]):
            for lo, hi, a, yy in part:
                act[lo:hi] = a
                y[lo:hi] = yy
    out = orc.blend(y, prob.topk_weights, rs.pair_pos)
    return {"sort": rs, "act": act, "y": y, "out": out}
