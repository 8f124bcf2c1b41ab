"""Seeded synthetic workloads for the grouped NVFP4 MoE expert forward.

Tensor layouts follow the pages (metrale_model_arch/tp_shard/quant_shard.rs,
the layout comment at the top of the file; metrale_model_layers/layers/ops/
nvfp4_moe_grouped.rs, the module doc):

* an NVFP4 weight of logical shape [N, K] is ``packed`` u8 [N, K/2] (two E2M1
  codes per byte), ``scale`` u8 [N, K/16] (one E4M3 code per 16 consecutive k)
  and one f32 ``weight_scale_2``;
* activations are BF16, held here as their raw uint16 bit patterns.

Gate and up have N = intermediate, K = hidden; down has N = hidden,
K = intermediate.

Value recipe:

* nibbles: every byte uniform over 0..255, so both nibbles are independent and
  uniform over the 16 E2M1 codes;
* block scales: "uniform in [2^-4, 2^2]" read as uniform over the E4M3 codes
  0x18..0x48, whose values are exactly 2^-4 .. 2^2;
* weight_scale_2 = f32(1/448) per tensor;
* x: f32 N(0, 1) rounded to BF16 (round to nearest even);
* router: logits N(0, 1) [M, E] (plus a Zipf(s) bias log p_e, p_e ~ r_e^-s over a
  seeded rank permutation r, for the skewed decode workload), softmax, top-k
  with ties to the lower expert id, renormalised so a token's k weights sum
  to 1.  Routing sits upstream of the expert forward; it is input generation.

Every (matrix, expert) weight is drawn from its own seeded stream, so any single
expert can be regenerated without drawing the others.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np

MATRIX_GATE = 0
MATRIX_UP = 1
MATRIX_DOWN = 2

# E4M3 codes 0x18 (= 2^-4) .. 0x48 (= 2^2), both ends included.
SCALE_CODE_LO = 0x18
SCALE_CODE_HI = 0x48


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    hidden: int       # H: K of gate/up, N of down
    inter: int        # I: N of gate/up, K of down
    experts: int      # E
    topk: int         # k
    tokens: int       # M
    router: str       # "uniform" | "zipf" | "hot"
    seed: int
    zipf_s: float = 1.1

    @property
    def pairs(self) -> int:
        return self.tokens * self.topk


# The five workloads: a tiny parity case, three decode shapes and one prefill.
CONFIGS: Dict[str, MoEConfig] = {
    "tiny": MoEConfig("tiny", 256, 512, 8, 2, 1, "uniform", 1000),
    "decode_m1": MoEConfig("decode_m1", 2048, 1536, 128, 8, 1, "uniform", 1001),
    "decode_m32": MoEConfig("decode_m32", 4096, 1536, 128, 8, 32, "zipf", 1002),
    "decode_m256": MoEConfig("decode_m256", 7168, 2048, 256, 8, 256, "uniform", 1003),
    "prefill_m8192": MoEConfig("prefill_m8192", 4096, 1536, 128, 8, 8192, "uniform", 1004),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round f32 values to BF16 (nearest, ties to even); return uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def matrix_shape(cfg: MoEConfig, matrix: int) -> Tuple[int, int]:
    """Logical [N, K] of one projection."""
    if matrix in (MATRIX_GATE, MATRIX_UP):
        return cfg.inter, cfg.hidden
    if matrix == MATRIX_DOWN:
        return cfg.hidden, cfg.inter
    raise ValueError(f"unknown matrix id {matrix}")


def draw_expert_weight(cfg: MoEConfig, matrix: int, expert: int) -> Tuple[np.ndarray, np.ndarray]:
    """Packed E2M1 bytes [N, K/2] and E4M3 scale codes [N, K/16] of one expert."""
    n, k = matrix_shape(cfg, matrix)
    rng = np.random.default_rng([cfg.seed, 1 + matrix, expert])
    packed = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    scale = rng.integers(SCALE_CODE_LO, SCALE_CODE_HI + 1, size=(n, k // 16), dtype=np.uint8)
    return packed, scale


def draw_shared_weight(cfg: MoEConfig, matrix: int) -> Tuple[np.ndarray, np.ndarray]:
    """Packed bytes and scale codes of the shared expert's projection ``matrix``.

    Same recipe and shapes as a routed expert, from a stream of its own.
    """
    n, k = matrix_shape(cfg, matrix)
    rng = np.random.default_rng([cfg.seed, 4 + matrix, 0])
    packed = rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    scale = rng.integers(SCALE_CODE_LO, SCALE_CODE_HI + 1, size=(n, k // 16), dtype=np.uint8)
    return packed, scale


def draw_routing(cfg: MoEConfig) -> Tuple[np.ndarray, np.ndarray]:
    """topk_ids int32 [M, k] and topk_weights f32 [M, k]."""
    m, e, k = cfg.tokens, cfg.experts, cfg.topk
    logits = np.random.default_rng([cfg.seed, 0, 1]).standard_normal((m, e))
    if cfg.router == "zipf":
        ranks = np.random.default_rng([cfg.seed, 0, 2]).permutation(e) + 1
        p = ranks.astype(np.float64) ** (-cfg.zipf_s)
        p /= p.sum()
        logits = logits + np.log(p)[None, :]
    elif cfg.router == "hot":
        # Every token prefers the first k experts: k experts carry M rows each,
        # which exercises experts far larger than any tile.
        logits = logits.copy()
        logits[:, :k] += 20.0
    elif cfg.router != "uniform":
        raise ValueError(f"unknown router {cfg.router!r}")
    z = logits - logits.max(axis=1, keepdims=True)
    prob = np.exp(z)
    prob /= prob.sum(axis=1, keepdims=True)
    # Stable sort of -prob: among equal probabilities the lower expert id wins.
    order = np.argsort(-prob, axis=1, kind="stable")[:, :k]
    w = np.take_along_axis(prob, order, axis=1)
    w = w / w.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def draw_activations(cfg: MoEConfig) -> np.ndarray:
    """x as BF16 bit patterns, uint16 [M, H]."""
    x = np.random.default_rng([cfg.seed, 0, 0]).standard_normal((cfg.tokens, cfg.hidden), dtype=np.float32)
    return f32_to_bf16_bits(x)


class MoEProblem:
    """One seeded instance of a workload.

    ``null_experts`` lists experts whose three weights are absent (the caller's
    NULL expert: one this rank does not own under expert parallelism).
    """

    def __init__(self, cfg: MoEConfig, null_experts=()):
        self.cfg = cfg
        self.x_bf16 = draw_activations(cfg)
        self.topk_ids, self.topk_weights = draw_routing(cfg)
        self.scale2 = np.full((3, cfg.experts), np.float32(1.0 / 448.0), dtype=np.float32)
        self.null_experts = frozenset(int(e) for e in null_experts)
        self._cache: Dict[Tuple[int, int], Tuple[np.ndarray, np.ndarray]] = {}

    def expert_weight(self, matrix: int, expert: int, cache: bool = False
                      ) -> Optional[Tuple[np.ndarray, np.ndarray, np.float32]]:
        """(packed, scale, weight_scale_2) of one expert, or None for a NULL expert."""
        if expert in self.null_experts:
            return None
        key = (matrix, expert)
        if key in self._cache:
            packed, scale = self._cache[key]
        else:
            packed, scale = draw_expert_weight(self.cfg, matrix, expert)
            if cache:
                self._cache[key] = (packed, scale)
        return packed, scale, self.scale2[matrix, expert]

    def shared_weight(self, matrix: int) -> Tuple[np.ndarray, np.ndarray, np.float32]:
        """(packed, scale, weight_scale_2) of the shared expert's projection."""
        packed, scale = draw_shared_weight(self.cfg, matrix)
        return packed, scale, np.float32(1.0 / 448.0)

    def stacked_weight(self, matrix: int) -> Tuple[np.ndarray, np.ndarray]:
        """All experts' bytes stacked: packed [E, N, K/2], scale [E, N, K/16].

        NULL experts hold zero bytes here; the caller passes a NULL pointer for them.
        """
        n, k = matrix_shape(self.cfg, matrix)
        e_count = self.cfg.experts
        packed = np.zeros((e_count, n, k // 2), dtype=np.uint8)
        scale = np.zeros((e_count, n, k // 16), dtype=np.uint8)
        for e in range(e_count):
            if e in self.null_experts:
                continue
            packed[e], scale[e] = draw_expert_weight(self.cfg, matrix, e)
        return packed, scale


def make_problem(cfg, null_experts=(), **overrides) -> MoEProblem:
    """Build a problem from a config name or a MoEConfig, with optional field overrides."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if overrides:
        cfg = dataclasses.replace(cfg, **overrides)
    return MoEProblem(cfg, null_experts=null_experts)
