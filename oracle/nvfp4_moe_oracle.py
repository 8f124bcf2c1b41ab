"""Plain fp64 CPU oracle of the grouped NVFP4 MoE expert forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` call this module.  The product
path (CUDA library + binding) never imports it, and it imports nothing from
the product package.  It is deliberately slow and obvious: numpy in float64,
the library matmul and stable argsort as its only primitives, no blocking and
no fusion.

Sources (rustdoc source pages of the "metrale" project; cited by page and item):

* metrale_model_arch/tp_shard/quant_shard.rs, layout comment at the top of the
  file: NVFP4 ``weight`` [N, K/2] u8 packed E2M1, ``weight_scale``
  [N, K/group] u8 E4M3, one f32 ``weight_scale_2``.
* metrale_model_layers/weight_map/quantized/transpose.rs,
  ``transpose_for_gemm``: the NVFP4 group is 16; the host fallback of
  ``transpose_for_gemm_gs`` is the byte loop that defines ``transpose_u8``.
* metrale_model_layers/layers/ops/nvfp4_moe_grouped.rs, module doc: rows are
  grouped by expert and the active experts listed (``moe_fp8_grouped_sort``);
  intermediates are laid out by sorted position; the router-weighted blend
  (``moe_weighted_sum_blend_fp8_grouped``) returns to token order.  Doc of
  ``moe_expert_gate_up_act_nvfp4_grouped``: the gate+up kernel writes the FP32
  product of SiLU(gate) and up, ``[positions, n]``.  Doc of
  ``moe_expert_down_act_nvfp4_grouped``: down runs over that product; rows of
  its output are sorted positions.
* metrale_model_arch/nemotron_moe/prefill_weights.rs, the shared-expert comment
  of ``prepare_prefill_weights``: the E4M3 cast saturates at 448, which fixes
  the E4M3 variant as the finite "FN" one (max 448, no infinities).
* metrale_model_layers/weight_map/expert.rs, ``ExpertWeight::null``: a NULL
  expert is skipped by the MoE kernels.
* nvfp4_moe_grouped.rs, doc of ``nvfp4_tc_lean_repack``: a negative or NaN
  block scale leaves the matrix unusable and is flagged at load time.
* transpose.rs, ``transpose_concat_for_gemm_gs`` / ``_padded`` and the host
  loops of ``transpose_impl``: several parts' twins side by side along N in a
  row pitch ``stride``, pad columns zero; group size 16 (NVFP4) or 32 (MXFP4).
* metrale_model_arch/tp_shard/quant_shard.rs, ``shard_quantized_nvfp4``:
  column-parallel keeps a rank's rows of packed and scale, row-parallel a
  rank's K slice of both; weight_scale_2 is replicated.
* metrale_model_arch/nemotron_moe/prefill_weights.rs,
  ``prepare_prefill_weights``: the routed experts of that model have only an
  up and a down projection (no gate); the forward of such a non-gated expert
  is act = f(x Wu^T), y = act Wd^T.  The pages do not name f: it is a
  parameter here (ReLU squared or SiLU).
* nvfp4_moe_grouped.rs, docs of the two projection launchers: the shared
  expert runs in the same gate+up and down launches as the routed experts,
  over every token, one row per token, with its own weights; its SiLU product
  and down output (``sh_act``, ``sh_down_out``) are laid out by token.

Readings where the pages are silent (each also listed in the design notes):

* nibble order: the low nibble of byte j holds k = 2j, the high nibble k = 2j+1;
* E2M1 and E4M3 follow the OCP 8-bit / MX element definitions; the two E4M3
  NaN codes 0x7F and 0xFF are rejected (ValueError);
* the weight value is E2M1(code) * E4M3(scale of its 16-block) * weight_scale_2;
* gate and up are not rounded to BF16 before SiLU: the product is formed from
  the exact sums ("kept in FP32" on the GPU, fp64 here);
* SiLU(z) = z / (1 + exp(-z));
* sort ties are broken by pair id (pair p = token * k + slot), so the sort is
  stable and unique; ``active_experts`` is ascending and padded with -1;
  an expert id outside [0, E) drops its pair (pair_pos = -1, contributes 0);
* a NULL expert's rows of ``act`` and ``y`` are zero;
* the shared expert has the routed experts' shapes (the fused launches take
  one width pair for both) and its down output joins the token's sum with a
  per-token weight, 1 unless the caller gives one;
* a "negative" block scale is one whose value is below zero: -0 (0x80) is
  valid.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import math
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "E2M1_GROUP",
    "e2m1_value",
    "e2m1_table",
    "e4m3_value",
    "e4m3_table",
    "bf16_bits_to_f64",
    "dequantize_nvfp4",
    "silu",
    "route_sort",
    "gate_up_silu",
    "down_proj",
    "blend",
    "moe_forward",
    "moe_forward_tokens",
    "transpose_u8",
    "shared_expert",
    "moe_forward_shared",
    "relu2",
    "ACTIVATIONS",
    "up_act",
    "moe_forward_nongated",
    "append_shared_routing",
    "count_bad_scales",
    "shard_nvfp4",
    "expert_owner_range",
    "transpose_concat",
    "RouteSort",
]

# NVFP4 block-scale group (transpose.rs, transpose_for_gemm).
E2M1_GROUP = 16


# --------------------------------------------------------------------------- #
# Element formats
# --------------------------------------------------------------------------- #

def e2m1_value(code: int) -> float:
    """Value of one 4-bit E2M1 code: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.

    Exponent field 0 is subnormal: mantissa * 2^-1.  No NaN or infinity codes.
    """
    if not 0 <= code <= 15:
        raise ValueError(f"E2M1 code out of range: {code}")
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        mag = man * 0.5
    else:
        mag = 2.0 ** (exp - 1) * (1.0 + man / 2.0)
    return sign * mag


def e2m1_table() -> np.ndarray:
    """All 16 E2M1 codes decoded, float64 [16]."""
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e4m3_value(code: int) -> float:
    """Value of one E4M3 (FN) code: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.

    Exponent field 0 is subnormal: mantissa/8 * 2^-6.  The codes 0x7F and 0xFF
    are NaN and are rejected with ValueError; there are no infinities, so the
    largest finite magnitude is 0x7E = 448.
    """
    if not 0 <= code <= 255:
        raise ValueError(f"E4M3 code out of range: {code}")
    if code & 0x7F == 0x7F:
        raise ValueError(f"E4M3 code 0x{code:02X} is NaN")
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0:
        mag = (man / 8.0) * 2.0 ** -6
    else:
        mag = 2.0 ** (exp - 7) * (1.0 + man / 8.0)
    return sign * mag


def e4m3_table() -> np.ndarray:
    """All 256 E4M3 codes decoded, float64 [256]; the two NaN codes hold NaN."""
    out = np.empty(256, dtype=np.float64)
    for c in range(256):
        try:
            out[c] = e4m3_value(c)
        except ValueError:
            out[c] = np.nan
    return out


_E2M1 = e2m1_table()
_E4M3 = e4m3_table()


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) to float64, exactly."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def dequantize_nvfp4(packed: np.ndarray, scale: np.ndarray, scale2) -> np.ndarray:
    """Dense float64 [N, K] of one NVFP4 weight.

    W[n, k] = E2M1(nibble k of row n) * E4M3(scale[n, k // 16]) * weight_scale_2,
    nibble k being the low nibble of packed[n, k // 2] for even k and the high
    nibble for odd k.  A NaN scale code raises ValueError.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    scale = np.asarray(scale, dtype=np.uint8)
    n, half_k = packed.shape
    k = 2 * half_k
    if scale.shape != (n, k // E2M1_GROUP):
        raise ValueError(f"scale shape {scale.shape} does not match packed {packed.shape}")
    if np.any((scale & 0x7F) == 0x7F):
        raise ValueError("E4M3 block scale holds a NaN code")
    codes = np.empty((n, k), dtype=np.uint8)
    codes[:, 0::2] = packed & 0x0F
    codes[:, 1::2] = packed >> 4
    w = _E2M1[codes]
    w *= np.repeat(_E4M3[scale], E2M1_GROUP, axis=1)
    w *= float(np.float32(scale2))
    return w


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z / (1 + exp(-z)), float64."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


# --------------------------------------------------------------------------- #
# Step 1: group the routed pairs by expert
# --------------------------------------------------------------------------- #

class RouteSort:
    """Result of :func:`route_sort`.

    expert_offsets  int32 [E+1]  exclusive prefix of per-expert pair counts
    sorted_pair_ids int32 [P]    pair ids (token * k + slot) in sorted order;
                                 only the first expert_offsets[E] are defined
    pair_pos        int32 [P]    sorted position of each pair, -1 if dropped
    active_experts  int32 [E]    experts with at least one pair, ascending, -1 padded
    active_count    int          number of such experts
    dropped         int          pairs whose expert id was outside [0, E)
    """

    def __init__(self, expert_offsets, sorted_pair_ids, pair_pos, active_experts,
                 active_count, dropped):
        self.expert_offsets = expert_offsets
        self.sorted_pair_ids = sorted_pair_ids
        self.pair_pos = pair_pos
        self.active_experts = active_experts
        self.active_count = active_count
        self.dropped = dropped


def _stable_order(keys: np.ndarray) -> np.ndarray:
    """Indices that sort ``keys`` ascending, equal keys kept in index order."""
    return np.argsort(keys, kind="stable")


def route_sort(topk_ids: np.ndarray, num_experts: int) -> RouteSort:
    """Order the routed (token, expert) pairs by expert, ties by pair id.

    Follows the grouping that nvfp4_moe_grouped.rs (module doc) takes from
    ``moe_fp8_grouped_sort``: rows grouped by expert, the active experts listed,
    intermediates laid out by sorted position.
    """
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    p_total = ids.size
    valid = (ids >= 0) & (ids < num_experts)
    valid_pairs = np.nonzero(valid)[0]
    order = valid_pairs[_stable_order(ids[valid_pairs])]
    counts = np.bincount(ids[valid_pairs], minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pair_ids = np.full(p_total, -1, dtype=np.int32)
    sorted_pair_ids[: order.size] = order
    pair_pos = np.full(p_total, -1, dtype=np.int32)
    pair_pos[order] = np.arange(order.size, dtype=np.int32)
    active = np.nonzero(counts > 0)[0]
    active_experts = np.full(num_experts, -1, dtype=np.int32)
    active_experts[: active.size] = active
    return RouteSort(offsets.astype(np.int32), sorted_pair_ids, pair_pos, active_experts,
                     int(active.size), int(p_total - order.size))


# --------------------------------------------------------------------------- #
# Steps 2-4
# --------------------------------------------------------------------------- #

WeightFn = Callable[[int], Optional[Tuple[np.ndarray, np.ndarray, float]]]


def _dense(weight_fn: WeightFn, expert: int) -> Optional[np.ndarray]:
    w = weight_fn(expert)
    if w is None:
        return None
    packed, scale, s2 = w
    return dequantize_nvfp4(packed, scale, s2)


def gate_up_silu(x_bf16: np.ndarray, topk: int, rs: RouteSort,
                 gate_fn: WeightFn, up_fn: WeightFn, inter: int) -> np.ndarray:
    """act [P, I] by sorted position: SiLU(x Wg^T) * (x Wu^T), float64.

    nvfp4_moe_grouped.rs, ``moe_expert_gate_up_act_nvfp4_grouped``: for each
    active expert and each of its rows (a pair, whose token is pair // k), the
    gate and up projections of that token's row and their SiLU product.  Rows of
    a NULL expert are zero.  Rows past expert_offsets[E] are zero.
    """
    x = bf16_bits_to_f64(x_bf16)
    p_total = rs.sorted_pair_ids.size
    act = np.zeros((p_total, inter), dtype=np.float64)
    for a in range(rs.active_count):
        e = int(rs.active_experts[a])
        lo, hi = int(rs.expert_offsets[e]), int(rs.expert_offsets[e + 1])
        wg, wu = _dense(gate_fn, e), _dense(up_fn, e)
        if wg is None or wu is None:
            continue
        tokens = rs.sorted_pair_ids[lo:hi] // topk
        xe = x[tokens]
        g = xe @ wg.T
        u = xe @ wu.T
        act[lo:hi] = silu(g) * u
    return act


def down_proj(act: np.ndarray, rs: RouteSort, down_fn: WeightFn, hidden: int) -> np.ndarray:
    """y [P, H] by sorted position: act Wd^T per expert, float64.

    nvfp4_moe_grouped.rs, ``moe_expert_down_act_nvfp4_grouped``.
    """
    p_total = act.shape[0]
    y = np.zeros((p_total, hidden), dtype=np.float64)
    for a in range(rs.active_count):
        e = int(rs.active_experts[a])
        lo, hi = int(rs.expert_offsets[e]), int(rs.expert_offsets[e + 1])
        wd = _dense(down_fn, e)
        if wd is None:
            continue
        y[lo:hi] = act[lo:hi] @ wd.T
    return y


def blend(y: np.ndarray, topk_weights: np.ndarray, pair_pos: np.ndarray) -> np.ndarray:
    """out [M, H] = sum over slots s of w[t, s] * y[pair_pos[t*k + s]], float64.

    The router-weighted blend back into token order named in the module doc of
    nvfp4_moe_grouped.rs (``moe_weighted_sum_blend_fp8_grouped``).  A dropped
    pair (pair_pos = -1) contributes nothing.
    """
    w = np.asarray(topk_weights, dtype=np.float64)
    m, k = w.shape
    out = np.zeros((m, y.shape[1]), dtype=np.float64)
    for t in range(m):
        for s in range(k):
            pos = int(pair_pos[t * k + s])
            if pos >= 0:
                out[t] += w[t, s] * y[pos]
    return out


def moe_forward(x_bf16, topk_ids, topk_weights, num_experts, gate_fn, up_fn, down_fn,
                hidden: int, inter: int) -> Dict[str, object]:
    """The four steps in order; returns every intermediate."""
    topk = np.asarray(topk_ids).shape[1]
    rs = route_sort(topk_ids, num_experts)
    act = gate_up_silu(x_bf16, topk, rs, gate_fn, up_fn, inter)
    y = down_proj(act, rs, down_fn, hidden)
    out = blend(y, topk_weights, rs.pair_pos)
    return {"sort": rs, "act": act, "y": y, "out": out}


def moe_forward_tokens(x_bf16, topk_ids, topk_weights, num_experts, gate_fn, up_fn, down_fn,
                       tokens: Sequence[int], hidden: int) -> np.ndarray:
    """out rows for the listed tokens only, computed token by token, float64.

    The same expert forward written per token: each routed slot of a token adds
    the expert's gated MLP of that token's row, weighted by its router weight.
    It shares no grouping with :func:`moe_forward`, so the two check each other,
    and it lets a full-size problem be checked on a sample of tokens.  Experts
    are visited one at a time (each dequantised once, then released), so only
    one expert's dense weights are held at a time.
    """
    x = bf16_bits_to_f64(x_bf16)
    ids = np.asarray(topk_ids)
    w = np.asarray(topk_weights, dtype=np.float64)
    out = np.zeros((len(tokens), hidden), dtype=np.float64)
    uses: Dict[int, List[Tuple[int, int, int]]] = {}
    for i, t in enumerate(tokens):
        for s in range(ids.shape[1]):
            e = int(ids[t, s])
            if 0 <= e < num_experts:
                uses.setdefault(e, []).append((i, int(t), s))
    for e in sorted(uses):
        mats = [_dense(fn, e) for fn in (gate_fn, up_fn, down_fn)]
        if any(m is None for m in mats):
            continue
        wg, wu, wd = mats
        for i, t, s in uses[e]:
            h = silu(wg @ x[t]) * (wu @ x[t])
            out[i] += w[t, s] * (wd @ h)
    return out


# --------------------------------------------------------------------------- #
# Non-gated experts (up and down only)
# --------------------------------------------------------------------------- #

def relu2(z: np.ndarray) -> np.ndarray:
    """Squared ReLU: max(z, 0)^2, float64."""
    z = np.asarray(z, dtype=np.float64)
    return np.square(np.maximum(z, 0.0))


# Activations of a non-gated expert, by name.
ACTIVATIONS = {"relu2": relu2, "silu": silu}


def up_act(x_bf16: np.ndarray, topk: int, rs: RouteSort, up_fn: WeightFn, inter: int,
           activation: str) -> np.ndarray:
    """act [P, I] by sorted position: f(x Wu^T) for a non-gated expert, float64.

    prefill_weights.rs, ``prepare_prefill_weights``: the experts hold only up
    and down.  ``activation`` names f (a key of ACTIVATIONS).  Rows of a NULL
    expert, and rows past expert_offsets[E], are zero.
    """
    f = ACTIVATIONS[activation]
    x = bf16_bits_to_f64(x_bf16)
    p_total = rs.sorted_pair_ids.size
    act = np.zeros((p_total, inter), dtype=np.float64)
    for a in range(rs.active_count):
        e = int(rs.active_experts[a])
        lo, hi = int(rs.expert_offsets[e]), int(rs.expert_offsets[e + 1])
        wu = _dense(up_fn, e)
        if wu is None:
            continue
        tokens = rs.sorted_pair_ids[lo:hi] // topk
        act[lo:hi] = f(x[tokens] @ wu.T)
    return act


def moe_forward_nongated(x_bf16, topk_ids, topk_weights, num_experts, up_fn, down_fn,
                         hidden: int, inter: int, activation: str) -> Dict[str, object]:
    """The four steps for non-gated experts: sort, act = f(x Wu^T), down, blend."""
    topk = np.asarray(topk_ids).shape[1]
    rs = route_sort(topk_ids, num_experts)
    act = up_act(x_bf16, topk, rs, up_fn, inter, activation)
    y = down_proj(act, rs, down_fn, hidden)
    out = blend(y, topk_weights, rs.pair_pos)
    return {"sort": rs, "act": act, "y": y, "out": out}


# --------------------------------------------------------------------------- #
# Shared expert
# --------------------------------------------------------------------------- #

Weight = Tuple[np.ndarray, np.ndarray, float]


def shared_expert(x_bf16, gate: Weight, up: Weight, down: Weight) -> Tuple[np.ndarray, np.ndarray]:
    """(sh_act [M, I], sh_out [M, H]) of the shared expert, float64, rows by token.

    The launcher docs of nvfp4_moe_grouped.rs give the shared expert one row per
    token in both projections: sh_act[t] = SiLU(Wg x_t) * (Wu x_t) and
    sh_out[t] = Wd sh_act[t].
    """
    x = bf16_bits_to_f64(x_bf16)
    wg, wu, wd = (dequantize_nvfp4(*w) for w in (gate, up, down))
    h = silu(x @ wg.T) * (x @ wu.T)
    return h, h @ wd.T


def moe_forward_shared(x_bf16, topk_ids, topk_weights, num_experts, gate_fn, up_fn, down_fn,
                       hidden: int, inter: int, shared: Tuple[Weight, Weight, Weight],
                       shared_weights: Optional[np.ndarray] = None,
                       routed: Optional[Dict[str, object]] = None) -> Dict[str, object]:
    """The routed forward plus the shared expert: out[t] += c_t * sh_out[t].

    c_t is ``shared_weights[t]``, or 1 for every token when it is None.
    ``routed``, if given, is the result of :func:`moe_forward` on the same
    routed inputs, already computed (the weight functions are then unused).
    """
    res = dict(routed) if routed is not None else moe_forward(
        x_bf16, topk_ids, topk_weights, num_experts, gate_fn, up_fn, down_fn, hidden, inter)
    sh_act, sh_out = shared_expert(x_bf16, *shared)
    m = sh_out.shape[0]
    c = (np.ones(m) if shared_weights is None
         else np.asarray(shared_weights, dtype=np.float64).reshape(m))
    res["sh_act"] = sh_act
    res["sh_out"] = sh_out
    res["out"] = res["out"] + c[:, None] * sh_out
    return res


def append_shared_routing(topk_ids, topk_weights, num_experts: int, shared_rows: int,
                          shared_weights: Optional[np.ndarray] = None
                          ) -> Tuple[np.ndarray, np.ndarray]:
    """Routing [M, k+1] that sends every token to the shared expert as one more slot.

    Slot k of token t names expert num_experts + t // shared_rows: the shared
    expert is listed once per block of ``shared_rows`` tokens, each listing a
    table entry that holds the shared weights, so the grouped launches give it
    as many row groups as it has token blocks.  Its weight is
    ``shared_weights[t]`` (1 when None).  Slots 0..k-1 are copied unchanged.
    """
    ids = np.asarray(topk_ids, dtype=np.int32)
    w = np.asarray(topk_weights, dtype=np.float32)
    m, k = ids.shape
    if shared_rows < 1:
        raise ValueError("shared_rows must be >= 1")
    ids_out = np.empty((m, k + 1), dtype=np.int32)
    w_out = np.empty((m, k + 1), dtype=np.float32)
    for t in range(m):
        ids_out[t, :k] = ids[t]
        w_out[t, :k] = w[t]
        ids_out[t, k] = num_experts + t // shared_rows
        w_out[t, k] = 1.0 if shared_weights is None else np.float32(shared_weights[t])
    return ids_out, w_out


# --------------------------------------------------------------------------- #
# Load-time scale check
# --------------------------------------------------------------------------- #

def count_bad_scales(scale_codes: np.ndarray) -> int:
    """Number of E4M3 block-scale codes whose value is NaN or below zero.

    nvfp4_moe_grouped.rs, doc of ``nvfp4_tc_lean_repack``: a negative or NaN
    block scale makes the matrix unusable.  "Negative" is read as a value
    below zero, so -0 (0x80) passes.
    """
    v = _E4M3[np.asarray(scale_codes, dtype=np.uint8).reshape(-1)]
    return int(np.count_nonzero(np.isnan(v) | (v < 0.0)))


# --------------------------------------------------------------------------- #
# Sharding across ranks
# --------------------------------------------------------------------------- #

def shard_nvfp4(packed: np.ndarray, scale: np.ndarray, kind: str, rank: int, tp: int
                ) -> Tuple[np.ndarray, np.ndarray]:
    """This rank's part of one NVFP4 weight (packed [N, K/2], scale [N, K/16]).

    metrale_model_arch/tp_shard/quant_shard.rs, ``shard_quantized_nvfp4``:
    "column" (column-parallel) keeps rows rank*N/tp .. (rank+1)*N/tp - 1 of both
    tensors; "row" (row-parallel) keeps, in every row, the rank's K/2/tp
    packed bytes and K/16/tp scale bytes; "replicated" (or tp <= 1) keeps all.
    weight_scale_2 is per tensor and stays the same on every rank.  The page's
    divisibility rules raise ValueError.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    scale = np.asarray(scale, dtype=np.uint8)
    n, half_k = packed.shape
    k = 2 * half_k
    if k % E2M1_GROUP:
        raise ValueError("K is not a multiple of the group size")
    groups = k // E2M1_GROUP
    if tp <= 1 or kind == "replicated":
        return packed.copy(), scale.copy()
    if not 0 <= rank < tp:
        raise ValueError("rank out of range")
    if kind == "column":
        if n % tp:
            raise ValueError("N not divisible by tp")
        rows = n // tp
        return (packed[rank * rows:(rank + 1) * rows].copy(),
                scale[rank * rows:(rank + 1) * rows].copy())
    if kind == "row":
        if k % tp or half_k % tp or groups % tp:
            raise ValueError("K, K/2 or K/16 not divisible by tp")
        wb, sb = half_k // tp, groups // tp
        return (packed[:, rank * wb:(rank + 1) * wb].copy(),
                scale[:, rank * sb:(rank + 1) * sb].copy())
    raise ValueError(f"unknown shard kind {kind!r}")


def expert_owner_range(num_experts: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi): the experts rank owns under expert parallelism, in contiguous blocks.

    The pages fix only that a rank runs the experts it does not own as NULL
    experts (expert.rs, ``ExpertWeight::null``); the reading taken here is
    blocks of consecutive ids whose sizes differ by at most one:
    lo = rank * E // world.
    """
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * num_experts // world, (rank + 1) * num_experts // world


# --------------------------------------------------------------------------- #
# Load-time twin builder
# --------------------------------------------------------------------------- #

def transpose_u8(src: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Byte transpose [rows, cols] -> [cols, rows].

    The host fallback of ``transpose_for_gemm_gs`` (transpose.rs) defines it:
    t[j * rows + i] = b[i * cols + j].  Written as that double loop; it is only
    run on small inputs.
    """
    b = np.asarray(src, dtype=np.uint8).reshape(-1)
    if b.size != rows * cols:
        raise ValueError("size mismatch")
    t = np.empty(rows * cols, dtype=np.uint8)
    for i in range(rows):
        for j in range(cols):
            t[j * rows + i] = b[i * cols + j]
    return t.reshape(cols, rows)


def transpose_concat(parts: Sequence[Tuple[np.ndarray, np.ndarray]], k: int, group_size: int,
                     stride: int) -> Tuple[np.ndarray, np.ndarray]:
    """Transposed twins of several NVFP4 weights sharing K, side by side along N.

    transpose.rs, ``transpose_impl`` (behind ``transpose_concat_for_gemm_gs``
    and ``transpose_concat_for_gemm_padded``), host path: part p with n_p rows
    lands in columns n_off .. n_off + n_p - 1 of a [K/2, stride] packed twin
    and a [K/group_size, stride] scale twin, n_off being the rows of the parts
    before it; columns past the last part are zero.  One part with stride = N
    is ``transpose_for_gemm_gs``.  Written as the page's byte loops: small
    inputs only.
    """
    if not parts:
        raise ValueError("empty parts")
    half_k, groups = k // 2, k // group_size
    n_total = sum(p.shape[0] for p, _ in parts)
    if stride < n_total:
        raise ValueError("stride below the total rows")
    w = np.zeros(half_k * stride, dtype=np.uint8)
    sc = np.zeros(groups * stride, dtype=np.uint8)
    n_off = 0
    for packed, scale in parts:
        packed = np.asarray(packed, dtype=np.uint8)
        scale = np.asarray(scale, dtype=np.uint8)
        n = packed.shape[0]
        if packed.shape != (n, half_k) or scale.shape != (n, groups):
            raise ValueError("part shape does not match k / group_size")
        pb, sb = packed.reshape(-1), scale.reshape(-1)
        for i in range(n):
            for j in range(half_k):
                w[j * stride + n_off + i] = pb[i * half_k + j]
            for j in range(groups):
                sc[j * stride + n_off + i] = sb[i * groups + j]
        n_off += n
    return w.reshape(half_k, stride), sc.reshape(groups, stride)


def relative_l2(got: np.ndarray, ref: np.ndarray) -> float:
    """||got - ref||_2 / ||ref||_2 (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(got - ref))
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return num / den


__all__.append("relative_l2")
