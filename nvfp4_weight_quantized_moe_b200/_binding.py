"""ctypes binding of the C ABI in include/nvfp4_moe.h.

Argument marshalling only: each function checks dtypes, devices and
contiguity of the torch tensors it is given, passes their device pointers and
sizes to the library entry point of the same name, and raises
``NVFP4MoEError`` on a non-zero status.  Every step of the forward runs in
the library's CUDA kernels; there is no fallback.  If the library is missing
the import fails.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libnvfp4moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m nvfp4_weight_quantized_moe_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

c_void_p = ctypes.c_void_p
c_u32 = ctypes.c_uint32
c_int = ctypes.c_int


class ExpertTables(ctypes.Structure):
    """nvfp4_expert_tables: three device arrays of length num_experts."""
    _fields_ = [("packed_ptrs", c_void_p), ("scale_ptrs", c_void_p), ("scale2", c_void_p)]


class LaunchOpts(ctypes.Structure):
    """nvfp4_moe_launch_opts."""
    _fields_ = [("path", ctypes.c_int32), ("split", ctypes.c_int32), ("tiles", ctypes.c_int32),
                ("depth", ctypes.c_int32), ("staging", ctypes.c_int32)]


class Buffers(ctypes.Structure):
    """nvfp4_moe_buffers: the device outputs and intermediates of one forward."""
    _fields_ = [("expert_offsets", c_void_p), ("sorted_pair_ids", c_void_p), ("pair_pos", c_void_p),
                ("active_experts", c_void_p), ("active_count", c_void_p), ("status", c_void_p),
                ("act", c_void_p), ("y", c_void_p), ("out_f32", c_void_p), ("out_bf16", c_void_p)]


PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2
# nvfp4_moe_activation: the activation of a non-gated expert.
ACTIVATIONS = {"relu2": 1, "silu": 2}
SHARD_COLUMN, SHARD_ROW = 0, 1

_sig = {
    "nvfp4_moe_route_sort": (c_int, [c_void_p, c_u32, c_u32, c_u32, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p]),
    "nvfp4_moe_gate_up_silu": (c_int, [c_void_p, ExpertTables, ExpertTables, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_u32, c_u32, c_u32, c_u32,
                                       c_u32, c_void_p]),
    "nvfp4_moe_gate_up_silu_ex": (c_int, [c_void_p, ExpertTables, ExpertTables, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_u32, c_u32, c_u32, c_u32,
                                          c_u32, ctypes.POINTER(LaunchOpts), c_void_p]),
    "nvfp4_moe_down": (c_int, [c_void_p, ExpertTables, c_void_p, c_void_p, c_void_p, c_void_p,
                               c_u32, c_u32, c_u32, c_u32, c_u32, c_void_p]),
    "nvfp4_moe_down_ex": (c_int, [c_void_p, ExpertTables, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_u32, c_u32, c_u32, c_u32, c_u32, ctypes.POINTER(LaunchOpts),
                                  c_void_p]),
    "nvfp4_moe_blend": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_u32, c_u32,
                                c_u32, c_void_p]),
    "nvfp4_moe_transpose_u8": (c_int, [c_void_p, c_void_p, c_u32, c_u32, c_void_p]),
    "nvfp4_moe_gate_up_silu_ws": (c_int, [c_void_p, ExpertTables, ExpertTables, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_u32, c_u32, c_u32, c_u32,
                                          c_u32, c_u32, ctypes.POINTER(LaunchOpts), c_void_p,
                                          ctypes.c_size_t, c_void_p]),
    "nvfp4_moe_down_ws": (c_int, [c_void_p, ExpertTables, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_u32, c_u32, c_u32, c_u32, c_u32, c_u32, ctypes.POINTER(LaunchOpts),
                                  c_void_p, ctypes.c_size_t, c_void_p]),
    "nvfp4_moe_gate_up_silu_noalloc": (c_int, [c_void_p, ExpertTables, ExpertTables, c_void_p,
                                               c_void_p, c_void_p, c_void_p, c_void_p, c_u32,
                                               c_u32, c_u32, c_u32, c_u32, c_u32, c_void_p]),
    "nvfp4_moe_forward": (c_int, [c_void_p, c_void_p, c_void_p, ExpertTables, ExpertTables,
                                  ExpertTables, ctypes.POINTER(Buffers), c_u32, c_u32, c_u32, c_u32,
                                  c_u32, ctypes.POINTER(LaunchOpts), c_void_p, ctypes.c_size_t,
                                  c_void_p]),
    "nvfp4_moe_up_act": (c_int, [c_void_p, ExpertTables, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_u32, c_u32, c_u32, c_u32, c_u32, c_int,
                                 ctypes.POINTER(LaunchOpts), c_void_p]),
    "nvfp4_moe_up_act_ws": (c_int, [c_void_p, ExpertTables, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_u32, c_u32, c_u32, c_u32, c_u32, c_u32, c_int,
                                    ctypes.POINTER(LaunchOpts), c_void_p, ctypes.c_size_t, c_void_p]),
    "nvfp4_moe_forward_nongated": (c_int, [c_void_p, c_void_p, c_void_p, ExpertTables, ExpertTables,
                                           ctypes.POINTER(Buffers), c_u32, c_u32, c_u32, c_u32, c_u32,
                                           c_int, ctypes.POINTER(LaunchOpts), c_void_p,
                                           ctypes.c_size_t, c_void_p]),
    "nvfp4_moe_append_shared": (c_int, [c_void_p, c_void_p, c_void_p, c_u32, c_u32, c_u32, c_u32,
                                        c_void_p, c_void_p, c_void_p]),
    "nvfp4_moe_shared_slots": (c_u32, [c_u32, c_u32]),
    "nvfp4_moe_check_scales": (c_int, [ExpertTables, c_u32, c_u32, c_u32, c_void_p, c_void_p]),
    "nvfp4_moe_transpose_concat": (c_int, [ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                           ctypes.POINTER(c_u32), c_u32, c_u32, c_u32, c_u32,
                                           c_void_p, c_void_p, c_void_p]),
    "nvfp4_moe_shard_nvfp4": (c_int, [c_void_p, c_void_p, c_u32, c_u32, c_u32, c_int, c_u32, c_u32,
                                      c_void_p, c_void_p, c_void_p]),
    "nvfp4_moe_workspace_bytes": (ctypes.c_size_t, [c_u32, c_u32, c_u32, c_u32]),
    "nvfp4_moe_device_error": (c_int, [c_int]),
    "nvfp4_moe_wait_selftest": (c_int, [c_u32, c_int, c_void_p]),
    "nvfp4_moe_active_cap": (c_u32, [c_u32, c_u32]),
    "nvfp4_moe_status_string": (ctypes.c_char_p, [c_int]),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class NVFP4MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.nvfp4_moe_status_string(status).decode()
        super().__init__(f"{fn} returned {status} ({msg})")
        self.status = status


def exported_symbols():
    """Names the binding resolves in the library."""
    return sorted(_sig)


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise NVFP4MoEError(fn, status)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _opts(path=0, split=0, tiles=0, depth=0, staging=0):
    if not (path or split or tiles or depth or staging):
        return None
    return ctypes.byref(LaunchOpts(path, split, tiles, depth, staging))


def active_cap(num_experts: int, num_pairs: int) -> int:
    return int(_lib.nvfp4_moe_active_cap(num_experts, num_pairs))


def route_sort(topk_ids, num_experts, expert_offsets, sorted_pair_ids, pair_pos,
               active_experts, active_count, status=None, stream=None) -> None:
    m, k = topk_ids.shape
    _check("nvfp4_moe_route_sort", _lib.nvfp4_moe_route_sort(
        _ptr(topk_ids, torch.int32, "topk_ids"), m, k, num_experts,
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(sorted_pair_ids, torch.int32, "sorted_pair_ids"),
        _ptr(pair_pos, torch.int32, "pair_pos"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        _ptr(status, torch.int32, "status"), _stream(stream)))


def gate_up_silu(x, gate: ExpertTables, up: ExpertTables, act, expert_offsets, sorted_pair_ids,
                 active_experts, active_count, n_inter, k_hidden, cap, num_tokens, topk,
                 path=0, split=0, tiles=0, depth=0, staging=0, stream=None) -> None:
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    _check("nvfp4_moe_gate_up_silu_ex", _lib.nvfp4_moe_gate_up_silu_ex(
        _ptr(x, None, "x"), gate, up, _ptr(act, torch.float32, "act"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(sorted_pair_ids, torch.int32, "sorted_pair_ids"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_inter, k_hidden, cap, num_tokens, topk, _opts(path, split, tiles, depth, staging),
        _stream(stream)))


def down(act, down_w: ExpertTables, y, expert_offsets, active_experts, active_count,
         n_hidden, k_inter, cap, num_tokens, topk, path=0, split=0, tiles=0, depth=0, staging=0,
         stream=None) -> None:
    _check("nvfp4_moe_down_ex", _lib.nvfp4_moe_down_ex(
        _ptr(act, torch.float32, "act"), down_w, _ptr(y, torch.float32, "y"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_hidden, k_inter, cap, num_tokens, topk, _opts(path, split, tiles, depth, staging),
        _stream(stream)))


def blend(y, topk_weights, pair_pos, out_f32, out_bf16=None, stream=None) -> None:
    m, k = topk_weights.shape
    hidden = out_f32.shape[1]
    _check("nvfp4_moe_blend", _lib.nvfp4_moe_blend(
        _ptr(y, torch.float32, "y"), _ptr(topk_weights, torch.float32, "topk_weights"),
        _ptr(pair_pos, torch.int32, "pair_pos"), _ptr(out_f32, torch.float32, "out_f32"),
        _ptr(out_bf16, None, "out_bf16"), m, k, hidden, _stream(stream)))


def transpose_u8(src, dst, stream=None) -> None:
    rows, cols = src.shape
    if tuple(dst.shape) != (cols, rows):
        raise ValueError("dst must be [cols, rows]")
    _check("nvfp4_moe_transpose_u8", _lib.nvfp4_moe_transpose_u8(
        _ptr(src, torch.uint8, "src"), _ptr(dst, torch.uint8, "dst"), rows, cols, _stream(stream)))


def shared_slots(num_tokens: int, shared_rows: int) -> int:
    """Table entries the shared expert takes: ceil(num_tokens / shared_rows)."""
    return int(_lib.nvfp4_moe_shared_slots(num_tokens, shared_rows))


def append_shared(topk_ids, topk_weights, num_experts, shared_rows, ids_out, weights_out,
                  shared_weights=None, stream=None) -> None:
    """nvfp4_moe_append_shared: routing [M, k+1] with the shared expert as slot k."""
    m, k = topk_ids.shape
    if tuple(ids_out.shape) != (m, k + 1) or tuple(weights_out.shape) != (m, k + 1):
        raise ValueError("ids_out and weights_out must be [M, topk + 1]")
    if tuple(topk_weights.shape) != (m, k):
        raise ValueError("topk_weights must be [M, topk]")
    if shared_weights is not None and shared_weights.numel() != m:
        raise ValueError("shared_weights must hold one value per token")
    _check("nvfp4_moe_append_shared", _lib.nvfp4_moe_append_shared(
        _ptr(topk_ids, torch.int32, "topk_ids"), _ptr(topk_weights, torch.float32, "topk_weights"),
        _ptr(shared_weights, torch.float32, "shared_weights"), m, k, num_experts, shared_rows,
        _ptr(ids_out, torch.int32, "ids_out"), _ptr(weights_out, torch.float32, "weights_out"),
        _stream(stream)))


def check_scales(tables: ExpertTables, num_experts, n, k, bad, stream=None) -> None:
    """nvfp4_moe_check_scales: add each expert's count of NaN / negative scale codes to bad."""
    if bad.numel() < num_experts:
        raise ValueError("bad must hold num_experts counters")
    if bad.dtype not in (torch.int32, torch.uint32):
        raise TypeError("bad: expected 32-bit counters")
    _check("nvfp4_moe_check_scales", _lib.nvfp4_moe_check_scales(
        tables, num_experts, n, k, _ptr(bad, None, "bad"), _stream(stream)))


def transpose_concat(parts, group_size: int = 16, stride: Optional[int] = None, stream=None):
    """nvfp4_moe_transpose_concat: the [K/2, stride] and [K/group_size, stride] twins of
    ``parts`` (a list of (packed [n, K/2], scale [n, K/group_size]) device tensors)
    side by side, pad columns zero; ``stride`` defaults to the total rows."""
    if not parts:
        raise ValueError("empty parts")
    half_k = parts[0][0].shape[1]
    k = 2 * half_k
    rows = [int(p.shape[0]) for p, _ in parts]
    for p, sc in parts:
        if p.shape[1] != half_k or tuple(sc.shape) != (p.shape[0], k // group_size):
            raise ValueError("every part must be [n, K/2] and [n, K/group_size]")
    stride = sum(rows) if stride is None else int(stride)
    dev = parts[0][0].device
    w = torch.empty((half_k, stride), dtype=torch.uint8, device=dev)
    sc_out = torch.empty((k // group_size, stride), dtype=torch.uint8, device=dev)
    transpose_concat_into(parts, group_size, w, sc_out, stream=stream)
    return w, sc_out


def transpose_concat_into(parts, group_size: int, packed_out, scale_out, stream=None) -> None:
    """nvfp4_moe_transpose_concat into caller-allocated [K/2, stride] and
    [K/group_size, stride] outputs."""
    half_k = parts[0][0].shape[1]
    k = 2 * half_k
    rows = [int(p.shape[0]) for p, _ in parts]
    stride = packed_out.shape[1]
    if tuple(packed_out.shape) != (half_k, stride) or tuple(scale_out.shape) != (k // group_size, stride):
        raise ValueError("outputs must be [K/2, stride] and [K/group_size, stride]")
    n = len(parts)
    pp = (c_void_p * n)(*[_ptr(p, torch.uint8, "packed part") for p, _ in parts])
    sp = (c_void_p * n)(*[_ptr(sc, torch.uint8, "scale part") for _, sc in parts])
    rr = (c_u32 * n)(*rows)
    _check("nvfp4_moe_transpose_concat", _lib.nvfp4_moe_transpose_concat(
        pp, sp, rr, n, k, group_size, stride, _ptr(packed_out, torch.uint8, "packed_out"),
        _ptr(scale_out, torch.uint8, "scale_out"), _stream(stream)))


def shard_nvfp4(packed, scale, kind: int, rank: int, tp: int, stream=None):
    """nvfp4_moe_shard_nvfp4 over a stack [E, N, K/2] / [E, N, K/16] (or one [N, K/2]
    matrix): returns this rank's packed and scale tensors, newly allocated."""
    squeeze = packed.dim() == 2
    p3 = packed.unsqueeze(0) if squeeze else packed
    s3 = scale.unsqueeze(0) if squeeze else scale
    e, n, half_k = p3.shape
    k = 2 * half_k
    if tuple(s3.shape) != (e, n, k // 16):
        raise ValueError("scale must be [E, N, K/16]")
    if kind == SHARD_COLUMN:
        if tp < 1 or n % tp:
            raise ValueError("N must be divisible by tp")
        po = torch.empty((e, n // tp, half_k), dtype=torch.uint8, device=packed.device)
        so = torch.empty((e, n // tp, k // 16), dtype=torch.uint8, device=packed.device)
    elif kind == SHARD_ROW:
        if tp < 1 or half_k % tp or (k // 16) % tp:
            raise ValueError("K/2 and K/16 must be divisible by tp")
        po = torch.empty((e, n, half_k // tp), dtype=torch.uint8, device=packed.device)
        so = torch.empty((e, n, k // 16 // tp), dtype=torch.uint8, device=packed.device)
    else:
        raise ValueError("kind must be SHARD_COLUMN or SHARD_ROW")
    shard_nvfp4_into(p3, s3, kind, rank, tp, po, so, stream=stream)
    return (po[0], so[0]) if squeeze else (po, so)


def shard_nvfp4_into(packed, scale, kind: int, rank: int, tp: int, packed_out, scale_out,
                     stream=None) -> None:
    """nvfp4_moe_shard_nvfp4 into caller-allocated [E, ...] outputs."""
    e, n, half_k = packed.shape
    _check("nvfp4_moe_shard_nvfp4", _lib.nvfp4_moe_shard_nvfp4(
        _ptr(packed, torch.uint8, "packed"), _ptr(scale, torch.uint8, "scale"), e, n, 2 * half_k,
        kind, rank, tp, _ptr(packed_out, torch.uint8, "packed_out"),
        _ptr(scale_out, torch.uint8, "scale_out"), _stream(stream)))


def workspace_bytes(num_tokens, topk, hidden, inter) -> int:
    return int(_lib.nvfp4_moe_workspace_bytes(num_tokens, topk, hidden, inter))


def device_error(clear: bool = True) -> int:
    """The library's device error word (synchronises the device)."""
    return int(_lib.nvfp4_moe_device_error(1 if clear else 0))


def wait_selftest(cycle_limit: int, arrive: bool, stream=None) -> None:
    """nvfp4_moe_wait_selftest: one bounded barrier wait on the device that runs
    out (arrive=False: the device error word becomes 1) or completes."""
    _check("nvfp4_moe_wait_selftest", _lib.nvfp4_moe_wait_selftest(
        cycle_limit, 1 if arrive else 0, _stream(stream)))


def _ws(workspace):
    if workspace.dtype != torch.uint8 or workspace.device.type != "cuda" or not workspace.is_contiguous():
        raise ValueError("workspace: contiguous uint8 CUDA tensor")
    return workspace.data_ptr(), workspace.numel()


def gate_up_silu_ws(x, gate: ExpertTables, up: ExpertTables, act, expert_offsets, sorted_pair_ids,
                    active_experts, active_count, n_inter, k_hidden, cap, num_tokens, topk,
                    num_experts, workspace, path=0, split=0, tiles=0, depth=0, staging=0, stream=None) -> None:
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    wp, wn = _ws(workspace)
    _check("nvfp4_moe_gate_up_silu_ws", _lib.nvfp4_moe_gate_up_silu_ws(
        _ptr(x, None, "x"), gate, up, _ptr(act, torch.float32, "act"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(sorted_pair_ids, torch.int32, "sorted_pair_ids"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_inter, k_hidden, cap, num_tokens, topk, num_experts,
        _opts(path, split, tiles, depth, staging), wp, wn, _stream(stream)))


def down_ws(act, down_w: ExpertTables, y, expert_offsets, active_experts, active_count, n_hidden,
            k_inter, cap, num_tokens, topk, num_experts, workspace, path=0, split=0, tiles=0, depth=0, staging=0,
            stream=None) -> None:
    wp, wn = _ws(workspace)
    _check("nvfp4_moe_down_ws", _lib.nvfp4_moe_down_ws(
        _ptr(act, torch.float32, "act"), down_w, _ptr(y, torch.float32, "y"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_hidden, k_inter, cap, num_tokens, topk, num_experts,
        _opts(path, split, tiles, depth, staging), wp, wn, _stream(stream)))


def forward(x, topk_ids, topk_weights, gate: ExpertTables, up: ExpertTables, down: ExpertTables,
            buffers: Buffers, num_experts, hidden, inter, workspace=None, path=0, split=0, tiles=0,
            depth=0, staging=0, stream=None) -> None:
    """nvfp4_moe_forward: the four steps of one layer in one library call.
    ``buffers`` is a :class:`Buffers` of device pointers (see ``MoEBuffers.c_buffers``)."""
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    m, k = topk_ids.shape
    wp, wn = (None, 0) if workspace is None else _ws(workspace)
    _check("nvfp4_moe_forward", _lib.nvfp4_moe_forward(
        _ptr(x, None, "x"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_weights, torch.float32, "topk_weights"), gate, up, down, ctypes.byref(buffers),
        m, k, num_experts, hidden, inter, _opts(path, split, tiles, depth, staging), wp, wn, _stream(stream)))


def _activation(activation) -> int:
    if activation not in ACTIVATIONS:
        raise ValueError(f"activation must be one of {sorted(ACTIVATIONS)}")
    return ACTIVATIONS[activation]


def up_act(x, up: ExpertTables, act, expert_offsets, sorted_pair_ids, active_experts, active_count,
           n_inter, k_hidden, cap, num_tokens, topk, activation, path=0, split=0, tiles=0, depth=0, staging=0,
           stream=None) -> None:
    """nvfp4_moe_up_act: act = f(x Wu^T) by sorted position (non-gated experts)."""
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    _check("nvfp4_moe_up_act", _lib.nvfp4_moe_up_act(
        _ptr(x, None, "x"), up, _ptr(act, torch.float32, "act"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(sorted_pair_ids, torch.int32, "sorted_pair_ids"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_inter, k_hidden, cap, num_tokens, topk, _activation(activation),
        _opts(path, split, tiles, depth, staging), _stream(stream)))


def up_act_ws(x, up: ExpertTables, act, expert_offsets, sorted_pair_ids, active_experts,
              active_count, n_inter, k_hidden, cap, num_tokens, topk, num_experts, activation,
              workspace, path=0, split=0, tiles=0, depth=0, staging=0, stream=None) -> None:
    """nvfp4_moe_up_act_ws: nvfp4_moe_up_act with a workspace (tcgen05 path)."""
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    wp, wn = _ws(workspace)
    _check("nvfp4_moe_up_act_ws", _lib.nvfp4_moe_up_act_ws(
        _ptr(x, None, "x"), up, _ptr(act, torch.float32, "act"),
        _ptr(expert_offsets, torch.int32, "expert_offsets"),
        _ptr(sorted_pair_ids, torch.int32, "sorted_pair_ids"),
        _ptr(active_experts, torch.int32, "active_experts"),
        _ptr(active_count, torch.int32, "active_count"),
        n_inter, k_hidden, cap, num_tokens, topk, num_experts, _activation(activation),
        _opts(path, split, tiles, depth, staging), wp, wn, _stream(stream)))


def forward_nongated(x, topk_ids, topk_weights, up: ExpertTables, down: ExpertTables,
                     buffers: Buffers, num_experts, hidden, inter, activation, workspace=None,
                     path=0, split=0, tiles=0, depth=0, staging=0, stream=None) -> None:
    """nvfp4_moe_forward_nongated: the four steps of a layer of non-gated experts."""
    if x.dtype not in (torch.bfloat16, torch.uint16, torch.int16):
        raise TypeError("x: expected bf16 (or its uint16 bits)")
    m, k = topk_ids.shape
    wp, wn = (None, 0) if workspace is None else _ws(workspace)
    _check("nvfp4_moe_forward_nongated", _lib.nvfp4_moe_forward_nongated(
        _ptr(x, None, "x"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_weights, torch.float32, "topk_weights"), up, down, ctypes.byref(buffers),
        m, k, num_experts, hidden, inter, _activation(activation), _opts(path, split, tiles, depth, staging),
        wp, wn, _stream(stream)))
