"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments on the host before any CUDA call.  No compute runs."""

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"NVFP4_MOE_API\s+[\w\s\*]*?\b(nvfp4_moe_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    path = __graft_entry__._build_module().build()
    return ctypes.CDLL(path)


def test_header_declares_the_five_steps():
    names = _declared()
    for n in ("nvfp4_moe_route_sort", "nvfp4_moe_gate_up_silu", "nvfp4_moe_down",
              "nvfp4_moe_blend", "nvfp4_moe_transpose_u8"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_resolves_every_declared_symbol(lib):
    import nvfp4_weight_quantized_moe_b200 as m
    assert set(m.exported_symbols()) == _declared()


def test_host_validation_rejects_bad_shapes_without_a_gpu(lib):
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    t = B.ExpertTables(None, None, None)
    # route_sort: E = 0, E > 1024, topk > E
    args = [None, 1, 2, 0, ctypes.c_void_p(8), None, None, ctypes.c_void_p(8), ctypes.c_void_p(8), None, None]
    assert L.nvfp4_moe_route_sort(*args) == 2
    args[3] = 2048
    assert L.nvfp4_moe_route_sort(*args) == 2
    args[3] = 1
    assert L.nvfp4_moe_route_sort(*args) == 2
    # route_sort: missing outputs
    assert L.nvfp4_moe_route_sort(None, 1, 1, 4, None, None, None, None, None, None, None) == 1
    # gate_up: K not a multiple of 256, N not a multiple of 64
    assert L.nvfp4_moe_gate_up_silu(None, t, t, None, None, None, None, None, 64, 100, 1, 1, 1, None) == 2
    assert L.nvfp4_moe_gate_up_silu(None, t, t, None, None, None, None, None, 48, 256, 1, 1, 1, None) == 2
    # gate_up: NULL tables with work to do
    assert L.nvfp4_moe_gate_up_silu(None, t, t, None, None, None, None, None, 64, 256, 1, 1, 1, None) == 1
    # gate_up: no tokens is a no-op
    assert L.nvfp4_moe_gate_up_silu(None, t, t, None, None, None, None, None, 64, 256, 1, 0, 1, None) == 0
    # down: N not a multiple of 128
    assert L.nvfp4_moe_down(None, t, None, None, None, None, 64, 256, 1, 1, 1, None) == 2
    # blend: hidden % 4
    assert L.nvfp4_moe_blend(None, None, None, None, None, 1, 1, 6, None) == 2
    assert L.nvfp4_moe_blend(None, None, None, None, None, 0, 1, 8, None) == 0
    # transpose: overlap and NULL
    assert L.nvfp4_moe_transpose_u8(None, None, 4, 4, None) == 1
    assert L.nvfp4_moe_transpose_u8(ctypes.c_void_p(4096), ctypes.c_void_p(4100), 4, 4, None) == 1
    # launch options: bad path / split
    bad = B.LaunchOpts(7, 0, 0, 0)
    ok_t = B.ExpertTables(8, 8, 8)
    p8 = ctypes.c_void_p(8)
    assert L.nvfp4_moe_gate_up_silu_ex(p8, ok_t, ok_t, p8, p8, p8, p8, p8, 64, 256, 1, 1, 1,
                                       ctypes.byref(bad), None) == 1
    for opts in ((1, 8, 0, 0), (1, 3, 0, 0), (1, 0, 3, 0), (1, 0, 0, 5), (1, 1, 4, 0), (1, 4, 2, 2)):
        # split 8 or 3, tiles 3, depth 5, down with 4 tiles, split with 2 tiles
        bad = B.LaunchOpts(*opts)
        assert L.nvfp4_moe_down_ex(p8, ok_t, p8, p8, p8, p8, 128, 256, 1, 1, 1,
                                   ctypes.byref(bad), None) == 1, opts
    # staging: unknown choice; whole-K staging past the shared-memory limit
    # (K = 16384 on two tiles: 64 chunks x 8 KB) is refused before any launch
    for opts, k in (((1, 0, 0, 0, 3), 256), ((1, 1, 2, 2, 1), 16384)):
        bad = B.LaunchOpts(*opts)
        assert L.nvfp4_moe_gate_up_silu_ex(p8, ok_t, ok_t, p8, p8, p8, p8, p8, 64, k, 1, 1, 1,
                                           ctypes.byref(bad), None) == 1, opts


def test_nongated_calls_check_activation_and_shapes_on_the_host(lib):
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    t = B.ExpertTables(8, 8, 8)
    p8 = ctypes.c_void_p(8)
    # unknown activation (0, 3), then N not a multiple of 128, K not a multiple of 256
    for act in (0, 3):
        assert L.nvfp4_moe_up_act(p8, t, p8, p8, p8, p8, p8, 256, 512, 1, 1, 1, act, None, None) == 1
    assert L.nvfp4_moe_up_act(p8, t, p8, p8, p8, p8, p8, 192, 512, 1, 1, 1, 1, None, None) == 2
    assert L.nvfp4_moe_up_act(p8, t, p8, p8, p8, p8, p8, 256, 320, 1, 1, 1, 2, None, None) == 2
    # NULL up table with work to do; no tokens is a no-op
    t0 = B.ExpertTables(None, None, None)
    assert L.nvfp4_moe_up_act(p8, t0, p8, p8, p8, p8, p8, 256, 512, 1, 1, 1, 1, None, None) == 1
    assert L.nvfp4_moe_up_act(p8, t0, p8, p8, p8, p8, p8, 256, 512, 1, 0, 1, 1, None, None) == 0
    # tcgen05 path forced on a width that is not a multiple of 256; short workspace
    opts = B.LaunchOpts(2, 0, 0, 0)
    assert L.nvfp4_moe_up_act_ws(p8, t, p8, p8, p8, p8, p8, 384, 512, 8, 64, 4, 8, 1,
                                 ctypes.byref(opts), ctypes.c_void_p(1 << 20), 1 << 30, None) == 2
    assert L.nvfp4_moe_up_act_ws(p8, t, p8, p8, p8, p8, p8, 512, 512, 8, 64, 4, 8, 1,
                                 ctypes.byref(opts), ctypes.c_void_p(1 << 20), 1024, None) == 1
    assert L.nvfp4_moe_forward_nongated(p8, p8, p8, t, t, None, 1, 1, 8, 512, 512, 1, None, None, 0,
                                        None) == 1


def test_active_cap_and_status_strings(lib):
    import nvfp4_weight_quantized_moe_b200 as m
    assert m.active_cap(128, 8) == 8 and m.active_cap(8, 65536) == 8
    L = m._binding._lib
    for s in range(4):
        assert L.nvfp4_moe_status_string(s)


def test_workspace_calls_check_size_and_alignment_on_the_host(lib):
    # The tcgen05 path (path 2) needs nvfp4_moe_workspace_bytes of 256-byte aligned
    # workspace; a short or misaligned one is refused before anything is launched.
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    t = B.ExpertTables(8, 8, 8)
    p8 = ctypes.c_void_p(8)
    tokens, topk, hidden, inter, experts = 16, 4, 512, 256, 8
    need = L.nvfp4_moe_workspace_bytes(tokens, topk, hidden, inter)
    pairs = tokens * topk
    # sorted f16 rows, their scales, 512 KiB of tensor maps, act hi + lo, their scales, maps
    assert need >= pairs * hidden * 2 + pairs * inter * 4 + 2 * (512 << 10)
    opts = B.LaunchOpts(2, 0, 0, 0)
    cap = min(experts, pairs)

    def gate_up(ws, nbytes):
        return L.nvfp4_moe_gate_up_silu_ws(p8, t, t, p8, p8, p8, p8, p8, inter, hidden, cap, tokens, topk,
                                           experts, ctypes.byref(opts), ws, nbytes, None)

    def down(ws, nbytes):
        return L.nvfp4_moe_down_ws(p8, t, p8, p8, p8, p8, hidden, inter, cap, tokens, topk, experts,
                                   ctypes.byref(opts), ws, nbytes, None)

    for call in (gate_up, down):
        assert call(None, need) == 1
        assert call(ctypes.c_void_p(1 << 20), need - 1) == 1
        assert call(ctypes.c_void_p((1 << 20) + 128), need) == 1
    # path 2 with a width the tcgen05 kernels do not take
    assert L.nvfp4_moe_down_ws(p8, t, p8, p8, p8, p8, 128, inter, cap, tokens, topk, experts,
                               ctypes.byref(opts), ctypes.c_void_p(1 << 20), need, None) == 2


def test_shared_and_scale_check_calls_validate_on_the_host(lib):
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    p8 = ctypes.c_void_p(8)
    assert L.nvfp4_moe_shared_slots(8192, 512) == 16
    assert L.nvfp4_moe_shared_slots(7, 2) == 4
    assert L.nvfp4_moe_shared_slots(0, 16) == 0
    assert L.nvfp4_moe_shared_slots(5, 0) == 0
    # shared_rows = 0; too many table entries (1000 + 32); no tokens (nothing launched)
    assert L.nvfp4_moe_append_shared(p8, p8, None, 4, 2, 8, 0, p8, p8, None) == 1
    assert L.nvfp4_moe_append_shared(p8, p8, None, 512, 2, 1000, 16, p8, p8, None) == 2
    assert L.nvfp4_moe_append_shared(None, None, None, 0, 2, 8, 16, None, None, None) == 0
    assert L.nvfp4_moe_append_shared(None, p8, None, 4, 2, 8, 16, p8, p8, None) == 1
    t = B.ExpertTables(8, 8, None)
    # k not a multiple of 256; 0 or > 1024 experts; NULL counters or tables
    assert L.nvfp4_moe_check_scales(t, 4, 128, 300, p8, None) == 2
    assert L.nvfp4_moe_check_scales(t, 0, 128, 256, p8, None) == 2
    assert L.nvfp4_moe_check_scales(t, 1025, 128, 256, p8, None) == 2
    assert L.nvfp4_moe_check_scales(t, 4, 128, 256, None, None) == 1
    assert L.nvfp4_moe_check_scales(B.ExpertTables(None, 8, None), 4, 128, 256, p8, None) == 1


def test_shard_call_validates_on_the_host(lib):
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    a, b, c, d = (ctypes.c_void_p(1 << 20), ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20),
                  ctypes.c_void_p(4 << 20))
    col, row = B.SHARD_COLUMN, B.SHARD_ROW
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 256, 7, 0, 2, c, d, None) == 1   # bad kind
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 256, col, 2, 2, c, d, None) == 1  # rank >= tp
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 256, col, 0, 0, c, d, None) == 1  # tp = 0
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 100, col, 0, 2, c, d, None) == 2  # k % 16
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 66, 256, col, 0, 4, c, d, None) == 2  # n % tp
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 80, row, 0, 2, c, d, None) == 2   # k/16 = 5
    assert L.nvfp4_moe_shard_nvfp4(a, b, 0, 64, 256, row, 0, 2, c, d, None) == 0  # nothing to do
    assert L.nvfp4_moe_shard_nvfp4(a, None, 1, 64, 256, row, 0, 2, c, d, None) == 1
    assert L.nvfp4_moe_shard_nvfp4(a, b, 1, 64, 256, row, 0, 2, ctypes.c_void_p((1 << 20) + 64),
                                   d, None) == 1  # output overlaps the input


def test_expert_owner_blocks_match_the_oracle():
    import oracle as orc
    from nvfp4_weight_quantized_moe_b200 import expert_owner_range
    for e in (1, 7, 8, 128, 256, 1000):
        for world in (1, 2, 3, 8):
            if world > e:
                continue
            for r in range(world):
                assert expert_owner_range(e, world, r) == orc.expert_owner_range(e, world, r)


def test_transpose_concat_validates_on_the_host(lib):
    import nvfp4_weight_quantized_moe_b200._binding as B
    L = B._lib
    P = ctypes.c_void_p
    pp = (P * 2)(P(1 << 20), P(2 << 20))
    sp = (P * 2)(P(3 << 20), P(4 << 20))
    rr = (ctypes.c_uint32 * 2)(8, 4)
    out_w, out_s = P(5 << 20), P(6 << 20)
    assert L.nvfp4_moe_transpose_concat(pp, sp, rr, 0, 64, 16, 12, out_w, out_s, None) == 1  # no parts
    assert L.nvfp4_moe_transpose_concat(pp, sp, rr, 2, 63, 16, 12, out_w, out_s, None) == 2  # odd k
    assert L.nvfp4_moe_transpose_concat(pp, sp, rr, 2, 64, 24, 12, out_w, out_s, None) == 2  # group
    assert L.nvfp4_moe_transpose_concat(pp, sp, rr, 2, 64, 16, 11, out_w, out_s, None) == 2  # stride
    assert L.nvfp4_moe_transpose_concat(pp, sp, rr, 2, 64, 16, 12, None, out_s, None) == 1
    nulls = (P * 2)(P(1 << 20), None)
    assert L.nvfp4_moe_transpose_concat(nulls, sp, rr, 2, 64, 16, 12, out_w, out_s, None) == 1
