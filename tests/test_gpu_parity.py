"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Matching rules (the forward's stated bar):
  * route sort, transpose_u8: bit-exact;
  * act, y, out: compared in FP32 against the fp64 oracle, relative L2 error
    <= 1e-3 and max abs error <= 4e-3 * max|ref|.
"""

import numpy as np
import pytest
import torch

import oracle as orc
from workloads import CONFIGS, make_problem
from workloads.generators import MATRIX_DOWN, MATRIX_GATE, MATRIX_UP, MoEConfig

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS_FRAC = 4e-3


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _close(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rel = orc.relative_l2(got, ref)
    mx = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e}"
    assert err <= MAX_ABS_FRAC * mx + 1e-30, f"{what}: max abs {err:.3e} vs max|ref| {mx:.3e}"
    return rel


def _fns(prob):
    return [lambda e, m=m: prob.expert_weight(m, e, cache=True) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]


def _gpu_forward(prob, layer=None, ws=False, **opts):
    from workloads.device import upload_inputs, upload_layer
    import nvfp4_weight_quantized_moe_b200 as nvm
    layer = layer or upload_layer(prob)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(prob.cfg.tokens, out_bf16=True)
    bufs.act.fill_(float("nan"))
    bufs.y.fill_(float("nan"))
    bufs.out.fill_(float("nan"))
    workspace = layer.workspace(prob.cfg.tokens) if ws else None
    if workspace is not None:
        workspace.fill_(0xFF)  # NaN f16 patterns: anything read before it is written shows up
    layer.forward(x, ids, w, bufs, workspace=workspace, **opts)
    torch.cuda.synchronize()
    assert nvm.device_error() == 0
    return layer, bufs


def _check_sort(bufs, rs, num_experts, pairs):
    off = bufs.expert_offsets.cpu().numpy()
    np.testing.assert_array_equal(off, rs.expert_offsets)
    np.testing.assert_array_equal(bufs.sorted_pair_ids.cpu().numpy()[:pairs], rs.sorted_pair_ids)
    np.testing.assert_array_equal(bufs.pair_pos.cpu().numpy()[:pairs], rs.pair_pos)
    np.testing.assert_array_equal(bufs.active_experts.cpu().numpy(), rs.active_experts)
    assert int(bufs.active_count.item()) == rs.active_count


def _check_full(prob, bufs):
    cfg = prob.cfg
    ref = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *_fns(prob),
                          hidden=cfg.hidden, inter=cfg.inter)
    rs = ref["sort"]
    _check_sort(bufs, rs, cfg.experts, cfg.pairs)
    kept = int(rs.expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], ref["act"][:kept], "act")
    _close(bufs.y.cpu().numpy()[:kept], ref["y"][:kept], "y")
    rel = _close(bufs.out.cpu().numpy(), ref["out"], "out")
    # The BF16 copy is the FP32 output rounded to nearest even.
    ob = bufs.out_bf16.float().cpu().numpy()
    np.testing.assert_array_equal(ob, bufs.out.bfloat16().float().cpu().numpy())
    return rel


# --------------------------------------------------------------------------- #
# Element formats and layout on the device
# --------------------------------------------------------------------------- #

def test_nibble_order_and_decode_on_gpu():
    """One expert whose every row holds all 16 E2M1 codes in both nibble slots."""
    _need_gpu()
    cfg = MoEConfig("nib", hidden=256, inter=256, experts=1, topk=1, tokens=1, router="uniform", seed=5)
    prob = make_problem(cfg)
    from workloads.device import upload_inputs, upload_layer
    layer = upload_layer(prob)
    # Row n of gate: byte j = (code_hi << 4) | code_lo with varied codes; scales vary too.
    rng = np.random.default_rng(0)
    packed = rng.integers(0, 256, (256, 128), dtype=np.uint8)
    scale = rng.integers(0x00, 0x7F, (256, 16), dtype=np.uint8)  # all finite codes incl. subnormals
    layer.gate.packed[0].copy_(torch.from_numpy(packed))
    layer.gate.scale[0].copy_(torch.from_numpy(scale))
    prob._cache[(MATRIX_GATE, 0)] = (packed, scale)
    for k in (0, 1, 100, 255):
        prob.x_bf16[:] = 0
        prob.x_bf16[0, k] = 0x3F80  # x = e_k
        x, ids, w = upload_inputs(prob)
        bufs = layer.buffers(1)
        layer.forward(x, ids, w, bufs)
        torch.cuda.synchronize()
        wg = orc.dequantize_nvfp4(packed, scale, prob.scale2[MATRIX_GATE, 0])
        pu, su, s2u = prob.expert_weight(MATRIX_UP, 0)
        wu = orc.dequantize_nvfp4(pu, su, s2u)
        expect = orc.silu(wg[:, k]) * wu[:, k]
        got = bufs.act.cpu().numpy()[0]
        np.testing.assert_allclose(got, expect, rtol=2e-6, atol=1e-12)


# --------------------------------------------------------------------------- #
# Route sort: bit-exact
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", list(CONFIGS))
def test_route_sort_bit_exact(name):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    prob = make_problem(name)
    cfg = prob.cfg
    ids = torch.from_numpy(prob.topk_ids).cuda()
    bufs = nvm.MoEBuffers(cfg.tokens, cfg.topk, cfg.experts, 4, 4, "cuda")
    nvm.route_sort(ids, cfg.experts, bufs.expert_offsets, bufs.sorted_pair_ids, bufs.pair_pos,
                   bufs.active_experts, bufs.active_count, bufs.status)
    torch.cuda.synchronize()
    _check_sort(bufs, orc.route_sort(prob.topk_ids, cfg.experts), cfg.experts, cfg.pairs)
    assert int(bufs.status.item()) == 0


def test_route_sort_out_of_range_ids_and_max_experts():
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(4)
    for e, m, k in ((1024, 700, 8), (5, 3000, 3)):
        ids = rng.integers(-2, e + 3, (m, k)).astype(np.int32)
        bufs = nvm.MoEBuffers(m, k, e, 4, 4, "cuda")
        nvm.route_sort(torch.from_numpy(ids).cuda(), e, bufs.expert_offsets, bufs.sorted_pair_ids,
                       bufs.pair_pos, bufs.active_experts, bufs.active_count, bufs.status)
        torch.cuda.synchronize()
        rs = orc.route_sort(ids, e)
        assert rs.dropped > 0
        kept = int(rs.expert_offsets[-1])
        _check_sort(bufs, rs, e, m * k)
        assert np.all(bufs.sorted_pair_ids.cpu().numpy()[kept:] == -1)
        assert int(bufs.status.item()) == 1


def test_route_sort_large_batch_bit_exact():
    # 2^22 routed pairs over 1024 experts (the cluster sort: 512 Ki pairs per CTA),
    # with out-of-range ids, against the oracle's stable sort.
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(12)
    m, k, e = 1 << 19, 8, 1024
    ids = rng.integers(-1, e + 1, (m, k)).astype(np.int32)
    bufs = nvm.MoEBuffers(m, k, e, 4, 4, "cuda")
    nvm.route_sort(torch.from_numpy(ids).cuda(), e, bufs.expert_offsets, bufs.sorted_pair_ids,
                   bufs.pair_pos, bufs.active_experts, bufs.active_count, bufs.status)
    torch.cuda.synchronize()
    rs = orc.route_sort(ids, e)
    _check_sort(bufs, rs, e, m * k)
    assert int(bufs.status.item()) == 1


@pytest.mark.parametrize("name,ws", [("tiny", False), ("zipf", False), ("zipf", True), ("hot", True)])
def test_one_call_forward_equals_the_four_steps(name, ws):
    # nvfp4_moe_forward launches the same kernels as the four single-step calls:
    # every output is bit-identical.
    _need_gpu()
    prob = make_problem(SMALL[name])
    layer, one = _gpu_forward(prob, ws=ws)
    _, four = _gpu_forward(prob, layer=layer, ws=ws, steps=True)
    def bits(t):  # bit patterns, so that NaN rows left untouched compare equal too
        return t.view(torch.int16) if t.dtype == torch.bfloat16 else (
            t.view(torch.int32) if t.dtype == torch.float32 else t)

    for f in ("expert_offsets", "sorted_pair_ids", "pair_pos", "active_experts", "active_count", "act",
              "y", "out", "out_bf16"):
        assert torch.equal(bits(getattr(one, f)), bits(getattr(four, f))), f
    _check_full(prob, one)


def test_route_sort_small_batches_bit_exact():
    # Up to 32 pairs take the single-warp sort: cover every P in 1..33 (the
    # boundary on both sides), out-of-range ids, one expert, and 1024 experts.
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(11)
    for p in range(1, 34):
        for e in (1, 7, 128, 1024):
            k = int(rng.integers(1, min(e, 8) + 1))
            m = max(1, p // k)
            ids = rng.integers(-1, e + 1, (m, k)).astype(np.int32)
            bufs = nvm.MoEBuffers(m, k, e, 4, 4, "cuda")
            nvm.route_sort(torch.from_numpy(ids).cuda(), e, bufs.expert_offsets, bufs.sorted_pair_ids,
                           bufs.pair_pos, bufs.active_experts, bufs.active_count, bufs.status)
            torch.cuda.synchronize()
            rs = orc.route_sort(ids, e)
            _check_sort(bufs, rs, e, m * k)
            kept = int(rs.expert_offsets[-1])
            assert np.all(bufs.sorted_pair_ids.cpu().numpy()[kept:m * k] == -1)
            assert int(bufs.status.item()) == (1 if rs.dropped > 0 else 0)


# --------------------------------------------------------------------------- #
# transpose_u8: bit-exact
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("rows,cols", [(1, 1), (33, 65), (64, 128), (1536, 128), (257, 96)])
def test_transpose_u8_bit_exact(rows, cols):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    src = np.random.default_rng(rows + cols).integers(0, 256, (rows, cols), dtype=np.uint8)
    d_src = torch.from_numpy(src).cuda()
    d_dst = torch.empty((cols, rows), dtype=torch.uint8, device="cuda")
    nvm.transpose_u8(d_src, d_dst)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d_dst.cpu().numpy(), orc.transpose_u8(src, rows, cols))


# --------------------------------------------------------------------------- #
# The forward on small problems, every decode variant
# --------------------------------------------------------------------------- #

SMALL = {
    "tiny": CONFIGS["tiny"],
    # ragged: odd token count, k = 3, 5 experts; rows per expert not a tile multiple
    "ragged": MoEConfig("ragged", hidden=512, inter=256, experts=5, topk=3, tokens=7,
                        router="uniform", seed=21),
    # hot: the first k experts carry every token (> 32 rows each: several row groups)
    "hot": MoEConfig("hot", hidden=768, inter=512, experts=9, topk=2, tokens=70,
                     router="hot", seed=22),
    # skewed, more experts than pairs
    "zipf": MoEConfig("zipf", hidden=1024, inter=512, experts=64, topk=4, tokens=6,
                      router="zipf", seed=23),
    # long K: a 2-way K split runs 5 chunks per warp (past the pre-converted
    # activation buffers), a 4-way split 3 (within them)
    "longk": MoEConfig("longk", hidden=2560, inter=2560, experts=6, topk=2, tokens=3,
                       router="uniform", seed=24),
}


# Decode launch shapes: (split, tiles, depth, staging); zeros pick from the shape.
# Staging 1 holds every K chunk of a pass's token rows in shared memory, 2 a
# two-chunk ring; every forced shape runs both ways.
PLANS = [(0, 0, 0, 0)] + [(s, t, d, g) for (s, t, d) in
                          [(4, 1, 2), (2, 1, 2), (1, 1, 2), (1, 1, 3), (1, 2, 2), (1, 2, 3)]
                          for g in (1, 2)]


@pytest.mark.parametrize("plan", PLANS, ids=lambda p: "s%d-t%d-d%d-x%d" % p)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small(name, plan):
    _need_gpu()
    prob = make_problem(SMALL[name])
    split, tiles, depth, staging = plan
    _, bufs = _gpu_forward(prob, path=1 if any(plan) else 0, split=split, tiles=tiles, depth=depth,
                           staging=staging)
    _check_full(prob, bufs)


@pytest.mark.parametrize("staging", [1, 2])
def test_gate_up_four_tiles(staging):
    """Gate+up holding 32 rows per pass (the 17..32-token shape)."""
    _need_gpu()
    prob = make_problem(SMALL["hot"])
    import nvfp4_weight_quantized_moe_b200 as nvm
    from workloads.device import upload_inputs, upload_layer
    cfg = prob.cfg
    layer = upload_layer(prob)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(cfg.tokens)
    nvm.route_sort(ids, cfg.experts, bufs.expert_offsets, bufs.sorted_pair_ids, bufs.pair_pos,
                   bufs.active_experts, bufs.active_count, bufs.status)
    cap = nvm.active_cap(cfg.experts, cfg.pairs)
    nvm.gate_up_silu(x, layer.gate.tables, layer.up.tables, bufs.act, bufs.expert_offsets,
                     bufs.sorted_pair_ids, bufs.active_experts, bufs.active_count, cfg.inter,
                     cfg.hidden, cap, cfg.tokens, cfg.topk, path=1, split=1, tiles=4, depth=2,
                     staging=staging)
    torch.cuda.synchronize()
    ref = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *_fns(prob),
                          hidden=cfg.hidden, inter=cfg.inter)
    kept = int(ref["sort"].expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], ref["act"][:kept], "act")


# tcgen05 path: token rows per pass 16 (tiles=2) or 128 (tiles=16) on the one-CTA
# kernel, 32 (tiles=4), 192 (tiles=24) or 256 (tiles=32: gate+up with A in shared
# memory, down at 192) on the CTA-pair kernel; 0 = from the shape.
@pytest.mark.parametrize("tiles", [0, 2, 4, 16, 24, 32])
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_tcgen05(name, tiles):
    _need_gpu()
    prob = make_problem(SMALL[name])
    _, bufs = _gpu_forward(prob, ws=True, path=2, tiles=tiles)
    _check_full(prob, bufs)


@pytest.mark.parametrize("tiles", [0, 24])
def test_null_experts_tcgen05(tiles):
    _need_gpu()
    prob = make_problem(SMALL["ragged"], null_experts=[1, 3])
    _, bufs = _gpu_forward(prob, ws=True, path=2, tiles=tiles)
    _check_full(prob, bufs)


# Experts of 1 .. 400 rows on the pair kernel: every pass length 32 .. 192 and
# several passes per expert, two column blocks of gate+up (I = 256).
PAIR_CFG = MoEConfig("pairrows", hidden=512, inter=256, experts=12, topk=3, tokens=400,
                     router="zipf", seed=25)


@pytest.mark.parametrize("tiles", [32, 24, 16, 4])
def test_forward_pair_kernel_pass_lengths(tiles):
    _need_gpu()
    prob = make_problem(PAIR_CFG)
    counts = np.bincount(prob.topk_ids.reshape(-1), minlength=PAIR_CFG.experts)
    assert counts.max() > 192 and counts[counts > 0].min() < 32
    _, bufs = _gpu_forward(prob, ws=True, path=2, tiles=tiles)
    _check_full(prob, bufs)


def test_null_experts_write_zero_rows():
    _need_gpu()
    prob = make_problem(SMALL["ragged"], null_experts=[1, 3])
    _, bufs = _gpu_forward(prob)
    _check_full(prob, bufs)


def test_dropped_pairs_contribute_nothing():
    _need_gpu()
    prob = make_problem(SMALL["ragged"])
    prob.topk_ids[2, 1] = 99
    prob.topk_ids[5, 0] = -1
    _, bufs = _gpu_forward(prob)
    assert int(bufs.status.item()) == 1
    _check_full(prob, bufs)


def test_empty_batch_is_a_no_op():
    _need_gpu()
    prob = make_problem(SMALL["ragged"])
    from workloads.device import upload_layer
    layer = upload_layer(prob)
    x = torch.empty((0, prob.cfg.hidden), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((0, prob.cfg.topk), dtype=torch.int32, device="cuda")
    w = torch.empty((0, prob.cfg.topk), dtype=torch.float32, device="cuda")
    bufs = layer.buffers(0)
    layer.forward(x, ids, w, bufs)
    torch.cuda.synchronize()
    assert int(bufs.active_count.item()) == 0


def test_deterministic_and_graph_replay():
    _need_gpu()
    prob = make_problem(SMALL["zipf"])
    layer, b1 = _gpu_forward(prob)
    from workloads.device import upload_inputs
    x, ids, w = upload_inputs(prob)
    b2 = layer.buffers(prob.cfg.tokens)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        layer.forward(x, ids, w, b2)  # warm-up on the capture stream
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.forward(x, ids, w, b2)
    b2.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(b1.out, b2.out)


def test_large_activation_range():
    """x rows far outside the f16 range stay accurate (per-chunk power-of-two scaling)."""
    _need_gpu()
    prob = make_problem(SMALL["ragged"])
    from workloads.generators import f32_to_bf16_bits
    x = orc.bf16_bits_to_f64(prob.x_bf16).astype(np.float32)
    x[0] *= 1e12
    x[1] *= 1e-12
    x[2, :256] *= 1e8
    prob.x_bf16 = f32_to_bf16_bits(x)
    _, bufs = _gpu_forward(prob)
    cfg = prob.cfg
    ref = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *_fns(prob),
                          hidden=cfg.hidden, inter=cfg.inter)
    kept = int(ref["sort"].expert_offsets[-1])
    act, y, out = bufs.act.cpu().numpy(), bufs.y.cpu().numpy(), bufs.out.cpu().numpy()
    # Row by row: the rows differ by up to 48 orders of magnitude.
    for r in range(kept):
        _close(act[r], ref["act"][r], f"act row {r}")
        _close(y[r], ref["y"][r], f"y row {r}")
    for t in range(cfg.tokens):
        _close(out[t], ref["out"][t], f"out row {t}")


def test_bounded_wait_runs_out_reports_and_the_library_still_works():
    """A barrier wait that nothing completes gives up after its cycle limit, sets the
    device error word and returns; the word is cleared on read; later forwards run."""
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    assert nvm.device_error() == 0
    nvm.wait_selftest(4096, arrive=True)  # the phase completes: no error
    torch.cuda.synchronize()
    assert nvm.device_error() == 0
    nvm.wait_selftest(4096, arrive=False)  # nothing arrives: the wait runs out
    torch.cuda.synchronize()
    assert nvm.device_error(clear=True) == 1
    assert nvm.device_error() == 0
    prob = make_problem(SMALL["ragged"])
    for ws in (False, True):
        _, bufs = _gpu_forward(prob, ws=ws, **(dict(path=2) if ws else {}))
        _check_full(prob, bufs)


# --------------------------------------------------------------------------- #
# The five workloads at full size
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
@pytest.mark.parametrize("name", ["decode_m1", "decode_m32"])
def test_forward_full_decode(name, ws):
    _need_gpu()
    prob = make_problem(name)
    _, bufs = _gpu_forward(prob, ws=ws)
    _check_full(prob, bufs)


@pytest.mark.parametrize("name,staging", [("decode_m1", 2), ("decode_m32", 1)],
                         ids=["decode_m1-ring", "decode_m32-whole-k"])
def test_forward_full_decode_other_staging(name, staging):
    """The activation staging the automatic plan does not take at this size:
    the two-chunk ring at decode M=1, whole-K staging at decode M=32."""
    _need_gpu()
    prob = make_problem(name)
    _, bufs = _gpu_forward(prob, path=1, staging=staging)
    _check_full(prob, bufs)


# The oracle's full result at the two large sizes, computed once per session
# (expert blocks spread over host processes; see _oracle_pool.py).
_FULL_REF = {}


def _full_ref(name):
    if name not in _FULL_REF:
        from _oracle_pool import moe_forward_pooled
        _FULL_REF[name] = moe_forward_pooled(CONFIGS[name])
    return _FULL_REF[name]


def _check_against(ref, bufs, cfg):
    rs = ref["sort"]
    _check_sort(bufs, rs, cfg.experts, cfg.pairs)
    kept = int(rs.expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], ref["act"][:kept], "act")
    _close(bufs.y.cpu().numpy()[:kept], ref["y"][:kept], "y")
    _close(bufs.out.cpu().numpy(), ref["out"], "out")
    ob = bufs.out_bf16.float().cpu().numpy()
    np.testing.assert_array_equal(ob, bufs.out.bfloat16().float().cpu().numpy())


@pytest.mark.parametrize("ws,tiles", [(False, 0), (True, 0), (True, 4)],
                         ids=["decode-path", "tcgen05", "tcgen05-pair32"])
@pytest.mark.parametrize("name", ["decode_m256", "prefill_m8192"])
def test_forward_full_size_every_element(name, ws, tiles):
    """Full-size launch, every element of act, y and out against the oracle's full forward."""
    _need_gpu()
    if tiles and name != "decode_m256":
        pytest.skip("32-row pair passes are the decode-shaped launch")
    prob = make_problem(name)
    _, bufs = _gpu_forward(prob, ws=ws, **(dict(path=2, tiles=tiles) if tiles else {}))
    _check_against(_full_ref(name), bufs, prob.cfg)


# --------------------------------------------------------------------------- #
# Shared expert: appended routing slots through the same launches
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("m,k,e,rows,weighted", [(1, 2, 8, 16, False), (7, 3, 5, 2, True),
                                                 (33, 8, 128, 16, True), (70, 2, 9, 64, False),
                                                 (300, 8, 256, 7, True)])
def test_append_shared_bit_exact(m, k, e, rows, weighted):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(m * 7 + e)
    ids = rng.integers(0, e, (m, k)).astype(np.int32)
    w = rng.random((m, k)).astype(np.float32)
    sw = rng.random(m).astype(np.float32) if weighted else None
    ids_out = torch.full((m, k + 1), -7, dtype=torch.int32, device="cuda")
    w_out = torch.full((m, k + 1), float("nan"), dtype=torch.float32, device="cuda")
    nvm.append_shared(torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), e, rows, ids_out,
                      w_out, shared_weights=None if sw is None else torch.from_numpy(sw).cuda())
    torch.cuda.synchronize()
    ref_ids, ref_w = orc.append_shared_routing(ids, w, e, rows, sw)
    np.testing.assert_array_equal(ids_out.cpu().numpy(), ref_ids)
    np.testing.assert_array_equal(w_out.cpu().numpy().view(np.uint32), ref_w.view(np.uint32))
    assert nvm.shared_slots(m, rows) == -(-m // rows)


def _shared_ref(prob, sw):
    cfg = prob.cfg
    shared = tuple(prob.shared_weight(mt) for mt in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN))
    return orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                  *_fns(prob), hidden=cfg.hidden, inter=cfg.inter, shared=shared,
                                  shared_weights=sw)


def _gpu_forward_shared(prob, sw=None, shared_rows=0, ws=False, layer=None, **opts):
    from workloads.device import upload_inputs, upload_layer
    import nvfp4_weight_quantized_moe_b200 as nvm
    layer = layer or upload_layer(prob, shared=True, shared_rows=shared_rows)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(prob.cfg.tokens, out_bf16=True)
    for t in (bufs.act, bufs.y, bufs.out):
        t.fill_(float("nan"))
    workspace = layer.workspace(prob.cfg.tokens) if ws else None
    if workspace is not None:
        workspace.fill_(0xFF)
    swd = None if sw is None else torch.from_numpy(sw).cuda()
    layer.forward(x, ids, w, bufs, workspace=workspace, shared_weights=swd, **opts)
    torch.cuda.synchronize()
    assert nvm.device_error() == 0
    return layer, bufs


SHARED_CASES = [("tiny", 0, False), ("ragged", 2, True), ("hot", 16, True), ("zipf", 0, False),
                ("longk", 1, True)]


@pytest.mark.parametrize("ws,tiles", [(False, 0), (True, 0), (True, 24), (True, 32)],
                         ids=["decode-path", "tcgen05", "tcgen05-pair192", "tcgen05-pair256"])
@pytest.mark.parametrize("name,rows,weighted", SHARED_CASES)
def test_forward_with_shared_expert(name, rows, weighted, ws, tiles):
    _need_gpu()
    prob = make_problem(SMALL[name])
    cfg = prob.cfg
    sw = (np.random.default_rng(cfg.seed).random(cfg.tokens).astype(np.float32)
          if weighted else None)
    opts = (dict(path=2, tiles=tiles) if tiles else dict(path=2)) if ws else {}
    layer, bufs = _gpu_forward_shared(prob, sw, rows, ws=ws, **opts)
    ref = _shared_ref(prob, sw)
    # The sort of the appended routing is bit-exact; the shared rows come last.
    r = layer.rows_per_shared_slot(cfg.tokens)
    slots = -(-cfg.tokens // r)
    ids2, _ = orc.append_shared_routing(prob.topk_ids, prob.topk_weights, cfg.experts, r, sw)
    rs = orc.route_sort(ids2, cfg.experts + slots)
    e2 = cfg.experts + slots
    np.testing.assert_array_equal(bufs.expert_offsets.cpu().numpy()[:e2 + 1], rs.expert_offsets)
    np.testing.assert_array_equal(bufs.sorted_pair_ids.cpu().numpy(), rs.sorted_pair_ids)
    np.testing.assert_array_equal(bufs.pair_pos.cpu().numpy(), rs.pair_pos)
    sh_act, sh_out = layer.shared_rows_of(bufs, cfg.tokens)
    _close(sh_act.cpu().numpy(), ref["sh_act"], "sh_act")
    _close(sh_out.cpu().numpy(), ref["sh_out"], "sh_out")
    _close(bufs.out.cpu().numpy(), ref["out"], "out")
    ob = bufs.out_bf16.float().cpu().numpy()
    np.testing.assert_array_equal(ob, bufs.out.bfloat16().float().cpu().numpy())


@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
def test_shared_one_call_equals_four_steps(ws):
    _need_gpu()
    prob = make_problem(SMALL["hot"])
    sw = np.random.default_rng(3).random(prob.cfg.tokens).astype(np.float32)
    layer, one = _gpu_forward_shared(prob, sw, 16, ws=ws)
    _, four = _gpu_forward_shared(prob, sw, 16, ws=ws, layer=layer, steps=True)
    e2 = prob.cfg.experts + -(-prob.cfg.tokens // 16)
    for f in ("expert_offsets", "sorted_pair_ids", "pair_pos", "act", "y", "out"):
        a, b = getattr(one, f), getattr(four, f)
        if f == "expert_offsets":  # the buffer has room for 1024 experts; e2 + 1 are written
            a, b = a[:e2 + 1], b[:e2 + 1]
        if a.dtype == torch.float32:
            a, b = a.view(torch.int32), b.view(torch.int32)
        assert torch.equal(a, b), f


@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
def test_forward_with_shared_full_decode_m32(ws):
    _need_gpu()
    prob = make_problem("decode_m32")
    _, bufs = _gpu_forward_shared(prob, ws=ws)
    _close(bufs.out.cpu().numpy(), _shared_ref(prob, None)["out"], "out")


def test_forward_with_shared_full_prefill_every_element():
    """prefill M=8192 with the shared expert (16 shared table entries): every element of
    out, sh_act, sh_out and the routed rows of act and y against the oracle."""
    _need_gpu()
    prob = make_problem("prefill_m8192")
    cfg = prob.cfg
    sw = np.random.default_rng(8).random(cfg.tokens).astype(np.float32)
    layer, bufs = _gpu_forward_shared(prob, sw, ws=True)
    assert layer.rows_per_shared_slot(cfg.tokens) == 512
    shared = tuple(prob.shared_weight(mt) for mt in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN))
    routed = _full_ref("prefill_m8192")
    ref = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                 None, None, None, hidden=cfg.hidden, inter=cfg.inter,
                                 shared=shared, shared_weights=sw, routed=routed)
    _close(bufs.out.cpu().numpy(), ref["out"], "out")
    g_act, g_out = layer.shared_rows_of(bufs, cfg.tokens)
    _close(g_act.cpu().numpy(), ref["sh_act"], "sh_act")
    _close(g_out.cpu().numpy(), ref["sh_out"], "sh_out")
    # The routed experts sort before the shared entries, in the plain routing's order.
    kept = int(routed["sort"].expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], routed["act"][:kept], "act (routed rows)")
    _close(bufs.y.cpu().numpy()[:kept], routed["y"][:kept], "y (routed rows)")


# --------------------------------------------------------------------------- #
# Non-gated experts (up and down only) with a chosen activation
# --------------------------------------------------------------------------- #

def _nongated_ref(prob, activation):
    cfg = prob.cfg
    fns = [lambda e, m=m: prob.expert_weight(m, e, cache=True) for m in (MATRIX_UP, MATRIX_DOWN)]
    return orc.moe_forward_nongated(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                    *fns, hidden=cfg.hidden, inter=cfg.inter, activation=activation)


def _check_nongated(prob, bufs, activation):
    ref = _nongated_ref(prob, activation)
    rs = ref["sort"]
    _check_sort(bufs, rs, prob.cfg.experts, prob.cfg.pairs)
    kept = int(rs.expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], ref["act"][:kept], "act")
    _close(bufs.y.cpu().numpy()[:kept], ref["y"][:kept], "y")
    _close(bufs.out.cpu().numpy(), ref["out"], "out")


def _gpu_forward_nongated(prob, activation, ws=False, null=(), **opts):
    from workloads.device import upload_inputs, upload_layer
    import nvfp4_weight_quantized_moe_b200 as nvm
    layer = upload_layer(prob, activation=activation)
    x, ids, w = upload_inputs(prob)
    bufs = layer.buffers(prob.cfg.tokens)
    for t in (bufs.act, bufs.y, bufs.out):
        t.fill_(float("nan"))
    workspace = layer.workspace(prob.cfg.tokens) if ws else None
    if workspace is not None:
        workspace.fill_(0xFF)
    layer.forward(x, ids, w, bufs, workspace=workspace, **opts)
    torch.cuda.synchronize()
    assert nvm.device_error() == 0
    return layer, bufs


# (path options): decode kernel automatic and forced shapes; tcgen05 16- and 128-row passes.
NONGATED_PATHS = [dict(), dict(path=1, split=4, tiles=1, depth=2, staging=1),
                  dict(path=1, split=4, tiles=1, depth=2, staging=2),
                  dict(path=1, split=1, tiles=2, depth=3, staging=1),
                  dict(path=1, split=1, tiles=2, depth=3, staging=2),
                  dict(ws=True, path=2, tiles=2), dict(ws=True, path=2, tiles=16),
                  dict(ws=True, path=2, tiles=4), dict(ws=True, path=2, tiles=24),
                  dict(ws=True, path=2, tiles=32)]


@pytest.mark.parametrize("opts", NONGATED_PATHS, ids=lambda o: "-".join(f"{k}{v}" for k, v in o.items()) or "auto")
@pytest.mark.parametrize("activation", ["relu2", "silu"])
@pytest.mark.parametrize("name", ["tiny", "ragged", "hot", "zipf", "longk"])
def test_nongated_forward_small(name, activation, opts):
    _need_gpu()
    prob = make_problem(SMALL[name])
    _, bufs = _gpu_forward_nongated(prob, activation, **opts)
    _check_nongated(prob, bufs, activation)


@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
def test_nongated_null_experts_and_four_step_calls(ws):
    _need_gpu()
    prob = make_problem(SMALL["hot"], null_experts=[0, 4])
    opts = dict(ws=True, path=2) if ws else {}
    _, one = _gpu_forward_nongated(prob, "relu2", **opts)
    _check_nongated(prob, one, "relu2")
    _, four = _gpu_forward_nongated(prob, "relu2", steps=True, **opts)
    for f in ("act", "y", "out"):
        assert torch.equal(getattr(one, f).view(torch.int32), getattr(four, f).view(torch.int32)), f


@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
def test_nongated_full_decode_m32(ws):
    # The skewed decode workload's shapes (H4096, I1536, 128 experts) as a non-gated layer.
    _need_gpu()
    prob = make_problem("decode_m32")
    _, bufs = _gpu_forward_nongated(prob, "relu2", ws=ws)
    _check_nongated(prob, bufs, "relu2")


def test_nongated_rejects_an_unknown_activation():
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    from nvfp4_weight_quantized_moe_b200 import _binding as B
    prob = make_problem(SMALL["tiny"])
    layer, bufs = _gpu_forward_nongated(prob, "silu")
    cfg = prob.cfg
    from workloads.device import upload_inputs
    x, ids, w = upload_inputs(prob)
    st = B._lib.nvfp4_moe_up_act(x.data_ptr(), layer.up.tables, bufs.act.data_ptr(),
                                 bufs.expert_offsets.data_ptr(), bufs.sorted_pair_ids.data_ptr(),
                                 bufs.active_experts.data_ptr(), bufs.active_count.data_ptr(),
                                 cfg.inter, cfg.hidden, 2, cfg.tokens, cfg.topk, 7, None, None)
    assert st == 1
    assert nvm.device_error() == 0


# --------------------------------------------------------------------------- #
# Load-time scale check: bit-exact counts
# --------------------------------------------------------------------------- #

def _scale_table(scales, null=()):
    """Tables over device scale arrays; packed entries only mark NULL experts."""
    import nvfp4_weight_quantized_moe_b200 as nvm
    dev = [torch.from_numpy(s).cuda() for s in scales]
    sp = torch.tensor([0 if i in null else d.data_ptr() for i, d in enumerate(dev)],
                      dtype=torch.int64, device="cuda")
    pp = sp.clone()
    return dev, sp, pp, nvm.ExpertTables(pp.data_ptr(), sp.data_ptr(), None)


@pytest.mark.parametrize("e,n,k,null", [(7, 96, 512, (2,)), (3, 4096, 2048, ()), (1, 16, 256, ())])
def test_check_scales_counts_bit_exact(e, n, k, null):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(e * n + k)
    scales = []
    for i in range(e):
        s = rng.integers(0x18, 0x49, (n, k // 16), dtype=np.uint8)
        planted = rng.integers(0, s.size, int(rng.integers(0, 40)))
        s.reshape(-1)[planted] = rng.choice(np.array([0x7F, 0xFF, 0x81, 0xB8, 0xFE, 0x80, 0x7E],
                                                     dtype=np.uint8), planted.size)
        scales.append(s)
    dev, sp, pp, t = _scale_table(scales, null)
    bad = torch.zeros(e, dtype=torch.int32, device="cuda")
    nvm.check_scales(t, e, n, k, bad)
    torch.cuda.synchronize()
    expect = np.array([0 if i in null else orc.count_bad_scales(s) for i, s in enumerate(scales)])
    np.testing.assert_array_equal(bad.cpu().numpy(), expect)
    nvm.check_scales(t, e, n, k, bad)  # the counts accumulate
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bad.cpu().numpy(), 2 * expect)


def test_check_scales_every_code_and_full_down_table():
    # Every code once per row (128 bad of 256), then the decode M=256 down
    # projection's scale table (256 experts of 7168 x 2048) with a few planted codes.
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    codes = np.tile(np.arange(256, dtype=np.uint8), (16, 1))  # 16 rows x k = 4096
    _, _, _, t = _scale_table([codes])
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    nvm.check_scales(t, 1, 16, 4096, bad)
    torch.cuda.synchronize()
    assert int(bad.item()) == 16 * 128 == orc.count_bad_scales(codes)

    e, n, k = 256, 7168, 2048
    rng = np.random.default_rng(77)
    big = rng.integers(0x18, 0x49, (e, n, k // 16), dtype=np.uint8)
    flat = big.reshape(-1)
    idx = rng.integers(0, flat.size, 300)
    flat[idx] = 0xFF
    flat[idx[:100]] = 0x80  # -0 passes
    d = torch.from_numpy(big).cuda()
    ptrs = torch.tensor([d.data_ptr() + i * d.stride(0) for i in range(e)], dtype=torch.int64,
                        device="cuda")
    t = nvm.ExpertTables(ptrs.data_ptr(), ptrs.data_ptr(), None)
    bad = torch.zeros(e, dtype=torch.int32, device="cuda")
    nvm.check_scales(t, e, n, k, bad)
    torch.cuda.synchronize()
    expect = np.array([orc.count_bad_scales(big[i]) for i in range(e)])
    np.testing.assert_array_equal(bad.cpu().numpy(), expect)


# --------------------------------------------------------------------------- #
# Sharding across ranks, each rank's forward run in turn on this GPU
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("kind", ["column", "row"])
@pytest.mark.parametrize("e,n,k,tp", [(3, 96, 512, 2), (2, 48, 768, 3), (1, 64, 320, 5),
                                       (4, 256, 1536, 6), (2, 26, 208, 13)])
def test_shard_nvfp4_bit_exact(kind, e, n, k, tp):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    if kind == "column" and n % tp or kind == "row" and ((k // 2) % tp or (k // 16) % tp):
        pytest.skip("shape not shardable at this tp")
    rng = np.random.default_rng(e * n + k + tp)
    packed = rng.integers(0, 256, (e, n, k // 2), dtype=np.uint8)
    scale = rng.integers(0, 256, (e, n, k // 16), dtype=np.uint8)
    dp, ds = torch.from_numpy(packed).cuda(), torch.from_numpy(scale).cuda()
    code = nvm.SHARD_COLUMN if kind == "column" else nvm.SHARD_ROW
    for r in range(tp):
        po, so = nvm.shard_nvfp4(dp, ds, code, r, tp)
        torch.cuda.synchronize()
        for i in range(e):
            ep, es = orc.shard_nvfp4(packed[i], scale[i], kind, r, tp)
            np.testing.assert_array_equal(po[i].cpu().numpy(), ep)
            np.testing.assert_array_equal(so[i].cpu().numpy(), es)


# I / tp stays a multiple of 256 for tp = 2, 3, 6 (the down projection's K rule).
SHARD_CFG = MoEConfig("shard", hidden=512, inter=1536, experts=6, topk=2, tokens=9,
                      router="uniform", seed=51)


def _sum_over_ranks(prob, layers, ws, shared=False, **opts):
    from workloads.device import upload_inputs
    import nvfp4_weight_quantized_moe_b200 as nvm
    x, ids, w = upload_inputs(prob)
    total = torch.zeros((prob.cfg.tokens, prob.cfg.hidden), dtype=torch.float64, device="cuda")
    for lay in layers:
        bufs = lay.buffers(prob.cfg.tokens)
        bufs.out.fill_(float("nan"))
        workspace = lay.workspace(prob.cfg.tokens) if ws else None
        lay.forward(x, ids, w, bufs, workspace=workspace, **opts)
        total += bufs.out[: prob.cfg.tokens].double()
    torch.cuda.synchronize()
    assert nvm.device_error() == 0
    return total.cpu().numpy()


# Kernels of the sharded forwards: decode kernel; tcgen05 from the shape; the
# CTA-pair kernel at 32- and 192-row passes (the shard widths I/tp = 768, 512,
# 256 all divide into its 128 / 256-row column blocks).
SHARD_PATHS = [dict(), dict(ws=True, path=2), dict(ws=True, path=2, tiles=4), dict(ws=True, path=2, tiles=24),
               dict(ws=True, path=2, tiles=32)]
SHARD_IDS = ["decode-path", "tcgen05", "tcgen05-pair32", "tcgen05-pair192", "tcgen05-pair256"]


@pytest.mark.parametrize("opts", SHARD_PATHS, ids=SHARD_IDS)
@pytest.mark.parametrize("tp", [2, 3, 6])
def test_tensor_parallel_ranks_sum_to_the_full_forward(tp, opts):
    _need_gpu()
    from workloads.device import upload_layer
    prob = make_problem(SHARD_CFG)
    cfg = prob.cfg
    full = upload_layer(prob, shared=True)
    layers = [full.tensor_parallel(r, tp) for r in range(tp)]
    assert layers[0].inter == cfg.inter // tp
    opts = dict(opts)
    got = _sum_over_ranks(prob, layers, opts.pop("ws", False), **opts)
    ref = _shared_ref(prob, None)["out"]
    _close(got, ref, f"sum of {tp} tensor-parallel ranks")


@pytest.mark.parametrize("opts", SHARD_PATHS, ids=SHARD_IDS)
@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_ranks_sum_to_the_full_forward(world, opts):
    _need_gpu()
    from workloads.device import upload_layer
    prob = make_problem(SHARD_CFG)
    full = upload_layer(prob, shared=True)
    layers = [full.expert_parallel(r, world) for r in range(world)]
    opts = dict(opts)
    got = _sum_over_ranks(prob, layers, opts.pop("ws", False), **opts)
    ref = _shared_ref(prob, None)["out"]
    _close(got, ref, f"sum of {world} expert-parallel ranks")


# --------------------------------------------------------------------------- #
# Concatenated / padded twins: bit-exact
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("group", [16, 32])
@pytest.mark.parametrize("ns,k,pad", [((37,), 256, 0), ((64, 5, 130), 512, 0), ((33, 7), 192, 11),
                                     ((1536, 1536), 2048, 0), ((100,), 64, 28)])
def test_transpose_concat_bit_exact(ns, k, pad, group):
    _need_gpu()
    import nvfp4_weight_quantized_moe_b200 as nvm
    rng = np.random.default_rng(sum(ns) + k + pad + group)
    parts = [(rng.integers(0, 256, (n, k // 2), dtype=np.uint8),
              rng.integers(0, 256, (n, k // group), dtype=np.uint8)) for n in ns]
    stride = sum(ns) + pad
    dparts = [(torch.from_numpy(p).cuda(), torch.from_numpy(s).cuda()) for p, s in parts]
    w, sc = nvm.transpose_concat(dparts, group, stride)
    torch.cuda.synchronize()
    ew, es = orc.transpose_concat(parts, k, group, stride)
    np.testing.assert_array_equal(w.cpu().numpy(), ew)
    np.testing.assert_array_equal(sc.cpu().numpy(), es)
