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


# Decode launch shapes: (split, tiles, depth); zeros pick from the shape.
PLANS = [(0, 0, 0), (4, 1, 2), (2, 1, 2), (1, 1, 2), (1, 1, 3), (1, 2, 2), (1, 2, 3)]


@pytest.mark.parametrize("plan", PLANS, ids=lambda p: "s%d-t%d-d%d" % p)
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small(name, plan):
    _need_gpu()
    prob = make_problem(SMALL[name])
    split, tiles, depth = plan
    _, bufs = _gpu_forward(prob, path=1 if any(plan) else 0, split=split, tiles=tiles, depth=depth)
    _check_full(prob, bufs)


def test_gate_up_four_tiles():
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
                     cfg.hidden, cap, cfg.tokens, cfg.topk, path=1, split=1, tiles=4, depth=2)
    torch.cuda.synchronize()
    ref = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *_fns(prob),
                          hidden=cfg.hidden, inter=cfg.inter)
    kept = int(ref["sort"].expert_offsets[-1])
    _close(bufs.act.cpu().numpy()[:kept], ref["act"][:kept], "act")


# tcgen05 path: token rows per pass 16 (tiles=2) or 128 (tiles=16); 0 = from the shape.
@pytest.mark.parametrize("tiles", [0, 2, 16])
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_tcgen05(name, tiles):
    _need_gpu()
    prob = make_problem(SMALL[name])
    _, bufs = _gpu_forward(prob, ws=True, path=2, tiles=tiles)
    _check_full(prob, bufs)


def test_null_experts_tcgen05():
    _need_gpu()
    prob = make_problem(SMALL["ragged"], null_experts=[1, 3])
    _, bufs = _gpu_forward(prob, ws=True, path=2)
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


def _check_sampled(prob, bufs, tokens):
    cfg = prob.cfg
    rs = orc.route_sort(prob.topk_ids, cfg.experts)
    _check_sort(bufs, rs, cfg.experts, cfg.pairs)
    ref = orc.moe_forward_tokens(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                 *_fns(prob), tokens=tokens, hidden=cfg.hidden)
    _close(bufs.out.cpu().numpy()[tokens], ref, "out (sampled tokens)")
    # act / y rows of those tokens' pairs, by sorted position
    x = orc.bf16_bits_to_f64(prob.x_bf16)
    act = bufs.act.cpu().numpy()
    y = bufs.y.cpu().numpy()
    for t in tokens[:1]:
        for s in range(cfg.topk):
            e = int(prob.topk_ids[t, s])
            pos = int(rs.pair_pos[t * cfg.topk + s])
            wg = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_GATE, e, cache=True))
            wu = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_UP, e, cache=True))
            wd = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_DOWN, e, cache=True))
            h = orc.silu(wg @ x[t]) * (wu @ x[t])
            _close(act[pos], h, f"act[{pos}]")
            _close(y[pos], wd @ h, f"y[{pos}]")


@pytest.mark.parametrize("ws", [False, True], ids=["decode-path", "tcgen05"])
@pytest.mark.parametrize("name", ["decode_m256", "prefill_m8192"])
def test_forward_full_size_sampled(name, ws):
    """Full-size launch, checked on a seeded sample of tokens (tokens are independent)."""
    _need_gpu()
    prob = make_problem(name)
    _, bufs = _gpu_forward(prob, ws=ws)
    mid = int(np.random.default_rng(99).integers(1, prob.cfg.tokens - 1))
    tokens = [0, mid, prob.cfg.tokens - 1]
    _check_sampled(prob, bufs, tokens)
