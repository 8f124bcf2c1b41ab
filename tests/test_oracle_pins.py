"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to a library routine, a closed form, a
brute-force evaluation on a tiny input, or an invariant of the expert forward,
chosen so that a plausible slip (swapped nibbles, a wrong scale index, a
transposed operand, a lost token index, an unstable sort) fails at least one
of them.  The last tests plant such slips in a copy of the oracle and check
that the pins catch them.
"""

import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle as orc
from workloads import make_problem
from workloads.generators import MATRIX_DOWN, MATRIX_GATE, MATRIX_UP, MoEConfig

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_e2m1_spot_values.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, code, val = line.split()
            rows.append((fmt, int(code, 16), float(val)))
    return rows


# --------------------------------------------------------------------------- #
# Element formats
# --------------------------------------------------------------------------- #

def test_e2m1_spot_values_from_spec():
    for fmt, code, val in _golden():
        if fmt == "e2m1":
            assert orc.e2m1_value(code) == val


def test_e2m1_table_matches_ml_dtypes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(orc.e2m1_table(), lib)


def test_e4m3_spot_values_from_spec():
    for fmt, code, val in _golden():
        if fmt != "e4m3":
            continue
        if math.isnan(val):
            with pytest.raises(ValueError):
                orc.e4m3_value(code)
        else:
            got = orc.e4m3_value(code)
            assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val)


def test_e4m3_exhaustive_against_torch_and_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ref_t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_m = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    table = orc.e4m3_table()
    finite = 0
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            assert math.isnan(ref_t[c]) and math.isnan(table[c])
            with pytest.raises(ValueError):
                orc.e4m3_value(c)
            continue
        finite += 1
        assert table[c] == ref_t[c] == ref_m[c], hex(c)
    assert finite == 254
    assert np.nanmax(table) == 448.0


def test_every_e2m1_e4m3_product_is_exact_in_bf16_and_f16():
    # The weight value before weight_scale_2 is a product of the two codes; it
    # must survive a BF16 (and an F16) round trip unchanged, which is what lets a
    # 16-bit tensor-core operand carry it exactly.
    e2 = orc.e2m1_table()
    e4 = orc.e4m3_table()
    prods = np.array([a * b for a in e2 for b in e4 if not math.isnan(b)])
    as_bf16 = torch.from_numpy(prods).to(torch.bfloat16).to(torch.float64).numpy()
    as_f16 = prods.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(as_bf16, prods)
    np.testing.assert_array_equal(as_f16, prods)


def test_bf16_decode_matches_torch():
    bits = np.random.default_rng(3).integers(0, 1 << 16, 4096, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # skip inf / NaN patterns
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.bf16_bits_to_f64(bits), ref)


def test_silu_special_values():
    assert orc.silu(np.array(0.0)) == 0.0
    assert abs(float(orc.silu(np.array(1.0))) - 0.7310585786300049) < 1e-15
    assert abs(float(orc.silu(np.array(-1.0))) - (-0.2689414213699951)) < 1e-15
    assert float(orc.silu(np.array(60.0))) == pytest.approx(60.0, rel=1e-15)
    assert abs(float(orc.silu(np.array(-60.0)))) < 1e-24
    assert float(orc.silu(np.array(-1000.0))) == 0.0  # no overflow warning escapes


# --------------------------------------------------------------------------- #
# Dequantisation
# --------------------------------------------------------------------------- #

def test_nibble_order_low_nibble_is_even_k():
    # byte 0x21: low nibble 1 (0.5) at k=0, high nibble 2 (1.0) at k=1.
    packed = np.zeros((1, 8), dtype=np.uint8)
    packed[0, 0] = 0x21
    scale = np.full((1, 1), 0x38, dtype=np.uint8)  # 1.0
    w = orc.dequantize_nvfp4(packed, scale, np.float32(1.0))
    assert w[0, 0] == 0.5 and w[0, 1] == 1.0 and not w[0, 2:].any()


def test_dequant_unit_scales_reduce_to_library_fp4():
    rng = np.random.default_rng(7)
    packed = rng.integers(0, 256, (5, 16), dtype=np.uint8)
    scale = np.full((5, 2), 0x38, dtype=np.uint8)
    w = orc.dequantize_nvfp4(packed, scale, np.float32(1.0))
    lo = (packed & 0xF).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (packed >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(w[:, 0::2], lo)
    np.testing.assert_array_equal(w[:, 1::2], hi)


def test_dequant_block_scale_touches_only_its_16_block():
    rng = np.random.default_rng(8)
    packed = rng.integers(0, 256, (4, 32), dtype=np.uint8)  # K = 64: 4 blocks
    scale = rng.integers(0x18, 0x49, (4, 4), dtype=np.uint8)
    base = orc.dequantize_nvfp4(packed, scale, np.float32(1 / 448))
    bumped = scale.copy()
    bumped[2, 1] += 8  # exponent + 1: that block doubles
    w = orc.dequantize_nvfp4(packed, bumped, np.float32(1 / 448))
    expect = base.copy()
    expect[2, 16:32] *= 2.0
    np.testing.assert_array_equal(w, expect)


def test_dequant_scale2_is_a_plain_factor():
    rng = np.random.default_rng(9)
    packed = rng.integers(0, 256, (3, 8), dtype=np.uint8)
    scale = rng.integers(0x18, 0x49, (3, 1), dtype=np.uint8)
    a = orc.dequantize_nvfp4(packed, scale, np.float32(1.0))
    b = orc.dequantize_nvfp4(packed, scale, np.float32(0.375))
    np.testing.assert_array_equal(b, a * 0.375)


def test_dequant_rejects_nan_scale():
    packed = np.zeros((1, 8), dtype=np.uint8)
    with pytest.raises(ValueError):
        orc.dequantize_nvfp4(packed, np.array([[0x7F]], dtype=np.uint8), np.float32(1.0))
    with pytest.raises(ValueError):
        orc.dequantize_nvfp4(packed, np.array([[0xFF]], dtype=np.uint8), np.float32(1.0))


# --------------------------------------------------------------------------- #
# Route sort
# --------------------------------------------------------------------------- #

def _brute_sort(ids, num_experts):
    flat = [int(v) for v in np.asarray(ids).reshape(-1)]
    order = []
    for e in range(num_experts):
        for p, v in enumerate(flat):
            if v == e:
                order.append(p)
    return order


@pytest.mark.parametrize("m,k,e", [(1, 2, 8), (7, 3, 5), (33, 8, 128), (64, 4, 3)])
def test_route_sort_brute_force(m, k, e):
    rng = np.random.default_rng(m * 1000 + e)
    ids = rng.integers(0, e, (m, k)).astype(np.int32)
    rs = orc.route_sort(ids, e)
    order = _brute_sort(ids, e)
    assert list(rs.sorted_pair_ids[: len(order)]) == order
    assert rs.expert_offsets[-1] == m * k and rs.dropped == 0
    counts = np.diff(rs.expert_offsets)
    for ex in range(e):
        assert counts[ex] == int((ids == ex).sum())
    for pos, p in enumerate(order):
        assert rs.pair_pos[p] == pos
    active = [ex for ex in range(e) if counts[ex] > 0]
    assert rs.active_count == len(active)
    assert list(rs.active_experts) == active + [-1] * (e - len(active))


def test_route_sort_drops_out_of_range_ids():
    ids = np.array([[0, 5], [-1, 2], [9, 2]], dtype=np.int32)
    rs = orc.route_sort(ids, 4)
    assert rs.dropped == 3
    assert list(rs.sorted_pair_ids[:3]) == [0, 3, 5]
    assert list(rs.pair_pos) == [0, -1, -1, 1, -1, 2]
    assert list(rs.expert_offsets) == [0, 1, 1, 3, 3]
    assert rs.active_count == 2 and list(rs.active_experts) == [0, 2, -1, -1]


# --------------------------------------------------------------------------- #
# The expert forward
# --------------------------------------------------------------------------- #

def _tiny_cfg(**kw):
    base = dict(name="pin", hidden=32, inter=16, experts=3, topk=2, tokens=5,
                router="uniform", seed=77)
    base.update(kw)
    return MoEConfig(**base)


def _run(prob, **kw):
    cfg = prob.cfg
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    return orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                           *fns, hidden=cfg.hidden, inter=cfg.inter, **kw)


def _scalar_weight(prob, m, e, n, k):
    packed, scale, s2 = prob.expert_weight(m, e)
    byte = int(packed[n, k // 2])
    code = (byte >> 4) if (k % 2) else (byte & 0xF)
    return orc.e2m1_value(code) * orc.e4m3_value(int(scale[n, k // 16])) * float(s2)


def test_expert_forward_brute_force_scalar_loops():
    prob = make_problem(_tiny_cfg())
    cfg = prob.cfg
    res = _run(prob)
    x = orc.bf16_bits_to_f64(prob.x_bf16)
    for t in range(cfg.tokens):
        acc = [0.0] * cfg.hidden
        for s in range(cfg.topk):
            e = int(prob.topk_ids[t, s])
            wt = float(prob.topk_weights[t, s])
            h = []
            for n in range(cfg.inter):
                g = sum(_scalar_weight(prob, MATRIX_GATE, e, n, k) * x[t, k] for k in range(cfg.hidden))
                u = sum(_scalar_weight(prob, MATRIX_UP, e, n, k) * x[t, k] for k in range(cfg.hidden))
                h.append(g / (1.0 + math.exp(-g)) * u)
            for j in range(cfg.hidden):
                acc[j] += wt * sum(_scalar_weight(prob, MATRIX_DOWN, e, j, i) * h[i] for i in range(cfg.inter))
        np.testing.assert_allclose(res["out"][t], acc, rtol=1e-12, atol=1e-12)


def test_single_expert_weight_one_is_dense_gated_mlp():
    prob = make_problem(_tiny_cfg(experts=1, topk=1, tokens=4, hidden=48, inter=32))
    res = _run(prob)
    assert np.all(prob.topk_weights == 1.0)
    x = orc.bf16_bits_to_f64(prob.x_bf16)
    wg = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_GATE, 0))
    wu = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_UP, 0))
    wd = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_DOWN, 0))
    dense = (orc.silu(x @ wg.T) * (x @ wu.T)) @ wd.T
    np.testing.assert_allclose(res["out"], dense, rtol=1e-13, atol=1e-13)


def test_unit_vector_input_picks_a_weight_column():
    # x = e_j: gate/up reduce to column j of Wg / Wu, which fails for a
    # transposed operand or a wrong k index.
    prob = make_problem(_tiny_cfg(experts=2, topk=1, tokens=3))
    j = [3, 17, 30]
    prob.x_bf16[:] = 0
    for t in range(3):
        prob.x_bf16[t, j[t]] = 0x3F80  # 1.0
    res = _run(prob)
    rs = res["sort"]
    for t in range(3):
        e = int(prob.topk_ids[t, 0])
        wg = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_GATE, e))
        wu = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_UP, e))
        expect = orc.silu(wg[:, j[t]]) * wu[:, j[t]]
        np.testing.assert_array_equal(res["act"][rs.pair_pos[t]], expect)


def test_token_permutation_invariance():
    prob = make_problem(_tiny_cfg(tokens=9, experts=4, topk=2, seed=5))
    base = _run(prob)["out"]
    perm = np.random.default_rng(1).permutation(9)
    prob.x_bf16 = prob.x_bf16[perm].copy()
    prob.topk_ids = prob.topk_ids[perm].copy()
    prob.topk_weights = prob.topk_weights[perm].copy()
    out = _run(prob)["out"]
    np.testing.assert_allclose(out, base[perm], rtol=1e-13, atol=1e-13)


def test_blend_is_linear_and_one_hot_selects_a_pair():
    prob = make_problem(_tiny_cfg(tokens=4, experts=3, topk=2, seed=6))
    res = _run(prob)
    y, pos = res["y"], res["sort"].pair_pos
    w1 = np.random.default_rng(2).random((4, 2))
    w2 = np.random.default_rng(3).random((4, 2))
    np.testing.assert_allclose(orc.blend(y, w1 + w2, pos),
                               orc.blend(y, w1, pos) + orc.blend(y, w2, pos), rtol=1e-13)
    onehot = np.zeros((4, 2))
    onehot[:, 1] = 1.0
    sel = orc.blend(y, onehot, pos)
    for t in range(4):
        np.testing.assert_array_equal(sel[t], y[pos[t * 2 + 1]])


def test_grouped_forward_equals_per_token_forward():
    prob = make_problem(_tiny_cfg(tokens=11, experts=6, topk=3, hidden=64, inter=48, seed=11))
    cfg = prob.cfg
    res = _run(prob)
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    per_tok = orc.moe_forward_tokens(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                     *fns, tokens=range(cfg.tokens), hidden=cfg.hidden)
    np.testing.assert_allclose(res["out"], per_tok, rtol=1e-12, atol=1e-12)


def test_null_expert_contributes_zero():
    prob = make_problem(_tiny_cfg(tokens=6, experts=3, topk=2, seed=12), null_experts=[1])
    res = _run(prob)
    rs = res["sort"]
    lo, hi = rs.expert_offsets[1], rs.expert_offsets[2]
    assert hi > lo  # expert 1 is routed to
    assert not res["act"][lo:hi].any() and not res["y"][lo:hi].any()
    # Same as zero weights for that expert's slots.
    w = prob.topk_weights.astype(np.float64).copy()
    w[prob.topk_ids == 1] = 0.0
    np.testing.assert_allclose(res["out"], orc.blend(res["y"], w, rs.pair_pos), rtol=1e-13)


def test_down_is_linear_in_scale2():
    prob = make_problem(_tiny_cfg(seed=13))
    a = _run(prob)["y"]
    prob.scale2[MATRIX_DOWN, :] *= np.float32(4.0)
    b = _run(prob)["y"]
    np.testing.assert_allclose(b, 4.0 * a, rtol=1e-14)


# --------------------------------------------------------------------------- #
# Non-gated experts (up and down only)
# --------------------------------------------------------------------------- #

def _run_nongated(prob, activation):
    cfg = prob.cfg
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_UP, MATRIX_DOWN)]
    return orc.moe_forward_nongated(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                    *fns, hidden=cfg.hidden, inter=cfg.inter,
                                    activation=activation)


def test_relu2_special_values():
    z = np.array([-3.0, -1e-30, -0.0, 0.0, 0.5, 1.5, 7.0, -np.inf, np.inf])
    np.testing.assert_array_equal(orc.relu2(z), [0.0, 0.0, 0.0, 0.0, 0.25, 2.25, 49.0, 0.0, np.inf])
    assert orc.ACTIVATIONS["silu"] is orc.silu


@pytest.mark.parametrize("activation", ["relu2", "silu"])
def test_nongated_forward_brute_force_scalar_loops(activation):
    prob = make_problem(_tiny_cfg(seed=78))
    cfg = prob.cfg
    res = _run_nongated(prob, activation)
    x = orc.bf16_bits_to_f64(prob.x_bf16)
    f = ((lambda z: max(z, 0.0) * max(z, 0.0)) if activation == "relu2"
         else (lambda z: z / (1.0 + math.exp(-z))))
    for t in range(cfg.tokens):
        acc = [0.0] * cfg.hidden
        for s in range(cfg.topk):
            e = int(prob.topk_ids[t, s])
            wt = float(prob.topk_weights[t, s])
            h = [f(sum(_scalar_weight(prob, MATRIX_UP, e, n, k) * x[t, k] for k in range(cfg.hidden)))
                 for n in range(cfg.inter)]
            for j in range(cfg.hidden):
                acc[j] += wt * sum(_scalar_weight(prob, MATRIX_DOWN, e, j, i) * h[i] for i in range(cfg.inter))
        np.testing.assert_allclose(res["out"][t], acc, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("activation", ["relu2", "silu"])
def test_nongated_single_expert_weight_one_is_the_dense_mlp(activation):
    prob = make_problem(_tiny_cfg(experts=1, topk=1, tokens=4, hidden=48, inter=32, seed=79))
    res = _run_nongated(prob, activation)
    x = orc.bf16_bits_to_f64(prob.x_bf16)
    wu = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_UP, 0))
    wd = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_DOWN, 0))
    z = x @ wu.T
    h = np.maximum(z, 0.0) ** 2 if activation == "relu2" else z / (1.0 + np.exp(-z))
    np.testing.assert_allclose(res["out"], h @ wd.T, rtol=1e-13, atol=1e-13)


def test_nongated_unit_vector_input_picks_an_up_column():
    # x = e_j: act = f(column j of Wu) (a transposed operand or the gate's
    # matrix in its place fails this).
    prob = make_problem(_tiny_cfg(experts=2, topk=1, tokens=3, seed=80))
    j = [3, 17, 30]
    prob.x_bf16[:] = 0
    for t in range(3):
        prob.x_bf16[t, j[t]] = 0x3F80
    res = _run_nongated(prob, "relu2")
    rs = res["sort"]
    for t in range(3):
        e = int(prob.topk_ids[t, 0])
        wu = orc.dequantize_nvfp4(*prob.expert_weight(MATRIX_UP, e))
        np.testing.assert_array_equal(res["act"][rs.pair_pos[t]], np.maximum(wu[:, j[t]], 0.0) ** 2)


def test_nongated_null_expert_rows_are_zero():
    prob = make_problem(_tiny_cfg(experts=3, topk=1, tokens=6, seed=81), null_experts=[1])
    res = _run_nongated(prob, "silu")
    rs = res["sort"]
    lo, hi = int(rs.expert_offsets[1]), int(rs.expert_offsets[2])
    assert hi > lo
    assert not res["act"][lo:hi].any() and not res["y"][lo:hi].any()


# --------------------------------------------------------------------------- #
# Shared expert
# --------------------------------------------------------------------------- #

def _shared(prob):
    return tuple(prob.shared_weight(m) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN))


def test_shared_expert_all_ones_closed_form():
    # Every weight 1.0 (E2M1 code 2 in both nibbles, E4M3 scale 0x38 = 1,
    # s2 = 1): g = u = S = sum_k x_k, every act entry is SiLU(S) * S and every
    # output entry I * SiLU(S) * S.
    h, i = 64, 32
    ones = lambda n, k: (np.full((n, k // 2), 0x22, np.uint8), np.full((n, k // 16), 0x38, np.uint8),
                         np.float32(1.0))
    x = np.array([[0x3F80] * h, [0xBF00] * h, [0x3E80] * (h // 2) + [0xC000] * (h // 2)],
                 dtype=np.uint16)  # 1, -0.5, (0.25 | -2)
    sums = np.array([h * 1.0, h * -0.5, h // 2 * 0.25 + h // 2 * -2.0])
    sh_act, sh_out = orc.shared_expert(x, ones(i, h), ones(i, h), ones(h, i))
    expect_h = sums / (1.0 + np.exp(-sums)) * sums
    np.testing.assert_allclose(sh_act, np.repeat(expect_h[:, None], i, axis=1), rtol=1e-15)
    np.testing.assert_allclose(sh_out, np.repeat(i * expect_h[:, None], h, axis=1), rtol=1e-14)


def test_shared_expert_equals_a_routed_expert_with_its_weights():
    # Give routed expert 2 the shared weights and route every token to it alone
    # with weight 1: the per-token routed forward must reproduce the shared
    # expert's output (a gate/up swap or a transposed operand breaks this).
    prob = make_problem(_tiny_cfg(tokens=7, experts=4, topk=1, hidden=64, inter=48, seed=21))
    cfg = prob.cfg
    shared = _shared(prob)
    fns = [lambda e, m=m: shared[m] if e == 2 else prob.expert_weight(m, e)
           for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    ids = np.full((cfg.tokens, 1), 2, dtype=np.int32)
    w = np.ones((cfg.tokens, 1), dtype=np.float32)
    routed = orc.moe_forward_tokens(prob.x_bf16, ids, w, cfg.experts, *fns,
                                    tokens=range(cfg.tokens), hidden=cfg.hidden)
    _, sh_out = orc.shared_expert(prob.x_bf16, *shared)
    np.testing.assert_allclose(sh_out, routed, rtol=1e-12, atol=1e-12)


def test_forward_with_shared_adds_the_weighted_shared_output():
    prob = make_problem(_tiny_cfg(tokens=6, experts=4, topk=2, hidden=64, inter=32, seed=22))
    cfg = prob.cfg
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    c = np.random.default_rng(4).random(cfg.tokens)
    base = orc.moe_forward_tokens(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                  *fns, tokens=range(cfg.tokens), hidden=cfg.hidden)
    res1 = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                  *fns, hidden=cfg.hidden, inter=cfg.inter, shared=_shared(prob))
    res_c = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                   *fns, hidden=cfg.hidden, inter=cfg.inter, shared=_shared(prob),
                                   shared_weights=c)
    sh = res1["out"] - base
    np.testing.assert_allclose(res_c["out"], base + c[:, None] * sh, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sh, res1["sh_out"], rtol=1e-10, atol=1e-12)


def test_forward_with_shared_takes_a_precomputed_routed_result():
    prob = make_problem(_tiny_cfg(tokens=5, experts=4, topk=2, hidden=64, inter=32, seed=23))
    cfg = prob.cfg
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    c = np.random.default_rng(6).random(cfg.tokens)
    routed = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *fns,
                             hidden=cfg.hidden, inter=cfg.inter)
    a = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *fns,
                               hidden=cfg.hidden, inter=cfg.inter, shared=_shared(prob),
                               shared_weights=c)
    b = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                               None, None, None, hidden=cfg.hidden, inter=cfg.inter,
                               shared=_shared(prob), shared_weights=c, routed=routed)
    for key in ("act", "y", "out", "sh_act", "sh_out"):
        np.testing.assert_array_equal(a[key], b[key])
    np.testing.assert_array_equal(routed["out"], orc.moe_forward(
        prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *fns, hidden=cfg.hidden,
        inter=cfg.inter)["out"])  # the routed result was not modified in place


@pytest.mark.parametrize("m,k,e,rows", [(1, 2, 8, 1), (7, 3, 5, 2), (33, 8, 128, 16), (40, 1, 3, 64)])
def test_append_shared_routing_layout(m, k, e, rows):
    rng = np.random.default_rng(m + k + e)
    ids = rng.integers(0, e, (m, k)).astype(np.int32)
    w = rng.random((m, k)).astype(np.float32)
    sw = rng.random(m).astype(np.float32)
    ids2, w2 = orc.append_shared_routing(ids, w, e, rows, sw)
    assert ids2.shape == (m, k + 1) and w2.shape == (m, k + 1)
    np.testing.assert_array_equal(ids2[:, :k], ids)
    np.testing.assert_array_equal(w2[:, :k], w)
    np.testing.assert_array_equal(w2[:, k], sw)
    slots = -(-m // rows)
    for t in range(m):
        assert ids2[t, k] == e + t // rows
    assert ids2[:, k].max() == e + slots - 1
    _, w1 = orc.append_shared_routing(ids, w, e, rows)
    assert np.all(w1[:, k] == 1.0)
    # Grouped by expert, the shared rows come last, contiguous and in token order.
    rs = orc.route_sort(ids2, e + slots)
    lo = int(rs.expert_offsets[e])
    assert int(rs.expert_offsets[e + slots]) == lo + m == m * (k + 1)
    np.testing.assert_array_equal(rs.sorted_pair_ids[lo:lo + m] // (k + 1), np.arange(m))
    np.testing.assert_array_equal(rs.sorted_pair_ids[lo:lo + m] % (k + 1), np.full(m, k))


def test_shared_expert_as_extra_slots_equals_the_plain_definition():
    # The grouped forward over the appended routing, whose extra table entries
    # all hold the shared weights, reaches the plain definition, and its shared
    # rows are sh_act / sh_out in token order.
    prob = make_problem(_tiny_cfg(tokens=9, experts=5, topk=2, hidden=64, inter=48, seed=23))
    cfg = prob.cfg
    shared = _shared(prob)
    sw = np.random.default_rng(5).random(cfg.tokens).astype(np.float32)
    rows = 4
    slots = -(-cfg.tokens // rows)
    ids2, w2 = orc.append_shared_routing(prob.topk_ids, prob.topk_weights, cfg.experts, rows, sw)
    fns = [lambda e, m=m: shared[m] if e >= cfg.experts else prob.expert_weight(m, e)
           for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    grouped = orc.moe_forward(prob.x_bf16, ids2, w2, cfg.experts + slots, *fns,
                              hidden=cfg.hidden, inter=cfg.inter)
    plain = orc.moe_forward_shared(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                                   *fns, hidden=cfg.hidden, inter=cfg.inter, shared=shared,
                                   shared_weights=sw)
    np.testing.assert_allclose(grouped["out"], plain["out"], rtol=1e-12, atol=1e-12)
    lo = int(grouped["sort"].expert_offsets[cfg.experts])
    np.testing.assert_allclose(grouped["act"][lo:lo + cfg.tokens], plain["sh_act"], rtol=1e-13)
    np.testing.assert_allclose(grouped["y"][lo:lo + cfg.tokens], plain["sh_out"], rtol=1e-12,
                               atol=1e-13)


# --------------------------------------------------------------------------- #
# Load-time scale check
# --------------------------------------------------------------------------- #

def test_bad_scale_count_against_ml_dtypes_over_every_code():
    codes = np.arange(256, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    expect = [int(np.isnan(v) or v < 0) for v in lib]
    assert [orc.count_bad_scales(np.array([c], dtype=np.uint8)) for c in codes] == expect
    # Closed form: 0x7F and 0x81..0xFF fail (NaN 0x7F / 0xFF, negatives between),
    # 0x00..0x7E and -0 (0x80) pass.
    assert orc.count_bad_scales(codes) == 128
    assert orc.count_bad_scales(np.array([0x80, 0x7E, 0x00], dtype=np.uint8)) == 0
    assert orc.count_bad_scales(np.array([[0x7F, 0x81], [0xFF, 0xFE]], dtype=np.uint8)) == 4


def test_bad_scale_count_of_generated_scales_is_zero():
    prob = make_problem(_tiny_cfg())
    for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN):
        _, scale, _ = prob.expert_weight(m, 0)
        assert orc.count_bad_scales(scale) == 0


# --------------------------------------------------------------------------- #
# Sharding across ranks
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("tp", [2, 3, 4])
def test_shards_reassemble_and_dequantise_to_slices(tp):
    rng = np.random.default_rng(tp)
    n, k = 24, 192  # K/16 = 12 and N divisible by 2, 3, 4
    packed = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    scale = rng.integers(0x18, 0x49, (n, k // 16), dtype=np.uint8)
    s2 = np.float32(0.75)
    full = orc.dequantize_nvfp4(packed, scale, s2)
    cols = [orc.shard_nvfp4(packed, scale, "column", r, tp) for r in range(tp)]
    np.testing.assert_array_equal(np.vstack([c[0] for c in cols]), packed)
    np.testing.assert_array_equal(np.vstack([c[1] for c in cols]), scale)
    rows = [orc.shard_nvfp4(packed, scale, "row", r, tp) for r in range(tp)]
    np.testing.assert_array_equal(np.hstack([r_[0] for r_ in rows]), packed)
    np.testing.assert_array_equal(np.hstack([r_[1] for r_ in rows]), scale)
    for r in range(tp):
        # A row shard is the rank's K slice of the dense weight; a column shard its rows.
        np.testing.assert_array_equal(orc.dequantize_nvfp4(*rows[r], s2),
                                      full[:, r * k // tp:(r + 1) * k // tp])
        np.testing.assert_array_equal(orc.dequantize_nvfp4(*cols[r], s2),
                                      full[r * n // tp:(r + 1) * n // tp])


def test_shard_rules_follow_the_page():
    packed = np.zeros((6, 40), dtype=np.uint8)  # K = 80: K/16 = 5
    scale = np.zeros((6, 5), dtype=np.uint8)
    with pytest.raises(ValueError):
        orc.shard_nvfp4(packed, scale, "row", 0, 2)  # K/16 = 5 not divisible by 2
    with pytest.raises(ValueError):
        orc.shard_nvfp4(packed, scale, "column", 0, 4)  # N = 6 not divisible by 4
    p, s_ = orc.shard_nvfp4(packed, scale, "replicated", 1, 4)
    assert p.shape == packed.shape and s_.shape == scale.shape


def _sharded_fns(prob, tp, rank):
    """Weight callbacks of one tensor-parallel rank: gate/up by rows, down by K."""
    def fn(m):
        kind = "row" if m == MATRIX_DOWN else "column"

        def get(e):
            w = prob.expert_weight(m, e)
            if w is None:
                return None
            p, s_ = orc.shard_nvfp4(w[0], w[1], kind, rank, tp)
            return p, s_, w[2]
        return get
    return [fn(m) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]


@pytest.mark.parametrize("tp", [2, 4])
def test_tensor_parallel_partial_outputs_sum_to_the_full_forward(tp):
    prob = make_problem(_tiny_cfg(tokens=6, experts=4, topk=2, hidden=64, inter=64, seed=31))
    cfg = prob.cfg
    full = _run(prob)["out"]
    total = np.zeros_like(full)
    for r in range(tp):
        res = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts,
                              *_sharded_fns(prob, tp, r), hidden=cfg.hidden,
                              inter=cfg.inter // tp)
        total += res["out"]
    np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_expert_parallel_partial_outputs_sum_to_the_full_forward(world):
    cfg = _tiny_cfg(tokens=7, experts=8, topk=3, hidden=64, inter=48, seed=32)
    full = _run(make_problem(cfg))["out"]
    total = np.zeros_like(full)
    owned = []
    for r in range(world):
        lo, hi = orc.expert_owner_range(cfg.experts, world, r)
        owned += list(range(lo, hi))
        assert hi - lo in (cfg.experts // world, -(-cfg.experts // world))
        prob = make_problem(cfg, null_experts=[e for e in range(cfg.experts) if not lo <= e < hi])
        total += _run(prob)["out"]
    assert owned == list(range(cfg.experts))
    np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- #
# transpose_u8
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 5), (16, 9), (33, 64)])
def test_transpose_u8_against_numpy_and_involution(rows, cols):
    src = np.random.default_rng(rows * cols).integers(0, 256, (rows, cols), dtype=np.uint8)
    t = orc.transpose_u8(src, rows, cols)
    np.testing.assert_array_equal(t, src.T)
    np.testing.assert_array_equal(orc.transpose_u8(t, cols, rows), src)


@pytest.mark.parametrize("group", [16, 32])
def test_transpose_concat_is_side_by_side_transposes_with_zero_pad(group):
    rng = np.random.default_rng(group)
    k = 128
    ns = [5, 1, 12]
    parts = [(rng.integers(0, 256, (n, k // 2), dtype=np.uint8),
              rng.integers(0, 256, (n, k // group), dtype=np.uint8)) for n in ns]
    for stride in (sum(ns), 32):
        w, sc = orc.transpose_concat(parts, k, group, stride)
        assert w.shape == (k // 2, stride) and sc.shape == (k // group, stride)
        np.testing.assert_array_equal(w[:, :sum(ns)], np.hstack([p.T for p, _ in parts]))
        np.testing.assert_array_equal(sc[:, :sum(ns)], np.hstack([s_.T for _, s_ in parts]))
        assert not w[:, sum(ns):].any() and not sc[:, sum(ns):].any()
    # One part, stride = N: the single twin of transpose_for_gemm_gs (transpose_u8 twice).
    p, s_ = parts[2]
    w, sc = orc.transpose_concat([parts[2]], k, group, 12)
    np.testing.assert_array_equal(w, orc.transpose_u8(p, 12, k // 2))
    np.testing.assert_array_equal(sc, orc.transpose_u8(s_, 12, k // group))
    with pytest.raises(ValueError):
        orc.transpose_concat(parts, k, group, sum(ns) - 1)
    with pytest.raises(ValueError):
        orc.transpose_concat([], k, group, 8)


# --------------------------------------------------------------------------- #
# The parity metric: relative L2 error over all elements
# --------------------------------------------------------------------------- #

def test_relative_l2_hand_computed_pairs():
    # ref = (1, 2, 2): |ref| = 3; got - ref = (0.3, 0, 0.4): |diff| = 0.5, ratio 1/6.
    ref = np.array([1.0, 2.0, 2.0])
    assert orc.relative_l2(ref + np.array([0.3, 0.0, 0.4]), ref) == pytest.approx(1 / 6, rel=1e-14)
    # The sign of the error does not matter.
    assert orc.relative_l2(ref - np.array([0.3, 0.0, 0.4]), ref) == pytest.approx(1 / 6, rel=1e-14)
    # 2-D: one norm over every element (ref = diag(3, 4): |ref| = 5; one off-diagonal 1: 1/5),
    # not a mean of per-row ratios (that would give (1/3 + 0) / 2).
    ref2 = np.array([[3.0, 0.0], [0.0, 4.0]])
    got2 = ref2 + np.array([[0.0, 1.0], [0.0, 0.0]])
    assert orc.relative_l2(got2, ref2) == pytest.approx(0.2, rel=1e-14)
    # A float32 result is compared exactly as given: ref = (3, 4), got = (3, 4.5) as f32.
    assert orc.relative_l2(np.array([3.0, 4.5], np.float32), np.array([3.0, 4.0])) == 0.1
    assert orc.relative_l2(ref, ref) == 0.0


def test_relative_l2_zero_reference():
    z = np.zeros(5)
    assert orc.relative_l2(z, z) == 0.0
    assert orc.relative_l2(np.array([0.0, 0.0, 0.25, 0.0, 0.0]), z) == math.inf


def test_relative_l2_uniform_relative_error_is_that_error():
    # got = (1 + eps) * ref gives |eps| for any nonzero ref, at any common scale.
    ref = np.random.default_rng(5).standard_normal(1000)
    for eps in (1e-3, -2.5e-4, 0.5):
        assert orc.relative_l2((1 + eps) * ref, ref) == pytest.approx(abs(eps), rel=1e-9)
        assert orc.relative_l2((1 + eps) * 2.0 ** 60 * ref, 2.0 ** 60 * ref) == pytest.approx(
            abs(eps), rel=1e-9)


# --------------------------------------------------------------------------- #
# Planted mistakes: the pins above must catch them
# --------------------------------------------------------------------------- #

def test_pins_catch_swapped_nibble_order(monkeypatch):
    real = orc.dequantize_nvfp4

    def swapped(packed, scale, s2):
        p = np.asarray(packed, dtype=np.uint8)
        return real(((p & 0xF) << 4) | (p >> 4), scale, s2)

    monkeypatch.setattr(orc, "dequantize_nvfp4", swapped)
    with pytest.raises(AssertionError):
        test_nibble_order_low_nibble_is_even_k()


def test_pins_catch_a_transposed_operand(monkeypatch):
    import oracle.nvfp4_moe_oracle as mod
    real = mod._dense

    def transposed(fn, e):
        w = real(fn, e)
        if w is None or w.shape[0] != w.shape[1]:
            return w
        return np.ascontiguousarray(w.T)

    monkeypatch.setattr(mod, "_dense", transposed)
    prob = make_problem(_tiny_cfg(hidden=32, inter=32, experts=2, topk=1, tokens=3))
    j = [3, 17, 30]
    prob.x_bf16[:] = 0
    for t in range(3):
        prob.x_bf16[t, j[t]] = 0x3F80
    res = _run(prob)
    rs = res["sort"]
    bad = 0
    for t in range(3):
        e = int(prob.topk_ids[t, 0])
        wg = real(lambda ex: prob.expert_weight(MATRIX_GATE, ex), e)
        wu = real(lambda ex: prob.expert_weight(MATRIX_UP, ex), e)
        expect = orc.silu(wg[:, j[t]]) * wu[:, j[t]]
        bad += int(not np.array_equal(res["act"][rs.pair_pos[t]], expect))
    assert bad > 0


def test_pins_catch_swapped_gate_and_up_in_the_shared_expert(monkeypatch):
    real = orc.shared_expert

    def swapped(x, gate, up, down):
        return real(x, up, gate, down)

    monkeypatch.setattr(orc, "shared_expert", swapped)
    with pytest.raises(AssertionError):
        test_shared_expert_equals_a_routed_expert_with_its_weights()


def test_pins_catch_an_unstable_sort(monkeypatch):
    import oracle.nvfp4_moe_oracle as mod

    def ties_reversed(keys):
        keys = np.asarray(keys)
        return np.lexsort((-np.arange(keys.size), keys))

    monkeypatch.setattr(mod, "_stable_order", ties_reversed)
    with pytest.raises(AssertionError):
        test_route_sort_brute_force(33, 8, 128)


def test_pins_catch_a_scale_slice_off_by_one_group(monkeypatch):
    real = orc.shard_nvfp4

    def shifted(packed, scale, kind, rank, tp):
        p, s_ = real(packed, scale, kind, rank, tp)
        if kind == "row" and rank > 0:
            groups = np.asarray(scale).shape[1] // tp
            s_ = np.asarray(scale)[:, rank * groups - 1:(rank + 1) * groups - 1].copy()
        return p, s_

    monkeypatch.setattr(orc, "shard_nvfp4", shifted)
    with pytest.raises(AssertionError):
        test_shards_reassemble_and_dequantise_to_slices(2)


def test_pins_catch_interleaved_shared_slots(monkeypatch):
    real = orc.append_shared_routing

    def interleaved(ids, w, e, rows, sw=None):
        ids2, w2 = real(ids, w, e, rows, sw)
        m = ids2.shape[0]
        slots = -(-m // rows)
        ids2[:, -1] = e + np.arange(m) % slots  # round-robin instead of token blocks
        return ids2, w2

    monkeypatch.setattr(orc, "append_shared_routing", interleaved)
    with pytest.raises(AssertionError):
        test_append_shared_routing_layout(33, 8, 128, 16)


def test_pins_catch_flagging_negative_zero(monkeypatch):
    import oracle.nvfp4_moe_oracle as mod
    real = mod.count_bad_scales

    def sign_bit(codes):
        c = np.asarray(codes, dtype=np.uint8).reshape(-1)
        return real(c) + int(np.count_nonzero(c == 0x80))

    monkeypatch.setattr(orc, "count_bad_scales", sign_bit)
    with pytest.raises(AssertionError):
        test_bad_scale_count_against_ml_dtypes_over_every_code()


def test_pins_catch_a_missing_column_offset_in_the_twins(monkeypatch):
    def no_offset(parts, k, group, stride):
        half_k, groups = k // 2, k // group
        w = np.zeros((half_k, stride), np.uint8)
        sc = np.zeros((groups, stride), np.uint8)
        for p, s_ in parts:  # every part written at column 0
            w[:, :p.shape[0]] = np.asarray(p).T
            sc[:, :p.shape[0]] = np.asarray(s_).T
        return w, sc

    monkeypatch.setattr(orc, "transpose_concat", no_offset)
    with pytest.raises(AssertionError):
        test_transpose_concat_is_side_by_side_transposes_with_zero_pad(16)


def test_pins_catch_a_squared_or_misnormalised_relative_l2(monkeypatch):
    import oracle.nvfp4_moe_oracle as mod
    real = mod.relative_l2
    wrong = [lambda g, r: real(g, r) ** 2,                                      # no square root
             lambda g, r: float(np.max(np.abs(np.asarray(g, np.float64) - r))
                                / np.max(np.abs(r))),                          # max norm
             lambda g, r: float(np.linalg.norm(np.asarray(g, np.float64) - r)
                                / np.linalg.norm(g))]                          # divided by |got|
    for fn in wrong:
        monkeypatch.setattr(orc, "relative_l2", fn)
        with pytest.raises(AssertionError):
            test_relative_l2_hand_computed_pairs()


# --------------------------------------------------------------------------- #
# The pooled full-size driver of the oracle (tests/_oracle_pool.py)
# --------------------------------------------------------------------------- #

def test_pooled_oracle_equals_the_plain_oracle():
    # Expert blocks run in separate processes with the other experts NULL, then
    # gathered: the same act, y and out as one plain oracle call.
    from _oracle_pool import moe_forward_pooled
    cfg = MoEConfig("pool", hidden=512, inter=256, experts=13, topk=3, tokens=40,
                    router="zipf", seed=61)
    prob = make_problem(cfg)
    fns = [lambda e, m=m: prob.expert_weight(m, e) for m in (MATRIX_GATE, MATRIX_UP, MATRIX_DOWN)]
    ref = orc.moe_forward(prob.x_bf16, prob.topk_ids, prob.topk_weights, cfg.experts, *fns,
                          hidden=cfg.hidden, inter=cfg.inter)
    got = moe_forward_pooled(cfg, workers=3, block=2)
    np.testing.assert_array_equal(got["sort"].sorted_pair_ids, ref["sort"].sorted_pair_ids)
    for key in ("act", "y", "out"):
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-12, atol=1e-300)


def test_pins_catch_the_activation_applied_after_down(monkeypatch):
    import oracle.nvfp4_moe_oracle as mod
    real_down = mod.down_proj

    def late(x_bf16, topk_ids, topk_weights, num_experts, up_fn, down_fn, hidden, inter,
             activation):
        rs = mod.route_sort(topk_ids, num_experts)
        x = mod.bf16_bits_to_f64(x_bf16)
        act = np.zeros((rs.sorted_pair_ids.size, inter))
        for a in range(rs.active_count):
            e = int(rs.active_experts[a])
            lo, hi = int(rs.expert_offsets[e]), int(rs.expert_offsets[e + 1])
            act[lo:hi] = x[rs.sorted_pair_ids[lo:hi] // np.asarray(topk_ids).shape[1]] @ mod._dense(up_fn, e).T
        y = mod.ACTIVATIONS[activation](real_down(act, rs, down_fn, hidden))
        return {"sort": rs, "act": act, "y": y, "out": mod.blend(y, topk_weights, rs.pair_pos)}

    monkeypatch.setattr(orc, "moe_forward_nongated", late)
    with pytest.raises(AssertionError):
        test_nongated_single_expert_weight_one_is_the_dense_mlp("relu2")
