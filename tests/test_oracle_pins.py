"""Pins for the CPU oracle, independent of the oracle itself (CPU only).

Each check ties the oracle to something other than its own code: values the
pages print, small examples worked by hand, brute force in exact rational
arithmetic with an independent round-to-fp32, exhaustive enumeration over
small trit patterns, and algebraic invariants of the definitions.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from packed_ternary_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------- independent exact helpers
def rn_f32(fr: Fraction) -> Fraction:
    """Round an exact rational to the nearest fp32 value (ties to even), as a Fraction."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    q = a / quantum
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def rint_half_even(fr: Fraction) -> int:
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


def f32(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def bf16_bits(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


# ----------------------------------------------------------- pages' numbers
def test_bpw_matches_pages_tq():
    g = load("bpw_pages.json")
    for row in g["tq_g256"] + g["tq2p_groups"] + g["matched_bpw"]:
        got = oracle.bits_per_weight("tq", row["planes"], row["group"])
        assert round(got, row["digits"]) == pytest.approx(row["printed"]), row
    # exact values behind the rounded 2.06 and 4.1
    assert oracle.bits_per_weight("tq", 1, 256) == 2.0625
    assert oracle.bits_per_weight("tq", 2, 256) == 4.125


def test_bpw_matches_pages_bt3():
    g = load("bpw_pages.json")["bt3"]
    got = oracle.bt3_information_bpw(g["depth"], g["group"], g["scale_trits"])
    assert round(got, g["digits"]) == pytest.approx(g["printed"])
    assert got == pytest.approx(51 * math.log2(3) / 16)
    assert 3 ** g["depth"] == 27


def test_codebook_is_27_log_spaced_1e4_to_1e1():
    cb = synth.codebook27().astype(np.float64)
    assert cb.shape == (27,)
    assert cb[0] == pytest.approx(1e-4, rel=1e-7) and cb[-1] == pytest.approx(1e-1, rel=1e-7)
    ratio = cb[1:] / cb[:-1]
    assert np.allclose(ratio, 10 ** (3 / 26), rtol=1e-6)


# ------------------------------------------------------- quantisation
def test_quantize_act_worked_examples():
    for ex in load("worked_examples.json")["quantize_act"]:
        xq, sx = oracle.quantize_act(bf16_bits([ex["x"]]))
        assert xq[0].tolist() == ex["xq"], ex["note"]
        assert Fraction(float(sx[0])) == rn_f32(Fraction(ex["sx_num"], ex["sx_den"]))


def _quantize_fraction(x_vals):
    a = max(abs(Fraction(float(v))) for v in x_vals)
    if a == 0:
        return [0] * len(x_vals), Fraction(0)
    inv = rn_f32(Fraction(127) / a)
    q = [max(-127, min(127, rint_half_even(rn_f32(Fraction(float(v)) * inv)))) for v in x_vals]
    return q, rn_f32(a / 127)


def test_quantize_act_vs_exact_rationals():
    g = np.random.default_rng(11)
    for trial in range(40):
        k = int(g.integers(1, 40))
        x = synth.f32_to_bf16_bits((g.standard_normal(k) * 10 ** g.uniform(-3, 3)).astype(np.float32))
        xq, sx = oracle.quantize_act(x[None])
        xf = synth.bf16_bits_to_f32(x)
        q_ref, s_ref = _quantize_fraction(xf)
        assert xq[0].tolist() == q_ref
        assert Fraction(float(sx[0])) == s_ref
        assert np.max(np.abs(xq)) == 127


def test_quantize_act_zero_and_ties():
    xq, sx = oracle.quantize_act(np.zeros((2, 7), np.uint16))
    assert not xq.any() and not sx.any()
    # values at exact .5 after scaling: absmax 2 -> inv 63.5; x = 1 -> 63.5 -> 64 (even)
    xq, _ = oracle.quantize_act(bf16_bits([[2.0, 1.0, -1.0, 0.0]]))
    assert xq[0].tolist() == [127, 64, -64, 0]


# ---------------------------------------------------------- dequantise
def test_dequantize_brute_force_loops():
    g = np.random.default_rng(3)
    n, k, P, grp = 5, 48, 3, 16
    t = g.integers(-1, 2, size=(P, n, k)).astype(np.int8)
    s = (g.standard_normal((P, n, k // grp)) * 0.1).astype(np.float16)
    w = oracle.dequantize("tq", t, grp, scales=s)
    for r in range(n):
        for c in range(k):
            ref = sum(Fraction(float(s[p, r, c // grp])) * int(t[p, r, c]) for p in range(P))
            assert Fraction(w[r, c]) == ref
    idx = g.integers(0, 27, size=(n, k // 16)).astype(np.uint8)
    cb = synth.codebook27()
    w3 = oracle.dequantize("bt3", t, 16, idx=idx, codebook=cb)
    for r in range(n):
        for c in range(k):
            lvl = int(t[0, r, c]) + 3 * int(t[1, r, c]) + 9 * int(t[2, r, c])
            assert Fraction(w3[r, c]) == Fraction(float(cb[idx[r, c // 16]])) * lvl
    wb = oracle.dequantize("bitnet", t[:1], tensor_scale=0.02)
    assert np.array_equal(wb, float(np.float32(0.02)) * t[0])


def test_bt3_levels_cover_27_values():
    # every (t0, t1, t2) gives a distinct level in -13..13
    levels = {t0 + 3 * t1 + 9 * t2 for t0 in (-1, 0, 1) for t1 in (-1, 0, 1) for t2 in (-1, 0, 1)}
    assert levels == set(range(-13, 14))
    t = np.array([[[a for a in (-1, 0, 1) for _ in range(9)]],
                  [[b for _ in range(3) for b in (-1, 0, 1) for _ in range(3)]],
                  [[c for _ in range(9) for c in (-1, 0, 1)]]], dtype=np.int8)
    t = np.concatenate([t, np.zeros((3, 1, 5), np.int8)], axis=2)          # K = 32
    cb = np.ones(27, np.float32)
    w = oracle.dequantize("bt3", t, 16, idx=np.zeros((1, 2), np.uint8), codebook=cb)
    assert sorted(w[0, :27].tolist()) == list(range(-13, 14))


def test_worked_tq_and_bt3():
    ex = load("worked_examples.json")
    tq = ex["tq_bf16"]
    t = np.array(tq["trits"], np.int8)
    s = np.array(tq["scales"], np.float16)
    w = oracle.dequantize("tq", t, tq["group"], scales=s)
    y = oracle.gemv_bf16(w, bf16_bits([tq["x"]]))
    assert y[0, 0] == tq["y"]
    b = ex["bt3_bf16"]
    t = np.zeros((3, 1, 16), np.int8)
    t[0, 0, :4], t[1, 0, :4], t[2, 0, :4] = b["trits_t0"], b["trits_t1"], b["trits_t2"]
    cb = np.zeros(27, np.float32)
    cb[5] = b["scale"]
    w = oracle.dequantize("bt3", t, 16, idx=np.array([[5]], np.uint8), codebook=cb)
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = b["x"]
    assert oracle.gemv_bf16(w, synth.f32_to_bf16_bits(x))[0, 0] == b["y"]


# --------------------------------------------------------------- bf16 GEMV
def test_gemv_bf16_vs_exact_rationals():
    g = np.random.default_rng(5)
    n, k, m = 6, 64, 3
    t = g.integers(-1, 2, size=(2, n, k)).astype(np.int8)
    s = np.abs(g.standard_normal((2, n, k // 32)) * 0.02).astype(np.float16)
    x = synth.f32_to_bf16_bits(g.standard_normal((m, k)).astype(np.float32))
    y = oracle.gemv_bf16(oracle.dequantize("tq", t, 32, scales=s), x)
    xf = synth.bf16_bits_to_f32(x)
    for a in range(m):
        for r in range(n):
            ref = sum(Fraction(float(s[p, r, c // 32])) * int(t[p, r, c]) * Fraction(float(xf[a, c]))
                      for p in range(2) for c in range(k))
            assert abs(Fraction(y[a, r]) - ref) <= abs(ref) * Fraction(1, 10 ** 13) + Fraction(1, 10 ** 300)


# ---------------------------------------------------------- int8 paths
def test_bitnet_int8_worked():
    ex = load("worked_examples.json")["bitnet_int8"]
    t = np.array(ex["trits"], np.int8)[None]
    y = oracle.gemv_bitnet_int8(t, np.array([ex["xq"]], np.int8), np.array([ex["s_x"]], np.float32), ex["s_w"])
    assert y[0].tolist() == ex["y"]


def _bitnet_fraction(t_row, xq, sx, sw):
    acc = sum(int(a) * int(b) for a, b in zip(t_row, xq))
    return rn_f32(rn_f32(Fraction(acc) * f32(sw)) * f32(sx))


def test_bitnet_int8_exhaustive_small_patterns():
    # every trit pattern of length 6 (729 rows) against several activations
    k = 6
    pats = np.array(np.meshgrid(*[[-1, 0, 1]] * k, indexing="ij")).reshape(k, -1).T.astype(np.int8)
    g = np.random.default_rng(9)
    xq = g.integers(-127, 128, size=(4, k)).astype(np.int8)
    sx = np.array([0.013, 1.0 / 127, 0.77, 3.5e-3], np.float32)
    y = oracle.gemv_bitnet_int8(pats[None], xq, sx, 0.02)
    for a in range(4):
        for r in range(len(pats)):
            assert Fraction(float(y[a, r])) == _bitnet_fraction(pats[r], xq[a], sx[a], 0.02)


def test_bitnet_int8_random_rectangular():
    g = np.random.default_rng(21)
    n, k, m = 7, 131, 2
    t = synth.draw_trits(g, (1, n, k))
    xq = g.integers(-127, 128, size=(m, k)).astype(np.int8)
    sx = np.array([0.031, 0.0007], np.float32)
    y = oracle.gemv_bitnet_int8(t, xq, sx, 0.02)
    for a in range(m):
        for r in range(n):
            assert Fraction(float(y[a, r])) == _bitnet_fraction(t[0, r], xq[a], sx[a], 0.02)


def _tq_fraction(t, s, grp, xq_row, sx):
    P, _, k = t.shape
    out = []
    for r in range(t.shape[1]):
        tot = Fraction(0)
        for p in range(P):
            for G in range(k // grp):
                S = sum(int(t[p, r, c]) * int(xq_row[c]) for c in range(G * grp, (G + 1) * grp))
                tot += Fraction(float(s[p, r, G])) * S
        out.append(rn_f32(rn_f32(tot) * f32(sx)))
    return out


def test_tq_int8_vs_exact_rationals():
    g = np.random.default_rng(31)
    for P, grp, k in ((2, 32, 96), (3, 16, 64), (1, 64, 64), (4, 32, 64)):
        n = 5
        t = synth.draw_trits(g, (P, n, k))
        s = synth.draw_tq_scales(g, P, n, k // grp)
        s[0, 0, 0] = np.float16(6e-8)          # an fp16 subnormal scale
        s[-1, 1, 0] = -s[-1, 1, 0]            # a negative scale
        xq = g.integers(-127, 128, size=(2, k)).astype(np.int8)
        sx = np.array([0.021, 0.9], np.float32)
        y = oracle.gemv_tq_int8(t, s, grp, xq, sx)
        for a in range(2):
            ref = _tq_fraction(t, s, grp, xq[a], sx[a])
            assert [Fraction(float(v)) for v in y[a]] == ref


def test_tq_int8_exhaustive_patterns_two_planes():
    k = 4
    pats = np.array(np.meshgrid(*[[-1, 0, 1]] * k, indexing="ij")).reshape(k, -1).T.astype(np.int8)
    n = len(pats)
    t = np.stack([pats, pats[::-1]])                       # plane 1 reversed order
    s = np.empty((2, n, 2), np.float16)
    s[0] = np.float16(0.0199)
    s[1] = np.float16(0.00221)
    s[1, :, 1] = np.float16(-0.0007)
    xq = np.array([[100, -7, 33, -127]], np.int8)
    y = oracle.gemv_tq_int8(t, s, 2, xq, np.array([0.0123], np.float32))
    ref = _tq_fraction(t, s, 2, xq[0], 0.0123)
    assert [Fraction(float(v)) for v in y[0]] == ref


# ----------------------------------------------------------- invariants
def test_invariants_linearity_sign_columns():
    g = np.random.default_rng(41)
    P, n, k, grp = 3, 9, 128, 32
    t = synth.draw_trits(g, (P, n, k))
    s = synth.draw_tq_scales(g, P, n, k // grp)
    x = synth.f32_to_bf16_bits(g.standard_normal((2, k)).astype(np.float32))
    y = oracle.gemv_bf16(oracle.dequantize("tq", t, grp, scales=s), x)
    y_sum = sum(oracle.gemv_bf16(oracle.dequantize("tq", t[p:p + 1], grp, scales=s[p:p + 1]), x) for p in range(P))
    assert np.allclose(y, y_sum, rtol=1e-12, atol=1e-14)
    y_neg = oracle.gemv_bf16(oracle.dequantize("tq", -t, grp, scales=s), x)
    assert np.array_equal(y_neg, -y)
    # x = e_i returns column i of W
    w = oracle.dequantize("tq", t, grp, scales=s)
    e = np.zeros((1, k), np.float32)
    e[0, 77] = 1.0
    assert np.array_equal(oracle.gemv_bf16(w, synth.f32_to_bf16_bits(e))[0], w[:, 77])
    # int8 path: exact linearity over planes in the integer domain, and sign flip
    xq, sx = oracle.quantize_act(x)
    yi = oracle.gemv_tq_int8(t, s, grp, xq, sx)
    yi_neg = oracle.gemv_tq_int8(-t, s, grp, xq, sx)
    assert np.array_equal(yi_neg, -yi)
    assert not oracle.gemv_tq_int8(np.zeros_like(t), s, grp, xq, sx).any()


def test_tq_single_plane_constant_scale_is_bitnet():
    g = np.random.default_rng(51)
    n, k = 11, 256
    t = synth.draw_trits(g, (1, n, k))
    s16 = np.float16(0.02)
    s = np.full((1, n, 2), s16, np.float16)
    x = synth.f32_to_bf16_bits(g.standard_normal((3, k)).astype(np.float32))
    xq, sx = oracle.quantize_act(x)
    a = oracle.gemv_tq_int8(t, s, 128, xq, sx)
    b = oracle.gemv_bitnet_int8(t, xq, sx, float(s16))
    assert np.array_equal(a, b)
    wa = oracle.dequantize("tq", t, 128, scales=s)
    wb = oracle.dequantize("bitnet", t, tensor_scale=float(s16))
    assert np.array_equal(wa, wb)


def test_bt3_reduces_to_one_plane():
    g = np.random.default_rng(61)
    n, k = 4, 64
    t = synth.draw_trits(g, (3, n, k))
    t[1:] = 0
    idx = g.integers(0, 27, size=(n, k // 16)).astype(np.uint8)
    cb = synth.codebook27()
    w = oracle.dequantize("bt3", t, 16, idx=idx, codebook=cb)
    sc = cb[idx].astype(np.float64)
    assert np.array_equal(w, np.repeat(sc, 16, axis=1) * t[0])


# ------------------------------------------------------------ bf16 rounding
def _rn_bf16(fr: Fraction) -> Fraction:
    """Nearest bf16 value of an exact rational (8 significant bits, ties to even, fp32 exponent range)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 7)
    q = a / quantum
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def test_round_bf16_vs_exact_rationals_and_ties():
    g = np.random.default_rng(71)
    v = (g.standard_normal(400) * 10.0 ** g.uniform(-30, 30, 400)).astype(np.float32)
    # exact ties between two bf16 neighbours: 1 + 2^-8 (to even: 1), 1 + 3 * 2^-8 (to even: 1 + 2^-6)
    ties = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2.0 ** -126 * (1 + 2 ** -8)], np.float32)
    v = np.concatenate([v, ties, np.float32([0.0, -0.0, 1.0, 3.0e38])])
    got = oracle.round_bf16(v)
    for a, b in zip(v, got):
        assert Fraction(float(b)) == _rn_bf16(Fraction(float(a))), a
    assert got[400] == 1.0 and got[401] == 1 + 2 ** -6 and got[402] == -1.0


def test_round_bf16_matches_torch_cast():
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(72)
    v = (g.standard_normal(5000) * 10.0 ** g.uniform(-35, 35, 5000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(v), ref)


# ------------------------------------------- balanced ternary of depth d
def _all_tuples(d):
    """Every trit tuple of depth d as planes [d][1][3^d] (t_j of tuple i is base-3 digit j of i, minus 1)."""
    i = np.arange(3 ** d)
    return np.stack([((i // 3 ** j) % 3 - 1) for j in range(d)])[:, None, :].astype(np.int8)


@pytest.mark.parametrize("d", [2, 3, 4])
def test_bt_levels_are_a_bijection_onto_the_balanced_range(d):
    # 3^d tuples -> 3^d distinct integer levels -(3^d - 1)/2 .. (3^d - 1)/2 (balanced ternary)
    t = _all_tuples(d)
    k = -(-3 ** d // 16) * 16
    t = np.concatenate([t, np.zeros((d, 1, k - 3 ** d), np.int8)], axis=2)
    w = oracle.dequantize("bt3", t, 16, idx=np.zeros((1, k // 16), np.uint8), codebook=np.ones(27, np.float32))
    half = (3 ** d - 1) // 2
    assert sorted(w[0, :3 ** d].astype(int).tolist()) == list(range(-half, half + 1))


@pytest.mark.parametrize("d", [2, 4])
def test_bt_depth_brute_force_loops(d):
    g = np.random.default_rng(80 + d)
    n, k = 3, 48
    t = g.integers(-1, 2, size=(d, n, k)).astype(np.int8)
    idx = g.integers(0, 27, size=(n, k // 16)).astype(np.uint8)
    cb = synth.codebook27()
    w = oracle.dequantize("bt3", t, 16, idx=idx, codebook=cb)
    for r in range(n):
        for c in range(k):
            lvl = 0
            for j in range(d):            # Horner from the most significant trit
                lvl = 3 * lvl + int(t[d - 1 - j, r, c])
            assert Fraction(w[r, c]) == Fraction(float(cb[idx[r, c // 16]])) * lvl


def test_bt_depths_nest():
    # a zero top trit reduces depth d + 1 to depth d
    g = np.random.default_rng(90)
    n, k = 4, 32
    t = synth.draw_trits(g, (4, n, k))
    idx = g.integers(0, 27, size=(n, k // 16)).astype(np.uint8)
    cb = synth.codebook27()
    for d in (2, 3):
        top = t[:d + 1].copy()
        top[d] = 0
        assert np.array_equal(oracle.dequantize("bt3", top, 16, idx=idx, codebook=cb),
                              oracle.dequantize("bt3", t[:d], 16, idx=idx, codebook=cb))


def test_bt_bpw_steps_by_one_trit_from_the_printed_d3():
    printed = load("bpw_pages.json")["bt3"]
    b3 = oracle.bits_per_weight("bt3", 3)
    assert round(b3, printed["digits"]) == pytest.approx(printed["printed"])
    # each level of depth adds one trit (log2 3 bits) per weight; the codebook index is unchanged
    assert oracle.bits_per_weight("bt3", 4) - b3 == pytest.approx(math.log2(3))
    assert b3 - oracle.bits_per_weight("bt3", 2) == pytest.approx(math.log2(3))


def test_quantize_act_tiny_token():
    # absmax below 127 / FLT_MAX: 127 / a overflows to +inf, so every non-zero value
    # saturates to +-127, zeros stay 0, and sx = fl32(a / 127) is exact rational rounding
    a = np.float32(2.0 ** -126)                       # smallest normal, also a bf16 value
    x = bf16_bits([[a, 0.0, -a / 4, a / 2 ** 6]])    # the last two are bf16 subnormals
    xq, sx = oracle.quantize_act(x)
    assert xq[0].tolist() == [127, 0, -127, 127]
    assert Fraction(float(sx[0])) == rn_f32(Fraction(float(a)) / 127)
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(127.0) / a)        # the case this pins: inv overflows


def test_bitnet_workload_shapes_follow_the_page():
    # the BitNet b1.58-2B layer set's seven projections, as the page's architecture fixes them
    a = load("architecture_pages.json")["bitnet_2b"]
    h, q, kv, ffn = a["hidden"], a["q_heads"] * a["head_dim"], a["kv_heads"] * a["head_dim"], a["ffn"]
    want = {"q_proj": (q, h), "k_proj": (kv, h), "v_proj": (kv, h), "o_proj": (h, q),
            "gate_proj": (ffn, h), "up_proj": (ffn, h), "down_proj": (h, ffn)}
    assert {name: (n, k) for name, n, k in synth.BITNET_2B_SHAPES} == want
    assert synth.BITNET_2B_LAYERS == a["layers"]
