"""Pins for the decode-layer oracle (oracle/decode.py), independent of its code (CPU only).

Exact rational arithmetic for the RMSNorm factor, an independent complex-number
form of the rotation and the relative-position property of RoPE, closed cases
of attention (one position, equal keys, the GQA head map, a loop of math.exp),
torch's own bf16 cast, and properties of the layer composition that a dropped
or misplaced step would break (residual paths, squared ReLU, the sub-norm
before o_proj, power-of-two gains).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import decode as dec
from packed_ternary_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_layer_facts_match_pages():
    g = json.load(open(os.path.join(GOLDEN, "architecture_pages.json")))
    assert dec.ROPE_THETA == g["bitnet_2b_layer"]["rope_theta"]
    a = g["bitnet_2b"]
    shapes = dict((nm, (n, k)) for nm, n, k in synth.BITNET_2B_SHAPES)
    assert shapes["q_proj"] == (a["q_heads"] * a["head_dim"], a["hidden"])
    assert shapes["k_proj"] == (a["kv_heads"] * a["head_dim"], a["hidden"])
    assert shapes["down_proj"] == (a["hidden"], a["ffn"])


# ------------------------------------------------------------- RMSNorm
def _exact_inv_rounds_to(x, r32, eps):
    """r32 is the fp32 value nearest to 1/sqrt(A), A = mean(x^2) + eps, decided in exact
    rationals: r lies between the midpoints m- < r < m+ of r32 and its neighbours iff
    m+^2 A > 1 > m-^2 A."""
    A = sum(Fraction(float(v)) ** 2 for v in x) / len(x) + Fraction(eps)
    up = Fraction(float(np.nextafter(r32, np.float32(np.inf))))
    dn = Fraction(float(np.nextafter(r32, np.float32(0))))
    c = Fraction(float(r32))
    m_hi, m_lo = (c + up) / 2, (c + dn) / 2
    return m_hi * m_hi * A > 1 > m_lo * m_lo * A


@pytest.mark.parametrize("seed", range(12))
def test_rmsnorm_inv_correctly_rounded(seed):
    g = np.random.default_rng(seed)
    k = int(g.integers(1, 70))
    x = (g.standard_normal(k) * 10.0 ** g.uniform(-3, 3)).astype(np.float32)
    for eps in (dec.RMS_EPS, 0.0):
        r = dec.rmsnorm_inv(x, eps)
        assert r.dtype == np.float32 and _exact_inv_rounds_to(x, r, eps)


def test_rmsnorm_closed_forms():
    x = np.full(64, 3.0, np.float32)
    y = dec.rmsnorm(x, np.ones(64, np.float32), 0.0)
    assert np.all(y == np.float32(1.0))                    # 3 * fl(1/3), then * 1
    g = np.arange(64, dtype=np.float32)
    y = dec.rmsnorm(np.full(64, -2.0, np.float32), g, 0.0)
    assert np.array_equal(y, (-g).astype(np.float32))      # x / rms = -1 exactly, times g


def test_quantize_f32_reduces_to_bf16_rule():
    xb = synth.draw_x_bf16(5, 3, 333)
    xb[1] = 0
    qa, sa = oracle.quantize_act(xb)
    qf, sf = dec.quantize_f32(synth.bf16_bits_to_f32(xb)[0])
    assert np.array_equal(qf[0], qa[0]) and sf[0] == sa[0]
    for r in range(3):
        qf, sf = dec.quantize_f32(synth.bf16_bits_to_f32(xb)[r])
        assert np.array_equal(qf[0], qa[r]) and sf[0] == sa[r]


# ---------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    c, s = dec.rope_cos_sin(0, 128)
    assert np.all(c == 1) and np.all(s == 0)
    v = np.random.default_rng(0).standard_normal(128).astype(np.float32)
    assert np.array_equal(dec.rope(v, c, s), v)


def test_rope_matches_complex_rotation():
    # (x_i + j x_{i+64}) e^{j phi_i}: an independent form of rotate_half
    g = np.random.default_rng(1)
    for pos in (1, 17, 1023, 4095):
        c, s = dec.rope_cos_sin(pos, 128)
        v = g.standard_normal(128).astype(np.float32)
        z = (v[:64].astype(np.float64) + 1j * v[64:]) * (c.astype(np.float64) + 1j * s)
        out = dec.rope(v, c, s)
        assert np.allclose(out[:64], z.real, rtol=0, atol=1e-6 * np.abs(v).max())
        assert np.allclose(out[64:], z.imag, rtol=0, atol=1e-6 * np.abs(v).max())
        # the angles: cos^2 + sin^2 = 1 and the first frequency is pos radians
        assert np.allclose(c.astype(np.float64) ** 2 + s.astype(np.float64) ** 2, 1.0, atol=1e-6)
        assert c[0] == np.float32(math.cos(pos)) and s[0] == np.float32(math.sin(pos))


def test_rope_relative_position():
    # <rope(q, m), rope(k, n)> depends on m - n only (the frequencies scale with position)
    g = np.random.default_rng(2)
    q = g.standard_normal(128).astype(np.float32)
    k = g.standard_normal(128).astype(np.float32)

    def dot(m, n):
        return float(np.dot(dec.rope(q, *dec.rope_cos_sin(m)).astype(np.float64),
                            dec.rope(k, *dec.rope_cos_sin(n)).astype(np.float64)))
    for m, n, sft in ((5, 2, 7), (100, 3, 900), (0, 40, 1000)):
        assert dot(m, n) == pytest.approx(dot(m + sft, n + sft), abs=2e-4)
    assert dot(9, 2) != pytest.approx(dot(2, 9), abs=1e-3)  # not symmetric in general


def test_bf16_round_matches_torch():
    torch = pytest.importorskip("torch")
    v = np.random.default_rng(3).standard_normal(4096).astype(np.float32)
    v[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130]  # ties and a subnormal
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(dec.bf16_round(v), want)


# ----------------------------------------------------------- attention
def _bf(v):
    return dec.bf16_round(np.asarray(v, np.float32))


def test_attention_one_position_returns_value():
    g = np.random.default_rng(4)
    q = g.standard_normal((8, 16)).astype(np.float32)
    kc = _bf(g.standard_normal((2, 5, 16)))
    vc = _bf(g.standard_normal((2, 5, 16)))
    out = dec.attention_gqa(q, kc, vc, 1)
    for h in range(8):
        want = synth.bf16_bits_to_f32(vc[h // 4, 0])
        assert np.array_equal(out[h], want)


def test_attention_gqa_head_map_and_equal_keys():
    # equal keys: the output is the mean of the values; KV head j's values are the constant j + 1
    q = np.random.default_rng(5).standard_normal((20, 128)).astype(np.float32)
    kc = _bf(np.ones((5, 7, 128)))
    vc = np.stack([_bf(np.full((7, 128), j + 1.0)) for j in range(5)])
    out = dec.attention_gqa(q, kc, vc, 7)
    for h in range(20):
        assert np.all(out[h] == np.float32(h // 4 + 1))


def test_attention_against_explicit_loop():
    g = np.random.default_rng(6)
    H, KVH, d, n = 4, 2, 16, 9
    q = g.standard_normal((H, d)).astype(np.float32)
    kc = _bf(g.standard_normal((KVH, n + 3, d)) * 2)
    vc = _bf(g.standard_normal((KVH, n + 3, d)))
    out = dec.attention_gqa(q, kc, vc, n)
    kf, vf = synth.bf16_bits_to_f32(kc), synth.bf16_bits_to_f32(vc)
    for h in range(H):
        j = h // (H // KVH)
        sc = [sum(float(q[h, i]) * float(kf[j, t, i]) for i in range(d)) / math.sqrt(d) for t in range(n)]
        w = [math.exp(x - max(sc)) for x in sc]
        for i in range(d):
            ref = sum(w[t] * float(vf[j, t, i]) for t in range(n)) / sum(w)
            assert abs(float(out[h, i]) - ref) <= 1e-6 * max(1.0, abs(ref))


# ------------------------------------------------------ layer composition
D, F, H, KVH, HD = 64, 128, 4, 2, 16


def tiny_layer(seed, zero=()):
    shapes = [(H * HD, D), (KVH * HD, D), (KVH * HD, D), (D, H * HD), (F, D), (F, D), (D, F)]
    names = ["q", "k", "v", "o", "gate", "up", "down"]
    lw = []
    for i, (n, k) in enumerate(shapes):
        lay = synth.bitnet_layer(n, k, seed * 10 + i, 0.05)
        t = lay.trits * 0 if names[i] in zero else lay.trits
        lw.append((t, lay.tensor_scale))
    g = np.random.default_rng(seed)
    gains = [(1 + 0.1 * g.standard_normal(n)).astype(np.float32) for n in (D, D, D, F)]
    return lw, gains


def tiny_state(seed, pos=6, max_pos=8):
    g = np.random.default_rng(seed + 100)
    h = g.standard_normal(D).astype(np.float32)
    kc = _bf(g.standard_normal((KVH, max_pos, HD)))
    vc = _bf(g.standard_normal((KVH, max_pos, HD)))
    return h, kc, vc, dec.rope_cos_sin(pos, HD)


def test_layer_residual_paths():
    lw, gains = tiny_layer(1, zero=("o", "down"))
    h, kc, vc, cs = tiny_state(1)
    rec = {}
    out = dec.decode_layer(h, lw, gains, kc, vc, 6, cs, rec=rec)
    assert np.array_equal(out, h)                       # h + 0 + 0
    assert np.all(rec["o"] == 0) and np.all(rec["down"] == 0)
    lw, gains = tiny_layer(1)
    out = dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, rec=rec)
    assert np.array_equal(rec["h_attn"], (h + rec["o"]).astype(np.float32))
    assert np.array_equal(out, (rec["h_attn"] + rec["down"]).astype(np.float32))


def test_layer_squared_relu():
    # gate weights negated: relu(g)^2 and relu(-g)^2 split g^2 between them
    lw, gains = tiny_layer(2)
    h, kc, vc, cs = tiny_state(2)
    r1, r2 = {}, {}
    dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, rec=r1)
    lw2 = list(lw)
    lw2[4] = (-lw[4][0], lw[4][1])
    dec.decode_layer(h, lw2, gains, kc.copy(), vc.copy(), 6, cs, rec=r2)
    g, u = r1["gate"], r1["up"]
    assert np.array_equal(r2["gate"], -g)
    assert np.all(r1["m"] * r2["m"] == 0)
    assert np.array_equal(r1["m"] + r2["m"], ((g * g).astype(np.float32) * u).astype(np.float32))
    assert np.all(r1["m"][g <= 0] == 0) and np.all(r2["m"][g >= 0] == 0)


def test_layer_sub_norm_before_o_proj():
    # values doubled (cache and v_proj scale): the attention output doubles and the
    # sub-norm (eps = 0) removes it, so o_proj's output is unchanged
    lw, gains = tiny_layer(3)
    h, kc, vc, cs = tiny_state(3)
    r1, r2 = {}, {}
    dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, rec=r1, eps=0.0)
    lw2 = list(lw)
    lw2[2] = (lw[2][0], float(np.float32(2 * lw[2][1])))
    vc2 = dec.bf16_round(2 * synth.bf16_bits_to_f32(vc))
    dec.decode_layer(h, lw2, gains, kc.copy(), vc2, 6, cs, rec=r2, eps=0.0)
    assert np.array_equal(r2["attn"], 2 * r1["attn"])
    assert np.array_equal(r2["o"], r1["o"])


def test_layer_input_gain_power_of_two():
    # input_layernorm's gain doubled: the quantised codes are unchanged and the
    # activation scale doubles, so q, k, v double exactly
    lw, gains = tiny_layer(4)
    h, kc, vc, cs = tiny_state(4)
    r1, r2 = {}, {}
    dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, last=1, rec=r1)
    g2 = [gains[0] * 2] + gains[1:]
    dec.decode_layer(h, lw, g2, kc.copy(), vc.copy(), 6, cs, last=1, rec=r2)
    for key in ("q", "k", "v"):
        assert np.array_equal(r2[key], 2 * r1[key])


def test_layer_writes_cache_at_pos_only():
    lw, gains = tiny_layer(5)
    h, kc, vc, cs = tiny_state(5)
    k0, v0 = kc.copy(), vc.copy()
    rec = {}
    dec.decode_layer(h, lw, gains, kc, vc, 6, cs, last=2, rec=rec)
    keep = [p for p in range(8) if p != 6]
    assert np.array_equal(kc[:, keep], k0[:, keep]) and np.array_equal(vc[:, keep], v0[:, keep])
    assert np.array_equal(kc[:, 6], dec.bf16_round(rec["k_rope"].reshape(KVH, HD)))
    assert np.array_equal(vc[:, 6], dec.bf16_round(rec["v"].reshape(KVH, HD)))


def test_stage_split_composes():
    # running stages 1-2 and then 3-5 from the recorded attention equals one run
    lw, gains = tiny_layer(6)
    h, kc, vc, cs = tiny_state(6)
    rec = {}
    full = dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, rec=rec)
    part = dec.decode_layer(h, lw, gains, kc.copy(), vc.copy(), 6, cs, first=3, attn_in=rec["attn"])
    assert np.array_equal(full, part)
