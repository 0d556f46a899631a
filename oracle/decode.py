"""Plain CPU oracle of one BitNet b1.58 decode step -- TEST INFRASTRUCTURE ONLY.

Imported only by tests, by the smoke check and by the benchmark's CPU legs.
Nothing here is shared with the CUDA path.

The layer follows the QORA-LLM-2B page, "SubLN Pattern (4 norms per layer)"
and "Architecture" (hidden 2560, FFN 6912, GQA 20 query / 5 KV heads of 128,
squared ReLU, RoPE rotate_half with theta = 500,000):

    residual = h
    x = input_layernorm(h)                 RMSNorm
    q, k, v = q/k/v_proj(x)                ternary linears
    q, k = rope(q, k)
    attn = attention(q, k, v)              GQA over the KV cache
    attn = attn_sub_norm(attn)             RMSNorm
    h = residual + o_proj(attn)
    residual = h
    x = post_attention_layernorm(h)        RMSNorm
    gate = relu2(gate_proj(x)); up = up_proj(x)
    h = residual + down_proj(ffn_sub_norm(gate * up))

Each ternary linear quantises its input per token to int8 (absmax, the rule
of ``tern_oracle.quantize_act`` applied to fp32 values) and runs the exact
integer GEMV with the per-tensor scale at the end (``gemv_bitnet_int8``,
"Ternary GEMV (No Multiplication)" on the same page).

Readings where the page is silent (each stated where it is used):
* RMSNorm: y_i = fl32(fl32(x_i * r) * g_i) with r = 1 / sqrt(mean(x^2) + eps)
  computed in real arithmetic and rounded once to fp32; eps = 1e-5.
* RoPE: frequencies theta^(-2i/d), i < d/2, the angle pos * freq and its cosine
  and sine in double precision, each rounded once to fp32; the rotation of
  the pair (i, i + d/2) in fp32 with every product and sum rounded:
  out_i = x_i c - x_{i+d/2} s, out_{i+d/2} = x_{i+d/2} c + x_i s.
* KV cache: bf16 (keys after RoPE), the current position included; the
  attention itself (scores scaled by 1/sqrt(d), softmax, weighted sum of
  values) is taken in fp64 and its result rounded to fp32.
* relu2(g) = max(0, g)^2 and the product with up in fp32, each step rounded.
* Residual adds in fp32.
"""
from __future__ import annotations

import math

import numpy as np

from .tern_oracle import gemv_bitnet_int8

__all__ = [
    "RMS_EPS",
    "ROPE_THETA",
    "rmsnorm_inv",
    "rmsnorm",
    "quantize_f32",
    "ternary_linear",
    "rope_cos_sin",
    "rope",
    "bf16_round",
    "attention_gqa",
    "decode_layer",
    "decode_step",
]

RMS_EPS = 1e-5
ROPE_THETA = 500000.0
STAGES = (1, 2, 3, 4, 5)   # qkv, attention, o_proj, gate/up, down


def rmsnorm_inv(x: np.ndarray, eps: float = RMS_EPS) -> np.float32:
    """fl32(1 / sqrt(mean(x^2) + eps)) for fp32 x. Each x_i^2 is exact in fp64
    (24-bit mantissas), math.fsum gives their sum correctly rounded, and the
    remaining operations add a few fp64 roundings before the one rounding to
    fp32."""
    x = np.asarray(x, dtype=np.float32)
    s = math.fsum(float(v) * float(v) for v in x.astype(np.float64))
    return np.float32(1.0 / math.sqrt(s / x.size + eps))


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """y_i = fl32(fl32(x_i * r) * g_i), r = rmsnorm_inv(x)."""
    r = rmsnorm_inv(x, eps)
    x = np.asarray(x, dtype=np.float32)
    return ((x * r).astype(np.float32) * np.asarray(g, dtype=np.float32)).astype(np.float32)


def quantize_f32(x: np.ndarray):
    """Per-token absmax int8 quantisation of fp32 values, the rule of
    quantize_act: a = max|x|, inv = fl32(127 / a), q = clamp(rint(fl32(x * inv)),
    -127, 127) with ties to even, s = fl32(a / 127); a = 0 gives q = 0, s = 0.
    Returns (q int8 [1][K], s float32 [1])."""
    x = np.atleast_2d(np.asarray(x, dtype=np.float32))
    q = np.zeros(x.shape, dtype=np.int8)
    s = np.zeros(x.shape[0], dtype=np.float32)
    for r in range(x.shape[0]):
        a = np.float32(np.max(np.abs(x[r])))
        if a == 0:
            continue
        with np.errstate(over="ignore", invalid="ignore"):
            inv = np.float32(np.float32(127.0) / a)
            v = (x[r] * inv).astype(np.float32)
        v = np.where(x[r] == 0, np.float32(0), v)
        q[r] = np.clip(np.rint(v), -127, 127).astype(np.int8)
        s[r] = np.float32(a / np.float32(127.0))
    return q, s


def ternary_linear(trits: np.ndarray, tensor_scale: float, x: np.ndarray) -> np.ndarray:
    """A BitNet linear on fp32 input: quantise, exact integer GEMV, scales at the end. fp32 [N]."""
    q, s = quantize_f32(x)
    return gemv_bitnet_int8(trits, q, s, tensor_scale)[0]


def rope_cos_sin(pos: int, head_dim: int = 128, theta: float = ROPE_THETA):
    """cos and sin of pos * theta^(-2i/d), i < d/2, each computed in double and rounded to fp32."""
    half = head_dim // 2
    c = np.empty(half, np.float32)
    s = np.empty(half, np.float32)
    for i in range(half):
        ang = pos * theta ** (-2.0 * i / head_dim)
        c[i] = np.float32(math.cos(ang))
        s[i] = np.float32(math.sin(ang))
    return c, s


def rope(v: np.ndarray, c: np.ndarray, s: np.ndarray) -> np.ndarray:
    """rotate_half on one head (fp32 [d]): out_i = x_i c_i - x_{i+h} s_i,
    out_{i+h} = x_{i+h} c_i + x_i s_i, h = d/2, every product and sum rounded."""
    v = np.asarray(v, dtype=np.float32)
    h = v.size // 2
    a, b = v[:h], v[h:]
    out = np.empty_like(v)
    out[:h] = ((a * c).astype(np.float32) - (b * s).astype(np.float32)).astype(np.float32)
    out[h:] = ((b * c).astype(np.float32) + (a * s).astype(np.float32)).astype(np.float32)
    return out


def bf16_round(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (nearest, ties to even), returned as bf16 bit patterns (uint16)."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def attention_gqa(q: np.ndarray, kc: np.ndarray, vc: np.ndarray, n_pos: int) -> np.ndarray:
    """GQA attention of one token. q fp32 [H][d] (after RoPE); kc, vc bf16 bits
    [KVH][>= n_pos][d], positions 0 .. n_pos-1 attended (the current one
    included). Query head h reads KV head h // (H / KVH). fp64, result rounded
    to fp32 [H][d]."""
    H, d = q.shape
    kvh = kc.shape[0]
    rep = H // kvh
    out = np.empty((H, d), np.float32)
    for h in range(H):
        j = h // rep
        k = _bf16_to_f64(kc[j, :n_pos])
        v = _bf16_to_f64(vc[j, :n_pos])
        sc = k @ q[h].astype(np.float64) / math.sqrt(d)
        sc -= sc.max()
        p = np.exp(sc)
        p /= p.sum()
        out[h] = (p @ v).astype(np.float32)
    return out


def decode_layer(h, lw, gains, kc, vc, pos, cos_sin, first=1, last=5, attn_in=None, rec=None,
                 eps: float = RMS_EPS):
    """One decode layer on fp32 h [D], stages first..last (1 qkv, 2 attention,
    3 o_proj, 4 gate/up, 5 down; starting at 3 takes attn_in as the attention
    output). lw: seven (trits [1][N][K], tensor_scale) in the order q, k, v, o,
    gate, up, down. gains: four fp32 vectors (input, attn_sub, post_attention,
    ffn_sub). kc, vc: this layer's bf16 caches [KVH][max_pos][d], updated in
    place at `pos`. rec: optional dict that receives the intermediate values.
    Returns h after the last stage run (its residual add included)."""
    h = np.asarray(h, dtype=np.float32).copy()
    rec = {} if rec is None else rec
    (wq, sq), (wk, sk), (wv, sv), (wo, so), (wg, sg), (wu, su), (wd, sd) = lw
    kvh, _, d = kc.shape
    H = wq.shape[1] // d
    attn = None if attn_in is None else np.asarray(attn_in, dtype=np.float32)
    q = k = v = gate = up = None
    for st in range(first, last + 1):
        if st == 1:
            x = rmsnorm(h, gains[0], eps)
            q = ternary_linear(wq, sq, x)
            k = ternary_linear(wk, sk, x)
            v = ternary_linear(wv, sv, x)
            rec.update(q=q, k=k, v=v)
        elif st == 2:
            c, s = cos_sin
            qr = np.stack([rope(q[i * d:(i + 1) * d], c, s) for i in range(H)])
            kr = np.stack([rope(k[j * d:(j + 1) * d], c, s) for j in range(kvh)])
            kc[:, pos] = bf16_round(kr)
            vc[:, pos] = bf16_round(v.reshape(kvh, d))
            attn = attention_gqa(qr, kc, vc, pos + 1).reshape(-1)
            rec.update(q_rope=qr.reshape(-1), k_rope=kr.reshape(-1), attn=attn)
        elif st == 3:
            a = rmsnorm(attn, gains[1], eps)
            o = ternary_linear(wo, so, a)
            h = (h + o).astype(np.float32)
            rec.update(o=o, h_attn=h.copy())
        elif st == 4:
            x = rmsnorm(h, gains[2], eps)
            gate = ternary_linear(wg, sg, x)
            up = ternary_linear(wu, su, x)
            rec.update(gate=gate, up=up)
        else:
            r = np.maximum(gate, np.float32(0)).astype(np.float32)
            m = ((r * r).astype(np.float32) * up).astype(np.float32)
            dn = ternary_linear(wd, sd, rmsnorm(m, gains[3], eps))
            h = (h + dn).astype(np.float32)
            rec.update(m=m, down=dn, h_out=h.copy())
    return h


def decode_step(h0, layers, gains, kcache, vcache, pos, cos_sin, eps: float = RMS_EPS, recs=None):
    """All layers in order on the token at `pos`; kcache/vcache [L][KVH][max_pos][d] updated in place."""
    h = np.asarray(h0, dtype=np.float32)
    for li, lw in enumerate(layers):
        rec = {} if recs is None else recs.setdefault(li, {})
        h = decode_layer(h, lw, gains[li], kcache[li], vcache[li], pos, cos_sin, rec=rec, eps=eps)
    return h
