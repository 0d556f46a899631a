"""Plain CPU oracle of the packed ternary-weight GEMV -- TEST INFRASTRUCTURE ONLY.

Imported only by tests, by the smoke check and by the CPU-baseline leg of the
benchmark. Nothing here is shared with the CUDA path.

What it computes, with the passage each step follows:

* ``dequantize`` -- the plain weight matrix. For the additive multi-plane
  format, W = sum over planes p of s[p, n, group(k)] * t[p, n, k]
  (sasori README, "How it works" and "K and g"); for the single-plane BitNet
  layout, W = s_w * t with one per-tensor scale (QORA-LLM-2B, "Ternary GEMV
  (No Multiplication)"); for balanced ternary of depth 3,
  W = cb[idx] * (9 t2 + 3 t1 + t0), 27 levels, group 16, 27-entry log-spaced
  codebook (Entrit Llama-3.1-8B-trit-uniform-d3 card, "Quantization details");
  depth d in general (the card's d = 3; 2 and 4 by the same positional rule):
  W = cb[idx] * sum_j 3^j t_j, 3^d levels. All exact in fp64.
* ``gemv_bf16`` -- y = W x in fp64 for bf16 activations (dequantise then
  matmul: the fake-quant reference the sasori kernel is said to reproduce,
  sasori README, "g (group-size)").
* ``quantize_act`` -- per-token absmax int8 quantisation of bf16 activations
  (the single-GEMV workload's "per-token absmax"; the pages give no rounding
  rule, so this follows the reading: fp32 arithmetic, IEEE division, round half
  to even, clamp to [-127, 127]).
* ``gemv_bitnet_int8`` -- integer sum of +-x over the row, then one multiply by
  the layer scale at the end (QORA-LLM-2B, "Ternary GEMV"), then one by the
  activation scale, both fp32 round-to-nearest.
* ``gemv_tq_int8`` -- group-scaled int8 path: the exact sum over planes and
  groups of s * (integer group sum), rounded once to fp32, times the
  activation scale.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against brute force in exact rational arithmetic, closed forms and the pages'
printed values; none is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64",
    "quantize_act",
    "dequantize",
    "gemv_bf16",
    "gemv_bitnet_int8",
    "gemv_tq_int8",
    "bits_per_weight",
    "bt3_information_bpw",
    "round_bf16",
]


# ------------------------------------------------------------------ helpers
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 numbers given as uint16 bit patterns."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns fp64 values."""
    f = np.asarray(v, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


# ------------------------------------------------------- activation quant
def quantize_act(x_bits: np.ndarray):
    """Per-token absmax int8 quantisation.

    x_bits: bf16 bits [M][K]. Returns (xq int8 [M][K], sx float32 [M]) with
      a   = max_i |x_i|                     (exact, bf16 -> fp32)
      inv = fl32(127 / a)
      xq  = clamp(rint_half_even(fl32(x_i * inv)), -127, 127)
      sx  = fl32(a / 127)
    and xq = 0, sx = 0 for an all-zero token. When a is so small that 127 / a
    overflows fp32 (a < 127 / FLT_MAX, about 3.7e-37), inv is +inf: non-zero x
    give +-inf, clamped to +-127, and x = 0 gives 0 (the product 0 * inf is
    taken as 0; the pages say nothing about this case).
    """
    x = (np.asarray(x_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    x = np.atleast_2d(x)
    m = x.shape[0]
    xq = np.zeros(x.shape, dtype=np.int8)
    sx = np.zeros(m, dtype=np.float32)
    for r in range(m):
        a = np.float32(np.max(np.abs(x[r]))) if x.shape[1] else np.float32(0)
        if a == 0:
            continue
        with np.errstate(over="ignore", invalid="ignore"):
            inv = np.float32(np.float32(127.0) / a)
            v = (x[r] * inv).astype(np.float32)      # one fp32 multiply each
        v = np.where(x[r] == 0, np.float32(0), v)     # 0 * inf (inv overflowed) counts as 0
        q = np.clip(np.rint(v), -127, 127)            # numpy rint: half to even
        xq[r] = q.astype(np.int8)
        sx[r] = np.float32(a / np.float32(127.0))
    return xq, sx


# ------------------------------------------------------------- dequantise
def dequantize(fmt: str, trits: np.ndarray, group: int = 0, tensor_scale: float = 0.0,
               scales: np.ndarray | None = None, idx: np.ndarray | None = None,
               codebook: np.ndarray | None = None) -> np.ndarray:
    """Plain weight matrix W [N][K] in fp64 from the logical format inputs."""
    t = np.asarray(trits, dtype=np.int64)
    _, n, k = t.shape
    if fmt == "bitnet":
        return float(np.float32(tensor_scale)) * t[0].astype(np.float64)
    if fmt == "tq":
        s = np.asarray(scales, dtype=np.float16).astype(np.float64)   # [P][N][K/g]
        w = np.zeros((n, k), dtype=np.float64)
        for p in range(t.shape[0]):
            w += np.repeat(s[p], group, axis=1) * t[p]
        return w
    if fmt == "bt3":
        # depth d = number of trit planes: level = sum_j 3^j t_j (d = 3: -13 .. 13)
        cb = np.asarray(codebook, dtype=np.float32).astype(np.float64)
        level = np.zeros((n, k), dtype=np.int64)
        for j in range(t.shape[0]):
            level += 3 ** j * t[j]
        sc = cb[np.asarray(idx, dtype=np.int64)]           # [N][K/16]
        return np.repeat(sc, 16, axis=1) * level
    raise ValueError(fmt)


def gemv_bf16(w: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """y[m][n] = sum_k W[n][k] x[m][k] in fp64 (x given as bf16 bits)."""
    x = np.atleast_2d(bf16_to_f64(x_bits))
    return x @ np.asarray(w, dtype=np.float64).T


# ----------------------------------------------------------- int8 paths
def gemv_bitnet_int8(trits: np.ndarray, xq: np.ndarray, sx: np.ndarray, tensor_scale: float) -> np.ndarray:
    """y = fl32(fl32(float(acc) * s_w) * s_x), acc = sum_k t[n][k] * xq[m][k] exactly."""
    t = np.asarray(trits, dtype=np.int64).reshape(trits.shape[-2], trits.shape[-1])
    q = np.atleast_2d(np.asarray(xq, dtype=np.int64))
    acc = q @ t.T                                               # exact, [M][N]
    assert np.all(np.abs(acc) < 2 ** 24)                        # so float(acc) is exact
    y = (acc.astype(np.float32) * np.float32(tensor_scale)).astype(np.float32)
    return (y * np.asarray(sx, dtype=np.float32)[:, None]).astype(np.float32)


def _fp16_as_int_pow2(s: np.ndarray):
    """Split fp16 values into (mantissa integer, exponent) with s = m * 2**e exactly."""
    bits = np.asarray(s, dtype=np.float16).view(np.uint16).astype(np.int64)
    sign = np.where(bits & 0x8000, -1, 1)
    ex = (bits >> 10) & 0x1F
    man = bits & 0x3FF
    assert np.all(ex < 31), "non-finite scale"
    m = np.where(ex > 0, man + 1024, man) * sign
    e = np.where(ex > 0, ex - 25, -24)
    return m, e


def gemv_tq_int8(trits: np.ndarray, scales: np.ndarray, group: int, xq: np.ndarray, sx: np.ndarray) -> np.ndarray:
    """y = fl32( fl32( sum_{p,grp} s[p,n,grp] * S[p,n,grp] ) * s_x ), the inner sum exact.

    S[p,n,grp] = sum_{k in grp} t[p,n,k] * xq[m,k] (integers). Each fp16 scale is
    m * 2**e with e >= -24, so every product is an integer multiple of 2**-24 and
    the total is held exactly as an int64 count of 2**-24.
    """
    t = np.asarray(trits, dtype=np.int64)
    p_, n, k = t.shape
    q = np.atleast_2d(np.asarray(xq, dtype=np.int64))
    mm = q.shape[0]
    grp = k // group
    mant, ex = _fp16_as_int_pow2(scales)                        # [P][N][G]
    total = np.zeros((mm, n), dtype=np.int64)                   # count of 2**-24
    for p in range(p_):
        tg = t[p].reshape(n, grp, group)
        qg = q.reshape(mm, grp, group)
        s_int = np.einsum("ngi,mgi->mng", tg, qg)               # exact integer group sums
        unit = mant[p] * (np.int64(1) << (ex[p] + 24))          # s / 2**-24, exact integer
        assert np.all(np.abs(unit) < 2 ** 40)
        contrib = s_int * unit[None]
        bound = np.abs(unit).sum(axis=1).max() * 127 * group    # no int64 overflow below
        assert bound < 2 ** 62
        total += contrib.sum(axis=2)
    assert np.all(np.abs(total) < 2 ** 53)                      # int64 -> fp64 exact
    y0 = total.astype(np.float64).astype(np.float32) * np.float32(2.0 ** -24)  # one RN to fp32
    return (y0 * np.asarray(sx, dtype=np.float32)[:, None]).astype(np.float32)


# ---------------------------------------------------------- bpw accounting
def bits_per_weight(fmt: str, planes: int = 1, group: int = 256) -> float:
    """Bits per weight of the formats' logical content.

    TQ{K}P: K planes of 2-bit trits plus one fp16 scale per group of g per plane
    (sasori README, "K and g" table): K * (2 + 16 / g). Balanced ternary: the
    information content at depth d = ``planes`` (see ``bt3_information_bpw``).
    """
    if fmt == "tq":
        return planes * (2.0 + 16.0 / group)
    if fmt == "bitnet":
        return 2.0
    if fmt == "bt3":
        return bt3_information_bpw(depth=planes)
    raise ValueError(fmt)


def bt3_information_bpw(depth: int = 3, group: int = 16, scale_trits: int = 3) -> float:
    """Information content per weight of balanced ternary: (d * g + scale trits) * log2(3) / g."""
    return (depth * group + scale_trits) * math.log2(3.0) / group
