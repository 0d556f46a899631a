"""Plain decoder of the packed buffer format -- TEST INFRASTRUCTURE ONLY.

Written from the format's definition (below), independently of the product's
packer and kernels. It turns a packed buffer back into the logical inputs the
oracle consumes, so that tests can check the packer byte for byte and the
benchmark's CPU baseline can start from the same bytes the GPU reads.

Format (all little-endian):

* 256-byte header: u32 magic 0x4E524554, u32 version 2, u32 fmt (1 BitNet,
  2 TQ, 3 balanced ternary), u32 N, u32 K, u32 planes (balanced ternary: the
  depth d), u32 group,
  f32 tensor scale, u32 row tiles ceil(N/32), u32 columns, u64 trit offset,
  u64 trit bytes, u64 scale offset, u64 scale bytes; at byte 72 u32 "scale
  digits": TQ, the number of base-128 digits of the largest |s| / 2^-24 over
  all scales (at least 1); BitNet 1; balanced ternary 0. The 27 fp32 codebook
  entries at byte 128 (balanced ternary only). Everything else is zero.
* 2-bit planes (BitNet, TQ): a chunk is 16 bytes holding 64 consecutive k of
  one row of one plane, as four u32 words; word w holds k = 64c + 16w + j for
  j = 0..15 with the code of trit j in bits 8*(j%4) + 2*(j//4) .. +1. Codes:
  00 -> 0, 01 -> +1, 10 -> -1 (11 is invalid). Chunk (row tile T, column c,
  plane p, row r) lies at trit_offset + ((T*cols + c)*P + p)*512 + 16*r, for
  row n = 32T + r. Padding rows and columns hold code 00.
* TQ scales: fp16 scale of (T, group G, plane p, row r) at
  scale_offset + ((T*groups + G)*P + p)*64 + 2*r.
* Balanced ternary of depth d (2, 3 or 4; the Entrit card's d = 3): a column
  is 80 consecutive k of a 32-row tile, 512*d + 96 bytes at
  trit_offset + (T*cols + c)*(512*d + 96). Its first 512*d bytes hold, per
  row r, 16 byte tuples of d bytes: byte b (0..d-1) of tuple i at
  b*512 + 16*r + i. Every byte holds five base-3 digits u = t + 1 (first
  digit least significant); the 5d digits of tuple i, byte 0 first, are the
  trits t0 .. t(d-1) (weights 1, 3, 9, 27) of k = 80c + i, then of
  k = 80c + 16 + i, ..., then of k = 80c + 64 + i (weight j of the tuple,
  j = 0..4, is k = 80c + 16j + i; its trit p is digit d*j + p). The last 96
  bytes hold the scale indices of the column's five groups of 16 as one
  triple per row: byte b (0..2) of row r at 512*d + 32*b + r, five base-3
  digits each; digit 3j + q of the triple (byte 0 first) is base-3 digit q
  of the index of group 5c + j. Padding trits are 0 (digit 1), padding
  indices 0.
"""
from __future__ import annotations

import struct

import numpy as np

__all__ = ["parse_header", "unpack", "HEADER_BYTES"]

HEADER_BYTES = 256
MAGIC = 0x4E524554
FMT_NAMES = {1: "bitnet", 2: "tq", 3: "bt3"}


def parse_header(buf: np.ndarray) -> dict:
    b = bytes(np.asarray(buf, dtype=np.uint8)[:HEADER_BYTES])
    magic, version, fmt, n, k, planes, group = struct.unpack_from("<7I", b, 0)
    (tscale,) = struct.unpack_from("<f", b, 28)
    row_tiles, cols = struct.unpack_from("<2I", b, 32)
    toff, tbytes, soff, sbytes = struct.unpack_from("<4Q", b, 40)
    (digits,) = struct.unpack_from("<I", b, 72)
    cb = np.frombuffer(b, dtype="<f4", count=27, offset=128).copy()
    if magic != MAGIC or version != 2:
        raise ValueError("not a packed ternary buffer")
    return dict(fmt=FMT_NAMES[fmt], n=n, k=k, planes=planes, group=group, tensor_scale=tscale,
                row_tiles=row_tiles, cols=cols, trit_offset=toff, trit_bytes=tbytes,
                scale_offset=soff, scale_bytes=sbytes, scale_digits=digits, codebook=cb)


def _decode_2bit(code: np.ndarray) -> np.ndarray:
    if np.any(code == 3):
        raise ValueError("invalid 2-bit code 11")
    lut = np.array([0, 1, -1], dtype=np.int8)
    return lut[code]


def _unpack_2bit(buf: np.ndarray, h: dict) -> np.ndarray:
    n, k, P, T, C = h["n"], h["k"], h["planes"], h["row_tiles"], h["cols"]
    raw = np.asarray(buf, dtype=np.uint8)[h["trit_offset"]:h["trit_offset"] + h["trit_bytes"]]
    words = raw.view("<u4").reshape(T, C, P, 32, 4)              # [T][c][p][r][w]
    j = np.arange(16)
    shift = (8 * (j % 4) + 2 * (j // 4)).astype(np.uint32)        # bit of trit j in a word
    code = (words[..., None] >> shift) & 3                        # [T][c][p][r][w][j]
    t = _decode_2bit(code.astype(np.int64))
    # k = 64c + 16w + j ; n = 32T + r
    t = t.transpose(2, 0, 3, 1, 4, 5).reshape(P, T * 32, C * 64)
    return t[:, :n, :k].copy()


def _unpack_tq_scales(buf: np.ndarray, h: dict) -> np.ndarray:
    n, k, P, T, g = h["n"], h["k"], h["planes"], h["row_tiles"], h["group"]
    G = k // g
    raw = np.asarray(buf, dtype=np.uint8)[h["scale_offset"]:h["scale_offset"] + h["scale_bytes"]]
    s = raw.view("<f2").reshape(T, G, P, 32)                      # [T][G][p][r]
    return s.transpose(2, 0, 3, 1).reshape(P, T * 32, G)[:, :n, :].astype(np.float16)


def _base3_digits(byte: np.ndarray) -> np.ndarray:
    """Five base-3 digits of each byte (first digit least significant)."""
    if np.any(byte > 242):
        raise ValueError("base-3 byte above 242")
    v = byte.astype(np.int64)
    out = []
    for _ in range(5):
        out.append(v % 3)
        v = v // 3
    return np.stack(out, axis=-1)


def _unpack_bt3(buf: np.ndarray, h: dict):
    n, k, T, C, d = h["n"], h["k"], h["row_tiles"], h["cols"], h["planes"]
    raw = np.asarray(buf, dtype=np.uint8)[h["trit_offset"]:h["trit_offset"] + h["trit_bytes"]]
    col = raw.reshape(T, C, 512 * d + 96)
    tup = col[:, :, :512 * d].reshape(T, C, d, 32, 16)            # [T][c][b][r][i]
    dig = _base3_digits(tup)                                      # [T][c][b][r][i][q]
    # digit s = 5b + q of the tuple; trit p of weight j is digit d*j + p
    dig = dig.transpose(0, 1, 3, 4, 2, 5).reshape(T, C, 32, 16, 5, d)  # [T][c][r][i][j][p]
    t = (dig - 1).astype(np.int8)
    # k = 80c + 16j + i
    t = t.transpose(5, 0, 2, 1, 4, 3).reshape(d, T * 32, C * 80)
    ib = col[:, :, 512 * d:].reshape(T, C, 3, 32)                 # [T][c][b][r]
    idig = _base3_digits(ib)                                      # [T][c][b][r][q]
    idig = idig.transpose(0, 1, 3, 2, 4).reshape(T, C, 32, 5, 3)  # [T][c][r][j][digit]
    idx = idig[..., 0] + 3 * idig[..., 1] + 9 * idig[..., 2]      # [T][c][r][j]
    idx = idx.transpose(0, 2, 1, 3).reshape(T * 32, C * 5)        # group = 5c + j
    return t[:, :n, :k].copy(), idx[:n, : k // 16].astype(np.uint8)


def unpack(buf: np.ndarray) -> dict:
    """Decode a packed buffer into its logical inputs (trits [P][N][K] and scales)."""
    h = parse_header(buf)
    out = dict(h)
    if h["fmt"] in ("bitnet", "tq"):
        out["trits"] = _unpack_2bit(buf, h)
        if h["fmt"] == "tq":
            out["scales"] = _unpack_tq_scales(buf, h)
    else:
        out["trits"], out["idx"] = _unpack_bt3(buf, h)
    return out
