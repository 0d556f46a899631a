"""Host-side checks of the C-ABI library (no device calls).

* every function declared in include/tern.h is exported by libtern.so;
* the packer writes the documented layout: its output decodes, with the
  oracle's independent decoder, to exactly the logical inputs, and a few bytes
  are checked against values worked out by hand from the format definition;
* packed sizes follow the closed forms; bad inputs return the documented codes.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from packed_ternary_weight_b200 import synth
from packed_ternary_weight_b200 import tern

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "tern.h")).read()
    return sorted(set(re.findall(r"^\s*(?:tern_status|const char\*)\s+(tern_\w+)\s*\(", txt, re.M)))


def test_all_declared_symbols_exported():
    names = header_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(tern.lib, n), n
        assert ctypes.cast(getattr(tern.lib, n), ctypes.c_void_p).value


def test_binding_declares_every_argument():
    # every entry point of the header has ctypes argument types in the binding, one per C
    # parameter (an undeclared size_t or pointer would be passed as a 32-bit int)
    txt = open(os.path.join(ROOT, "include", "tern.h")).read()
    for name in header_functions():
        params = re.search(r"^\s*(?:tern_status|const char\*)\s+" + name + r"\s*\(([^)]*)\)\s*;", txt,
                           re.S | re.M).group(1)
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        fn = getattr(tern.lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_status_strings():
    for c in range(8):
        assert tern.status_string(c)
    assert tern.status_string(0) == "ok"


# ------------------------------------------------------------ round trips
def roundtrip(layer):
    d, buf = tern.pack_layer(layer)
    u = oracle.unpack(buf)
    assert u["n"] == layer.n and u["k"] == layer.k and u["planes"] == layer.planes
    assert np.array_equal(u["trits"], layer.trits)
    if layer.fmt == "tq":
        assert np.array_equal(u["scales"].view(np.uint16), layer.scales.view(np.uint16))
    if layer.fmt == "bt3":
        assert np.array_equal(u["idx"], layer.idx)
        assert np.array_equal(u["codebook"], layer.codebook)
    if layer.fmt == "bitnet":
        assert u["tensor_scale"] == np.float32(layer.tensor_scale)
    return buf


@pytest.mark.parametrize("n,k", [(1, 1), (37, 100), (32, 64), (64, 1024), (511, 130)])
def test_roundtrip_bitnet(n, k):
    roundtrip(synth.bitnet_layer(n, k, seed=n * 1000 + k))


@pytest.mark.parametrize("planes", [1, 2, 3, 4])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_roundtrip_tq(planes, group):
    roundtrip(synth.tq_layer(45, 512, planes, group, seed=planes * 10 + group))


@pytest.mark.parametrize("n,k", [(1, 16), (45, 96), (32, 160), (70, 4096)])
def test_roundtrip_bt3(n, k):
    roundtrip(synth.bt3_layer(n, k, seed=n + k))


def test_no_invalid_codes_or_bytes():
    lay = synth.tq_layer(33, 256, 3, 64, seed=5)
    buf = roundtrip(lay)
    h = oracle.parse_header(buf)
    words = buf[h["trit_offset"]:h["trit_offset"] + h["trit_bytes"]]
    codes = np.unpackbits(words[:, None], axis=1, bitorder="little").reshape(-1, 2)
    assert not np.any(codes.all(axis=1))            # no 11 code
    b3 = roundtrip(synth.bt3_layer(33, 160, seed=6))
    h = oracle.parse_header(b3)
    assert b3[h["trit_offset"]:].max() <= 242


# --------------------------------------------------- hand-worked byte pins
def test_bitnet_bytes_by_hand():
    # one row, K = 64: t[5] = +1 (code 01), t[17] = -1 (code 10), t[63] = +1.
    # trit j of word w sits at bit 8*(j%4) + 2*(j//4):
    #   k=5  -> word 0, j=5  -> bit 10 (code 01 -> bit 10 set)
    #   k=17 -> word 1, j=1  -> bit 8  (code 10 -> bit 9 set)
    #   k=63 -> word 3, j=15 -> bit 30 (code 01 -> bit 30 set)
    t = np.zeros((1, 1, 64), np.int8)
    t[0, 0, 5], t[0, 0, 17], t[0, 0, 63] = 1, -1, 1
    d = tern.make_desc("bitnet", 1, 64, 1, 64, 0.5)
    buf = tern.pack(d, t)
    assert len(buf) == 256 + 512                     # one 32-row tile, one column
    words = buf[256:256 + 16].view("<u4")
    assert words.tolist() == [1 << 10, 1 << 9, 0, 1 << 30]
    assert not buf[256 + 16:].any()                  # rows 1..31 are padding
    assert oracle.unpack(buf)["trits"].tolist() == t.tolist()


def test_tq_scale_bytes_by_hand():
    # N = 33 (two 32-row tiles), K = 128, two planes, g = 64: two groups, two
    # 64-k columns. Trit stream = 2 tiles * 2 columns * 2 planes * 512 B = 4096 B,
    # so the scale stream starts at 256 + 4096 = 4352. The fp16 scale of (tile T,
    # group G, plane p, row r) sits at 4352 + ((T*2 + G)*2 + p)*64 + 2r:
    #   n = 5  (T 0, r 5),  G 0, p 0 -> 4352 + 10          1.0    = 0x3C00
    #   n = 31 (T 0, r 31), G 1, p 0 -> 4352 + 128 + 62     2^-24 = 0x0001 (subnormal)
    #   n = 32 (T 1, r 0),  G 1, p 1 -> 4352 + 7*64         0.375 = 0x3600
    #   n = 32,             G 0, p 1 -> 4352 + 5*64        -2.0   = 0xC000
    t = np.zeros((2, 33, 128), np.int8)
    sc = np.zeros((2, 33, 2), np.float16)
    sc[0, 5, 0], sc[0, 31, 1], sc[1, 32, 1], sc[1, 32, 0] = 1.0, 2.0 ** -24, 0.375, -2.0
    d = tern.make_desc("tq", 33, 128, 2, 64)
    buf = tern.pack(d, t, sc)
    h = oracle.parse_header(buf)
    assert h["scale_offset"] == 4352 and h["scale_bytes"] == 2 * 2 * 2 * 32 * 2
    u16 = lambda off: int(buf[off]) | (int(buf[off + 1]) << 8)      # noqa: E731
    expect_at = {4352 + 10: 0x3C00, 4352 + 128 + 62: 0x0001, 4352 + 7 * 64: 0x3600, 4352 + 5 * 64: 0xC000}
    for off, v in expect_at.items():
        assert u16(off) == v, (off, hex(u16(off)))
    rest = np.array(buf[4352:], np.uint8).copy()
    for off in expect_at:
        rest[off - 4352:off - 4352 + 2] = 0
    assert not rest.any()                           # every other scale (padding rows included) is zero
    assert np.array_equal(oracle.unpack(buf)["scales"].view(np.uint16), sc.view(np.uint16))


def test_bt3_bytes_by_hand():
    # one row, K = 16 (one group): t0[3] = +1 (digit 2), everything else 0
    # (digit 1). Triple i holds the trits of k = 16 j + i (j = 0..4), weight by
    # weight, five digits per byte: triple 3 starts with the digits 2, 1, 1 of
    # k = 3, so its byte 0 is 2 + 3 + 9 + 27 + 81 = 122 and every other byte is
    # 1 + 3 + 9 + 27 + 81 = 121.
    # The group's index 14 = 2 + 1*3 + 1*9: the index triple holds its digits
    # 2, 1, 1 first and 0 for the padding groups: byte 0 = 2 + 1*3 + 1*9 = 14,
    # bytes 1 and 2 = 0.
    t = np.zeros((3, 1, 16), np.int8)
    t[0, 0, 3] = 1
    idx = np.array([[14]], np.uint8)
    cb = synth.codebook27()
    d = tern.make_desc("bt3", 1, 16, 3, 16)
    buf = tern.pack(d, t, scale_idx=idx, codebook=cb)
    assert len(buf) == 256 + 1632
    col = buf[256:]
    assert col[3] == 122 and col[0] == 121 and col[15] == 121
    assert col[512] == 121 and col[1024 + 7] == 121
    assert col[1536] == 14 and col[1536 + 32] == 0 and col[1536 + 64] == 0
    assert np.array_equal(buf[128:128 + 108].view("<f4"), cb)
    u = oracle.unpack(buf)
    assert np.array_equal(u["trits"], t) and u["idx"].tolist() == [[14]]


def test_bt3_triple_order_by_hand():
    # one row, K = 32 (two groups): t1[0] = -1 and t2[16] = +1, everything else
    # 0. Triple 0 carries k = 0, 16, 32, 48, 64 (the last three are padding,
    # digits 1 1 1). Its 15 digits, weight by weight (t0, t1, t2):
    #   k = 0: 1 0 1 | k = 16: 1 1 2 | padding: 1 1 1, 1 1 1, 1 1 1
    # byte 0 = digits 1 0 1 1 1 (s = 0..4)   -> 1 + 0*3 + 1*9 + 1*27 + 1*81 = 118
    # byte 1 = digits 2 1 1 1 1 (s = 5..9)   -> 2 + 3 + 9 + 27 + 81 = 122
    # byte 2 = digits 1 1 1 1 1 (s = 10..14) -> 121
    # (a plane-major layout, five k of one plane per byte, would give 121, 120
    # and 124 instead)
    t = np.zeros((3, 1, 32), np.int8)
    t[1, 0, 0] = -1
    t[2, 0, 16] = 1
    idx = np.array([[0, 26]], np.uint8)
    d = tern.make_desc("bt3", 1, 32, 3, 16)
    buf = tern.pack(d, t, scale_idx=idx, codebook=synth.codebook27())
    col = buf[256:]
    assert (col[0], col[512], col[1024]) == (118, 122, 121)
    assert col[1] == 121 and col[512 + 1] == 121 and col[1024 + 15] == 121
    # index triple: index 0 (digits 0 0 0), index 26 (digits 2 2 2), padding 0:
    # byte 0 = digits 0 0 0 2 2 -> 2*27 + 2*81 = 216; byte 1 = digits 2 0 0 0 0 -> 2
    assert (col[1536], col[1536 + 32], col[1536 + 64]) == (216, 2, 0)
    u = oracle.unpack(buf)
    assert np.array_equal(u["trits"], t) and u["idx"].tolist() == [[0, 26]]


# ------------------------------------------------------------------ sizes
def test_packed_size_closed_forms():
    cases = [
        (tern.make_desc("bitnet", 2560, 2560, 1, 2560, 0.02), 256 + 80 * 40 * 512),
        (tern.make_desc("bitnet", 640, 2560, 1, 2560, 0.02), 256 + 20 * 40 * 512),
        (tern.make_desc("bitnet", 2560, 6912, 1, 6912, 0.02), 256 + 80 * 108 * 512),
        (tern.make_desc("tq", 4096, 4096, 3, 256), 256 + 128 * 64 * 3 * 512 + 128 * 16 * 3 * 64),
        (tern.make_desc("tq", 14336, 4096, 2, 32), 256 + 448 * 64 * 2 * 512 + 448 * 128 * 2 * 64),
        (tern.make_desc("bt3", 4096, 4096, 3, 16), 256 + 128 * 52 * 1632),
        (tern.make_desc("bt3", 4096, 14336, 3, 16), 256 + 128 * 180 * 1632),
    ]
    for d, size in cases:
        assert tern.packed_size(d) == size
    # physical bits per weight match the pages' accounting (2K + 16K/g) exactly
    # when the shape fills whole tiles
    for planes, g in ((1, 256), (2, 256), (3, 256), (4, 256), (2, 64), (2, 32)):
        d = tern.make_desc("tq", 4096, 4096, planes, g)
        bpw = (tern.packed_size(d) - 256) * 8 / (4096 * 4096)
        assert bpw == oracle.bits_per_weight("tq", planes, g)
    # balanced ternary: five trits per byte -> (48 + 3) / 5 * 8 / 16 = 5.1 bits
    # per weight when K fills whole 80-k columns (information content 5.05)
    d = tern.make_desc("bt3", 32, 4000, 3, 16)
    assert (tern.packed_size(d) - 256) * 8 / (32 * 4000) == pytest.approx(5.1)


def test_c1_layer_set_total_bytes():
    total = 0
    for name, n, k in synth.BITNET_2B_SHAPES:
        total += tern.packed_size(tern.make_desc("bitnet", n, k, 1, k, 0.02)) - 256
    assert total * synth.BITNET_2B_LAYERS == 30 * (2 * 1638400 + 2 * 409600 + 3 * 4423680)


# ------------------------------------------------------------------ errors
def expect(code, fn):
    with pytest.raises(tern.TernError) as ei:
        fn()
    assert ei.value.code == code


def test_error_paths():
    lay = synth.tq_layer(8, 64, 2, 32, seed=1)
    d = tern.desc_of(lay)
    bad = lay.trits.copy()
    bad[1, 3, 7] = 2
    expect(tern.EFORMAT, lambda: tern.pack(d, bad, lay.scales))
    s = lay.scales.copy()
    s[0, 0, 0] = np.float16(np.inf)
    expect(tern.EFORMAT, lambda: tern.pack(d, lay.trits, s))
    expect(tern.EINVAL, lambda: tern.pack(d, lay.trits, None))
    expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("tq", 8, 64, 2, 48)))
    expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("tq", 8, 96, 2, 64)))
    expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("tq", 8, 64, 5, 32)))
    expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("bitnet", 0, 64, 1, 64)))
    expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("bt3", 8, 40, 3, 16)))
    b3 = synth.bt3_layer(8, 32, seed=2)
    idx = b3.idx.copy()
    idx[0, 0] = 27
    expect(tern.EFORMAT, lambda: tern.pack(tern.desc_of(b3), b3.trits, scale_idx=idx, codebook=b3.codebook))
    cb = b3.codebook.copy()
    cb[4] = np.nan
    expect(tern.EFORMAT, lambda: tern.pack(tern.desc_of(b3), b3.trits, scale_idx=b3.idx, codebook=cb))
    # output capacity too small
    out = np.empty(100, np.uint8)
    used = ctypes.c_size_t()
    t = np.ascontiguousarray(lay.trits)
    sc = np.ascontiguousarray(lay.scales).view(np.uint16)
    rc = tern.lib.tern_pack(ctypes.byref(d), t.ctypes.data_as(ctypes.c_void_p), sc.ctypes.data_as(ctypes.c_void_p),
                            None, None, out.ctypes.data_as(ctypes.c_void_p), 100, ctypes.byref(used))
    assert rc == tern.ENOSPACE and used.value == tern.packed_size(d)
    # exactness bound of the int8 path: huge scales are refused
    big_lay = synth.tq_layer(8, 65536, 4, 16, seed=3)
    big = np.full_like(big_lay.scales, np.float16(60000.0))
    expect(tern.EFORMAT, lambda: tern.pack(tern.desc_of(big_lay), big_lay.trits, big))


def test_workspace_size_host_only():
    d = tern.make_desc("bitnet", 640, 2560, 1, 2560, 0.02)
    assert tern.workspace_size(d, 1) >= 0
    assert tern.workspace_size(tern.make_desc("tq", 1024, 4096, 2, 32), 16) > 0


def test_binding_fails_loudly_without_library(tmp_path):
    # the binding copied where no libtern.so sits beside it: importing it must
    # raise (there is no CPU fallback to drop to)
    import importlib.util
    import shutil
    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "packed_ternary_weight_b200", "tern.py")
    dst = tmp_path / "tern_nolib.py"
    shutil.copy(src, dst)
    spec = importlib.util.spec_from_file_location("tern_nolib", dst)
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="libtern.so not built"):
        spec.loader.exec_module(mod)


# ------------------------------------------ balanced ternary of depth 2 and 4
@pytest.mark.parametrize("depth", [2, 4])
@pytest.mark.parametrize("n,k", [(1, 16), (33, 160), (70, 400), (5, 2576)])
def test_roundtrip_bt_depths(depth, n, k):
    roundtrip(synth.bt3_layer(n, k, seed=n + k + depth, depth=depth))


def test_bt_depth2_bytes_by_hand():
    # one row, K = 16: t1[3] = -1 (digit 0), everything else 0 (digit 1). Tuple 3
    # holds the digits of k = 3 (weight 0: t0, t1), then of the padding weights
    # k = 19, 35, ... (digit 1): byte 0 = 1 + 0*3 + 1*9 + 1*27 + 1*81 = 118, byte 1
    # = 121. The index 5 = 2 + 1*3: triple byte 0 = 2 + 1*3 + 0*9 = 5 at 2 * 512.
    t = np.zeros((2, 1, 16), np.int8)
    t[1, 0, 3] = -1
    d = tern.make_desc("bt3", 1, 16, 2, 16)
    buf = tern.pack(d, t, scale_idx=np.array([[5]], np.uint8), codebook=synth.codebook27())
    assert len(buf) == 256 + 2 * 512 + 96
    col = buf[256:]
    assert col[3] == 118 and col[512 + 3] == 121 and col[0] == 121 and col[512] == 121
    assert col[1024] == 5 and col[1024 + 32] == 0 and col[1024 + 64] == 0
    u = oracle.unpack(buf)
    assert np.array_equal(u["trits"], t) and u["idx"].tolist() == [[5]]


def test_bt_depth4_bytes_by_hand():
    # one row, K = 16: t3[5] = +1 (digit 2). Tuple 5, byte 0 holds t0..t3 of k = 5
    # (1, 1, 1, 2) and t0 of the padding weight k = 21 (1): 1 + 3 + 9 + 2*27 + 81 =
    # 148; its bytes 1..3 are 121. A weight's four trits straddle bytes from the
    # second weight on: byte 1 = t1..t3 of k = 21 and t0, t1 of k = 37.
    t = np.zeros((4, 1, 16), np.int8)
    t[3, 0, 5] = 1
    d = tern.make_desc("bt3", 1, 16, 4, 16)
    buf = tern.pack(d, t, scale_idx=np.array([[26]], np.uint8), codebook=synth.codebook27())
    assert len(buf) == 256 + 4 * 512 + 96
    col = buf[256:]
    assert col[5] == 148 and all(col[b * 512 + 5] == 121 for b in (1, 2, 3))
    assert col[2048] == 26        # 26 = 2 + 2*3 + 2*9: digits 2, 2, 2 of the first index
    u = oracle.unpack(buf)
    assert np.array_equal(u["trits"], t) and u["idx"].tolist() == [[26]]


def test_bt_depth_sizes_and_bits():
    for depth in (2, 3, 4):
        d = tern.make_desc("bt3", 4096, 4096, depth, 16)
        assert tern.packed_size(d) == 256 + 128 * 52 * (512 * depth + 96)
        # (16 d + 3) base-3 bytes per 80 weights of a row: (16 d + 3) / 10 bits per weight
        d = tern.make_desc("bt3", 32, 4000, depth, 16)
        assert (tern.packed_size(d) - 256) * 8 / (32 * 4000) == pytest.approx((16 * depth + 3) / 10)
    for depth in (1, 5):
        expect(tern.EINVAL, lambda: tern.packed_size(tern.make_desc("bt3", 8, 32, depth, 16)))


def test_bt_depths_take_bf16_only():
    # every depth has a kernel for bf16 activations; int8 activations are refused
    # on the host, before any device work
    torch = pytest.importorskip("torch")
    for depth in (2, 3, 4):
        lay = synth.bt3_layer(64, 160, seed=9, depth=depth)
        d, buf = tern.pack_layer(lay)
        packed = torch.from_numpy(buf).clone()          # torch's allocation: 64-byte aligned
        x = torch.zeros(160, dtype=torch.int8)
        sx = torch.ones(1, dtype=torch.float32)
        y = torch.zeros(64, dtype=torch.float32)
        expect(tern.EUNSUPPORTED, lambda: tern.gemv(d, packed, tern.ACT_INT8, x, sx, tern.OUT_F32, y, stream=0))


def test_selftest_limit_checked_on_host():
    for bad in (0, 999, 2_000_000_000):
        expect(tern.EINVAL, lambda: tern.selftest_wait(bad, stream=0))
