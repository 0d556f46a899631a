"""Host logic on CPU: the helpers that the host and the kernels both call (the
column-balanced CTA split of the one-CTA-per-SM GEMV, the token-pass and
shared-memory plans of the tensor-core GEMM, the level decoders of balanced
ternary at depth 2 and 4) are built with the host compiler and checked against
brute force, exhaustive enumeration, the packer's own bytes and the limits they
must respect (shared memory, tensor-memory columns, alignment)."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def h(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("plan") / "libplan.so")
    subprocess.run([cxx, "-O1", "-std=c++17", "-shared", "-fPIC", "-I", ROOT,
                    os.path.join(HERE, "plan_harness.cpp"), "-o", out], check=True)
    lib = ctypes.CDLL(out)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.h_cta_tile.argtypes = [ip, ip, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.h_passes.argtypes = [ctypes.c_int, ctypes.c_int, ip, ip]
    lib.h_layout.argtypes = [ctypes.c_int] * 5 + [ctypes.POINTER(ctypes.c_longlong)]
    return lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


# --------------------------------------------------- CTA split (mixed K)
def _split(h, row_tiles, cols, grid):
    tb = np.concatenate([[0], np.cumsum(row_tiles)]).astype(np.int32)
    cb = np.concatenate([[0], np.cumsum(np.asarray(row_tiles) * np.asarray(cols))]).astype(np.int32)
    return tb, cb, [h.h_cta_tile(_ptr(tb), _ptr(cb), len(row_tiles), c, grid) for c in range(grid + 1)]


def _brute(row_tiles, cols, grid):
    """CTA c starts at the first tile whose first column is at or after the c-th
    equal share of all columns (floor), or at the end."""
    starts = []
    pos = 0
    for rt, nc in zip(row_tiles, cols):
        for _ in range(rt):
            starts.append(pos)
            pos += nc
    tot = pos
    out = []
    for c in range(grid + 1):
        cg = tot * c // grid
        out.append(next((i for i, s in enumerate(starts) if s >= cg), len(starts)))
    return out


@pytest.mark.parametrize("seed", range(12))
def test_cta_split_matches_brute_force(h, seed):
    g = np.random.default_rng(seed)
    nprob = int(g.integers(1, 40))
    row_tiles = g.integers(1, 60, nprob).tolist()
    cols = g.choice([4, 16, 40, 108, 224], nprob).tolist()      # K = 256 .. 14336 at 64 k per column
    for grid in (1, 3, 37, 148):
        _, _, got = _split(h, row_tiles, cols, grid)
        assert got == _brute(row_tiles, cols, grid), (row_tiles, cols, grid)


def test_cta_split_bitnet_layer_set(h):
    # the 30-layer set in one launch: 180 problems of K = 2560 (40 columns), then
    # 30 of K = 6912 (108 columns); q, k, v, o, gate, up have 80, 20, 20, 80, 216, 216 row tiles
    row_tiles = [80, 20, 20, 80, 216, 216] * 30 + [80] * 30
    cols = [40] * 180 + [108] * 30
    tb, cb, t = _split(h, row_tiles, cols, 148)
    assert t[0] == 0 and t[-1] == tb[-1]
    assert all(b > a for a, b in zip(t, t[1:])), "a CTA without tiles"
    # columns per CTA: within one tile's columns of the equal share
    starts = np.repeat(cb[:-1], row_tiles) + np.concatenate([np.arange(r) * c for r, c in zip(row_tiles, cols)])
    starts = np.append(starts, cb[-1])
    share = cb[-1] / 148
    per = np.diff(starts[t])
    assert np.all(np.abs(per - share) < max(cols)), per
    assert per.sum() == cb[-1]


def test_cta_split_edges(h):
    # one problem, as many tiles as CTAs: one tile each
    _, _, t = _split(h, [148], [40], 148)
    assert t == list(range(149))
    # fewer equal-width tiles than CTAs would leave CTAs empty: the split shows it
    _, _, t = _split(h, [100], [40], 148)
    assert any(b == a for a, b in zip(t, t[1:]))
    # a single CTA takes everything
    _, _, t = _split(h, [3, 5, 7], [4, 108, 40], 1)
    assert t == [0, 15]


# ------------------------------------------------------------ token passes
def test_mt_pad(h):
    kmax = h.h_const(8)
    assert kmax == 8
    for mt in range(1, kmax + 1):
        p = h.h_mt_pad(mt)
        assert p >= mt and p in (1, 2, 4, 8)
        assert p == 1 or p // 2 < mt          # the smallest power of two that holds mt


def test_tensor_passes_fit_tensor_memory(h):
    tmax_tokens = h.h_const(4)
    for digits in range(1, h.h_const(5) + 1):
        for m16 in range(16, tmax_tokens + 1, 16):
            ps, tp = ctypes.c_int(), ctypes.c_int()
            h.h_passes(digits, m16, ctypes.byref(ps), ctypes.byref(tp))
            ps, tp = ps.value, tp.value
            assert tp % 16 == 0 and 16 <= tp <= tmax_tokens
            assert digits * tp <= 512, (digits, m16, tp)           # tensor-memory columns
            assert ps * tp >= m16 and (ps - 1) * tp < m16             # no empty pass
            tmax = min(tmax_tokens, (512 // digits) // 16 * 16)
            assert ps == -(-m16 // tmax)                              # fewest passes


def test_merged_digits_hold_every_scale(h):
    # fp16 magnitudes are below 2^40 units of 2^-24: D7 <= 6 digits of 7 bits;
    # merged digits of b bits (7, 6, 5 for 1, 2, 3-4 planes) must hold the same bits
    # and their per-plane sum must stay an int8 (planes * (2^b - 1) <= 127)
    for planes, b in ((1, 7), (2, 6), (3, 5), (4, 5)):
        assert planes * (2 ** b - 1) <= 127
        for d7 in range(1, h.h_const(6) + 1):
            dm = h.h_merged_digits(planes, d7)
            assert dm * b >= 7 * d7 and (dm - 1) * b < 7 * d7
            assert dm <= h.h_const(5)


# ------------------------------------------------- tensor shared-memory plan
def _routes():
    """Every (planes, tq, group, digit count) the host may hand the tensor kernel."""
    for planes in (1, 2, 3, 4):
        for group in (16, 32, 64, 128, 256):
            for d7 in range(1, 7):
                yield planes, 1, group, d7
    yield 1, 0, 0, 1                                                    # BitNet: one digit


def test_tensor_layout_fits_every_route(h):
    smem, slot_bytes = h.h_const(0), h.h_const(1)
    max_stages, max_slots = h.h_const(2), h.h_const(3)
    plane_col = h.h_const(7)
    out = (ctypes.c_longlong * 13)()
    for planes, tq, group, d7 in _routes():
        digits = h.h_merged_digits(planes, d7) if tq else 1
        for m16 in range(16, h.h_const(4) + 1, 16):
            ps, tp = ctypes.c_int(), ctypes.c_int()
            h.h_passes(digits, m16, ctypes.byref(ps), ctypes.byref(tp))
            ok = h.h_layout(planes, tq, group, digits, tp.value, out)
            bars, misc, stages, slots, raw, sc, xcol, stage, C, NS, nslot, NG, sg = list(out)
            case = (planes, tq, group, d7, m16)
            assert ok, case
            assert misc + 64 <= stages                                  # barriers and misc words first
            assert stages + NS * stage <= slots, case                   # input stages below the A tiles
            assert slots + nslot * slot_bytes == smem and slots % 1024 == 0
            assert stage % 128 == 0 and raw % 128 == 0 and xcol % 16 == 0
            assert 2 <= NS <= max_stages and nslot == NG * digits <= max_slots
            assert C in (1, 2, 4) and raw == 4 * C * planes * plane_col
            assert xcol == 64 * tp.value                                # one 64-k column of every token
            if tq:                                                      # the stage's scale blocks
                assert sg == (64 * C // group if 64 * C >= group else 1)
                assert sc >= 4 * sg * planes * 64


# ------------------------------------- balanced-ternary levels, depth 2 and 4
def _u32(a):
    return np.ascontiguousarray(a, dtype=np.uint32)


def _levels_ref(tuple_bytes, d):
    """Levels U_j = sum_p 3^p u_{dj+p} from the 5d base-3 digits of a tuple of d bytes (byte 0 first)."""
    digs = []
    for b in tuple_bytes:
        v = int(b)
        for _ in range(5):
            digs.append(v % 3)
            v //= 3
    return [sum(3 ** p * digs[d * j + p] for p in range(d)) for j in range(5)]


def _decode(h, d, cols):
    """cols: [d][n] packed words (two tuples per word, one per 16-bit lane)."""
    n = cols.shape[1]
    out = np.zeros(5 * n, np.uint32)
    P = ctypes.POINTER(ctypes.c_uint32)
    keep = [_u32(c) for c in cols]                      # the buffers stay alive during the call
    args = [k.ctypes.data_as(P) for k in keep]
    if d == 2:
        h.h_pair_levels(*args, n, out.ctypes.data_as(P))
    else:
        h.h_quad_levels(*args, n, out.ctypes.data_as(P))
    return out.reshape(n, 5)


def _check_lanes(h, d, lo, hi):
    """lo, hi: [n][d] bytes of the tuples in the low and high lanes."""
    cols = (hi.astype(np.uint32) << 16) | lo.astype(np.uint32)
    got = _decode(h, d, cols.T)
    for lane, tb in ((0, lo), (16, hi)):
        g = (got >> lane) & 0xFFFF
        ref = np.array([_levels_ref(t, d) for t in tb])
        assert np.array_equal(g, ref), (d, lane)


def test_pair_levels_exhaustive(h):
    # every tuple of two base-3 bytes (243^2), against a different tuple in the other lane
    b = np.arange(243)
    lo = np.stack(np.meshgrid(b, b, indexing="ij"), -1).reshape(-1, 2)
    _check_lanes(h, 2, lo, lo[::-1].copy())


def test_quad_levels_every_byte_pair(h):
    # each level reads at most two neighbouring bytes: every value pair of bytes (i, i + 1),
    # the other bytes random, both lanes
    g = np.random.default_rng(3)
    b = np.arange(243)
    pairs = np.stack(np.meshgrid(b, b, indexing="ij"), -1).reshape(-1, 2)
    for i in range(3):
        lo = g.integers(0, 243, size=(len(pairs), 4))
        lo[:, i:i + 2] = pairs
        hi = g.integers(0, 243, size=(len(pairs), 4))
        hi[:, (i + 1) % 3:(i + 1) % 3 + 2] = pairs[::-1]
        _check_lanes(h, 4, lo, hi)


@pytest.mark.parametrize("d", [2, 4])
def test_levels_from_packed_layers(h, d):
    # the decoders on the packer's own bytes give the oracle's levels: tuple i of row r in a
    # column holds k = 80c + 16j + i (j = 0..4)
    from packed_ternary_weight_b200 import synth, tern
    import oracle
    lay = synth.bt3_layer(64, 160, seed=40 + d, depth=d)
    _, buf = tern.pack_layer(lay)
    hdr = oracle.parse_header(buf)
    col = np.asarray(buf[hdr["trit_offset"]:], np.uint8)
    colb = 512 * d + 96
    level = sum(3 ** p * lay.trits[p].astype(np.int64) for p in range(d)) + (3 ** d - 1) // 2   # U of every weight
    for T in range(hdr["row_tiles"]):
        for c in range(hdr["cols"]):
            base = (T * hdr["cols"] + c) * colb
            tb = np.stack([col[base + b * 512: base + b * 512 + 512].reshape(32, 16) for b in range(d)], -1)
            tb = tb.reshape(-1, d)                                 # [(r, i)][b]
            half = len(tb) // 2
            cols = ((tb[half:].astype(np.uint32) << 16) | tb[:half]).T
            got = _decode(h, d, cols)
            U = np.concatenate([got & 0xFFFF, got >> 16])          # [(r, i)][j]
            r = np.arange(32).repeat(16)
            i = np.tile(np.arange(16), 32)
            for j in range(5):
                k = 80 * c + 16 * j + i
                n = 32 * T + r
                m = (k < lay.k) & (n < lay.n)
                assert np.array_equal(U[m, j], level[n[m], k[m]]), (T, c, j)
