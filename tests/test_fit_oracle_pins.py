"""Pins for the dense -> ternary fit oracle (oracle/fit.py), CPU only.

The pages give no fitting algorithm, so the readings in oracle/fit.py are
pinned by what any correct implementation of them must satisfy: matrices
already in the format come back exactly, each least-squares plane lowers the
error, power-of-two scaling and sign flips carry through exactly, the level
choice is the brute-force optimum, and the balanced-ternary digits are the
unique ones (checked against the pinned dequantiser).
"""
import numpy as np
import pytest

import oracle
from oracle import fit
from packed_ternary_weight_b200 import synth


def gauss(seed, n, k, scale=0.02):
    return (np.random.default_rng(seed).standard_normal((n, k)) * scale).astype(np.float32)


@pytest.mark.parametrize("group", [32, 256])
def test_tq_recovers_single_plane_matrices(group):
    g = np.random.default_rng(1)
    n, k = 12, 2 * group
    t = synth.draw_trits(g, (1, n, k))
    t[0, 0, :group] = 0                                 # an all-zero group: scale 0, trits 0
    s = (np.abs(g.standard_normal((1, n, k // group))) * 0.02).astype(np.float16)
    s[0, 0, 0] = 0
    w = (t[0] * np.repeat(s[0].astype(np.float32), group, axis=1)).astype(np.float32)
    for planes in (1, 2, 4):
        tr, sc = fit.fit_tq(w, planes, group)
        assert np.array_equal(tr[0], t[0]) and np.array_equal(sc[0].view(np.uint16), s[0].view(np.uint16))
        assert not tr[1:].any() and not sc[1:].astype(np.float32).any()
        assert np.array_equal(fit.reconstruct_tq(tr, sc, group), w.astype(np.float64))


def test_tq_planes_lower_the_error():
    w = gauss(2, 64, 512)
    tr, sc = fit.fit_tq(w, 4, 64)
    errs = [np.sum((w - fit.reconstruct_tq(tr[:p], sc[:p], 64)) ** 2) for p in range(5)]
    assert all(errs[p + 1] < errs[p] for p in range(4)), errs
    assert errs[3] < 0.05 * errs[0]                     # three planes: within a few percent


def test_tq_power_of_two_and_sign():
    w = gauss(3, 16, 256)
    tr, sc = fit.fit_tq(w, 3, 64)
    tr4, sc4 = fit.fit_tq(4 * w, 3, 64)
    assert np.array_equal(tr4, tr)
    assert np.array_equal(sc4.astype(np.float32), 4 * sc.astype(np.float32))
    trn, scn = fit.fit_tq(-w, 3, 64)
    assert np.array_equal(trn, -tr) and np.array_equal(scn.view(np.uint16), sc.view(np.uint16))


def test_tq_threshold_and_scale_by_hand():
    # one group of 16: |w| = 1, 3, 0.5, 2 and twelve zeros -> absmean 6.5 / 16 =
    # 0.40625, threshold 0.203125: the four non-zeros become +1, +1, +1, -1 and
    # the least-squares scale is (1 + 3 + 0.5 + 2) / 4 = 1.625 (exact in fp16)
    w = np.array([[1.0, 3.0, 0.5, -2.0] + [0.0] * 12], np.float32)
    tr, sc = fit.fit_tq(w, 1, 16)
    assert tr[0, 0].tolist() == [1, 1, 1, -1] + [0] * 12
    assert float(sc[0, 0, 0]) == 1.625
    # a value at 0.1 (below the threshold of its group) stays 0
    w2 = w.copy()
    w2[0, 5] = 0.1
    tr2, _ = fit.fit_tq(w2, 1, 16)
    assert tr2[0, 0, 5] == 0


def test_bt_digits_exhaustive():
    for d in (2, 3, 4):
        lmax = (3 ** d - 1) // 2
        L = np.arange(-lmax, lmax + 1)
        t = fit.balanced_digits(L, d)
        assert set(np.unique(t)) <= {-1, 0, 1}
        assert np.array_equal(sum(3 ** j * t[j].astype(np.int64) for j in range(d)), L)
        # the pinned dequantiser reads the same levels back (codebook entry 1.0), padded to groups of 16
        pad = (-L.size) % 16
        tp = np.concatenate([t, np.zeros((d, pad), np.int8)], axis=1)[:, None, :]
        w = oracle.dequantize("bt3", tp, 16, idx=np.zeros((1, tp.shape[2] // 16), np.uint8),
                              codebook=np.ones(27, np.float32))
        assert np.array_equal(w[0, :L.size], L)


@pytest.mark.parametrize("depth", [2, 3, 4])
def test_bt_recovers_matrices_in_the_format(depth):
    g = np.random.default_rng(4 + depth)
    n, k = 8, 64
    lmax = (3 ** depth - 1) // 2
    cb = synth.codebook27()
    # levels 0 and signed powers of two up to the depth's range, so that every
    # w = cb[idx] * L is exact in fp32 (the fit's input)
    pw = [0] + [s * 2 ** e for e in range(int(np.log2(lmax)) + 1) for s in (1, -1)]
    L = g.choice(pw, size=(n, k))
    L[:, ::16] = 2 ** int(np.log2(lmax))                # every group reaches its largest power of two
    idx = g.integers(0, 27, size=(n, k // 16)).astype(np.uint8)
    w = (np.repeat(cb[idx].astype(np.float64), 16, axis=1) * L).astype(np.float32)
    assert np.array_equal(w.astype(np.float64), np.repeat(cb[idx].astype(np.float64), 16, axis=1) * L)
    t, ix = fit.fit_bt(w, cb, depth)
    assert np.array_equal(ix, idx)
    assert np.array_equal(fit.reconstruct_bt(t, ix, cb), w.astype(np.float64))


def test_bt_levels_are_the_brute_force_optimum():
    g = np.random.default_rng(9)
    cb = synth.codebook27()
    w = (g.standard_normal((3, 32)) * 0.01).astype(np.float32)
    t, ix = fit.fit_bt(w, cb, 3)
    best = []
    for r in range(3):
        for G in range(2):
            x = w[r, 16 * G:16 * G + 16].astype(np.float64)
            errs = []
            for c in cb.astype(np.float64):
                cand = np.arange(-13, 14)
                e = ((x[:, None] - c * cand[None, :]) ** 2).min(axis=1).sum()
                errs.append(e)
            best.append(int(np.argmin(errs)))
    assert ix.reshape(-1).tolist() == best
    # and the reconstruction error never exceeds any single codebook entry's
    rec = fit.reconstruct_bt(t, ix, cb)
    assert np.sum((w - rec) ** 2) <= np.sum((w - fit.reconstruct_bt(t * 0, ix, cb)) ** 2)


def test_fit_feeds_the_packer_and_dequantiser():
    from packed_ternary_weight_b200 import tern
    w = gauss(11, 40, 256)
    tr, sc = fit.fit_tq(w, 3, 64)
    d = tern.make_desc("tq", 40, 256, 3, 64)
    buf = tern.pack(d, tr, sc)
    u = oracle.unpack(buf)
    assert np.array_equal(oracle.dequantize("tq", u["trits"], 64, scales=u["scales"]), fit.reconstruct_tq(tr, sc, 64))
    cb = synth.codebook27()
    t3, ix = fit.fit_bt(w, cb, 3)
    d = tern.make_desc("bt3", 40, 256, 3, 16)
    buf = tern.pack(d, t3, None, ix, cb)
    u = oracle.unpack(buf)
    assert np.array_equal(oracle.dequantize("bt3", u["trits"], 16, idx=u["idx"], codebook=u["codebook"]),
                          fit.reconstruct_bt(t3, ix, cb))
