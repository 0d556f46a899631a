"""Plain CPU oracle of the dense -> ternary fits -- TEST INFRASTRUCTURE ONLY.

Imported only by tests and the benchmark's CPU legs; nothing here is shared
with the CUDA path. The pages describe the fits but give no algorithm:

* sasori README, "How it works & paper": each weight matrix is fit on its own
  into a sum of K per-group-scaled trit planes, layer-local and weight-only,
  with no calibration data; "K and g": K planes, fp16 scale per group of g.
* Entrit card, "Quantization details": depth d = 3 (27 levels), group 16, a
  27-entry log-spaced scale codebook, "Uniform PTQ".

Readings taken here (the plainest ones the pages support):

* ``fit_tq`` -- greedy residual planes. R_0 = W; for plane p and each (row,
  group): gamma = mean |R| over the group; t = sign(R) where |R| > gamma / 2,
  else 0 (ternary rounding of R / gamma); the least-squares scale for these
  trits, s* = sum_{t != 0} |R| / #{t != 0} (0 when no trit is set), stored as
  fp16 (round to nearest even); R_{p+1} = R_p - s t.
* ``fit_bt`` -- uniform levels per group of 16: for every codebook entry c the
  levels L = clamp(rint(w / c), -(3^d - 1)/2, (3^d - 1)/2) (ties to even), and
  the entry with the smallest sum of squared errors (the lowest index on a
  tie); the trits are the balanced-ternary digits of L (L = sum_j 3^j t_j).

Arithmetic: fp64, sums taken element by element in index order within a group
(the same order the GPU kernels use), every product and sum rounded on its own.
Parity against these definitions is exact; against the pages it is unpinned
(they give no algorithm), so the tests pin properties instead: exact recovery
of matrices that are already in the format, the monotone error decrease of the
least-squares planes, power-of-two equivariance and brute force over levels.
"""
from __future__ import annotations

import numpy as np

__all__ = ["fit_tq", "fit_bt", "balanced_digits", "reconstruct_tq", "reconstruct_bt"]


def fit_tq(w: np.ndarray, planes: int, group: int):
    """w fp32 [N][K] -> (trits int8 [P][N][K], scales fp16 [P][N][K/g])."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % group == 0
    G = k // group
    R = w.astype(np.float64).reshape(n, G, group).copy()
    trits = np.zeros((planes, n, G, group), np.int8)
    scales = np.zeros((planes, n, G), np.float16)
    for p in range(planes):
        a = np.zeros((n, G))
        for i in range(group):                         # sum |R| in index order
            a = a + np.abs(R[:, :, i])
        gamma = a / group
        half = gamma / 2
        t = np.where(R > half[:, :, None], 1, np.where(R < -half[:, :, None], -1, 0)).astype(np.int8)
        t[gamma == 0] = 0
        num = np.zeros((n, G))
        cnt = np.zeros((n, G))
        for i in range(group):
            nz = t[:, :, i] != 0
            num = np.where(nz, num + np.abs(R[:, :, i]), num)
            cnt = cnt + nz
        s = np.where(cnt > 0, num / np.maximum(cnt, 1), 0.0).astype(np.float16)   # fp64 -> fp16, nearest even
        trits[p] = t
        scales[p] = s
        R = R - s.astype(np.float64)[:, :, None] * t
    return trits.reshape(planes, n, k), scales


def reconstruct_tq(trits, scales, group):
    t = np.asarray(trits, np.float64)
    s = np.repeat(np.asarray(scales, np.float16).astype(np.float64), group, axis=2)
    return (t * s).sum(axis=0)


def balanced_digits(levels: np.ndarray, depth: int) -> np.ndarray:
    """The balanced-ternary digits t_j (L = sum_j 3^j t_j, t_j in {-1,0,1}) of integer levels."""
    L = np.asarray(levels, dtype=np.int64).copy()
    out = np.zeros((depth,) + L.shape, np.int8)
    for j in range(depth):
        r = np.mod(L + 1, 3) - 1                       # digit in {-1, 0, 1} with L = r (mod 3)
        out[j] = r
        L = (L - r) // 3
    assert np.all(L == 0), "level outside the depth's range"
    return out


def fit_bt(w: np.ndarray, codebook: np.ndarray, depth: int = 3, group: int = 16):
    """w fp32 [N][K] -> (trits int8 [d][N][K], idx uint8 [N][K/16])."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % group == 0
    G = k // group
    lmax = (3 ** depth - 1) // 2
    x = w.astype(np.float64).reshape(n, G, group)
    cb = np.asarray(codebook, dtype=np.float32).astype(np.float64)
    best_err = np.full((n, G), np.inf)
    best_idx = np.zeros((n, G), np.int64)
    best_L = np.zeros((n, G, group), np.int64)
    for ci, c in enumerate(cb):
        L = np.clip(np.rint(x / c), -lmax, lmax)        # numpy rint: ties to even
        err = np.zeros((n, G))
        for i in range(group):                          # squared errors summed in index order
            d = x[:, :, i] - c * L[:, :, i]
            err = err + d * d
        better = err < best_err
        best_err = np.where(better, err, best_err)
        best_idx = np.where(better, ci, best_idx)
        best_L = np.where(better[:, :, None], L, best_L).astype(np.int64)
    trits = balanced_digits(best_L, depth).reshape(depth, n, k)
    return trits, best_idx.astype(np.uint8)


def reconstruct_bt(trits, idx, codebook, group=16):
    t = np.asarray(trits, np.int64)
    lev = sum((3 ** j) * t[j] for j in range(t.shape[0]))
    sc = np.asarray(codebook, np.float32).astype(np.float64)[np.asarray(idx, np.int64)]
    return np.repeat(sc, group, axis=1) * lev
