"""GPU parity of large single-token launches (one CTA per SM, warp column
ranges, shared tiles combined in warp order) against the CPU oracle.

Launches with at least four row tiles per SM take this path: grouped launches
of many GEMVs, and ragged mixes of problem sizes so that CTAs span several
problems and warps share tiles. int8 paths bit-exact; bf16 within the same
tolerance as the other bf16 tests.
"""
import numpy as np
import pytest

import oracle
from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

BF16_TOL = 1e-3


@pytest.fixture(scope="module")
def tern():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from packed_ternary_weight_b200 import tern as t
    return t


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_bf16(y32, yref):
    floor = 1e-2 * np.sqrt(np.mean(yref ** 2))
    err = np.abs(y32.astype(np.float64) - yref) / np.maximum(np.abs(yref), floor)
    assert err.max() <= BF16_TOL, f"max rel err {err.max():.3g}"


def sample_rows(n, count, seed):
    if n <= count:
        return np.arange(n)
    rows = np.random.default_rng(seed).choice(n, count, replace=False)
    # always include both ends and the tile boundaries next to them
    return np.unique(np.concatenate([rows, [0, 31, 32, n - 33, n - 1] if n > 33 else [0, n - 1]]))


def run_grouped(tern, layers, act, out=None, flags=0, reps=1):
    """One grouped launch over the layers; returns outputs (host), bf16 inputs and int8 inputs."""
    out = tern.OUT_F32 if out is None else out
    descs, packs, xs, xqs, sxs, ys, xbits = [], [], [], [], [], [], []
    for lay in layers:
        d, buf = tern.pack_layer(lay, flags=flags)
        descs.append(d)
        packs.append(dev(buf))
        x = synth.draw_x_bf16(lay.seed, 1, lay.k)
        xbits.append(x)
        xs.append(dev(x.view(np.int16))[0])
        q, s = oracle.quantize_act(x)
        xqs.append(dev(q)[0])
        sxs.append(dev(s))
        ys.append(torch.empty(lay.n, dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda"))
    results = []
    for _ in range(reps):
        for y in ys:
            y.fill_(0)
        if act == tern.ACT_INT8:
            tern.gemv_grouped(descs, packs, act, xqs, sxs, out, ys)
        else:
            tern.gemv_grouped(descs, packs, act, xs, None, out, ys)
        torch.cuda.synchronize()
        assert tern.device_error() == tern.OK
        results.append([y.cpu().numpy().copy() for y in ys])
    return results, xbits


def int8_reference(lay, x, rows):
    q, s = oracle.quantize_act(x)
    if lay.fmt == "bitnet":
        return oracle.gemv_bitnet_int8(lay.trits[:, rows], q, s, lay.tensor_scale)[0]
    return oracle.gemv_tq_int8(lay.trits[:, rows], lay.scales[:, rows], lay.group, q, s)[0]


def check_int8_group(tern, layers, act, nrows=256, flags=0):
    (ys,), xbits = run_grouped(tern, layers, act, flags=flags)
    for i, (lay, y, x) in enumerate(zip(layers, ys, xbits)):
        rows = sample_rows(lay.n, nrows, i)
        ref = int8_reference(lay, x, rows)
        got = y[rows]
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), \
            f"problem {i}: mismatch at rows {rows[np.flatnonzero(got != ref)[:5]]}"


def test_bitnet_gate_x30_fused_quant(tern):
    layers = [synth.bitnet_layer(6912, 2560, 5000 + i) for i in range(30)]
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, flags=tern.F_PDL)


def test_bitnet_down_x30_int8_full_rows(tern):
    layers = [synth.bitnet_layer(2560, 6912, 5100 + i) for i in range(30)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=2560)


def test_bitnet_kv_x30(tern):
    layers = [synth.bitnet_layer(640, 2560, 5200 + i) for i in range(30)]
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, nrows=640)


def test_ragged_problem_mix_spans_and_shared_tiles(tern):
    # row counts that are not multiples of 32, problems far smaller than a
    # CTA's share, ragged K (scalar activation loads): CTAs span up to three
    # problems and warp boundaries cut tiles
    ns = [90, 22400, 17, 150, 2870, 40, 9590]
    layers = [synth.bitnet_layer(n, 1000, 5300 + i) for i, n in enumerate(ns)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=4096)
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, nrows=4096)


def test_tq2p_g32_int8_x2(tern):
    layers = [synth.tq_layer(14336, 4096, 2, 32, seed=5400 + i) for i in range(2)]
    check_int8_group(tern, layers, tern.ACT_INT8)


def test_tq3p_g256_fused_quant_x20(tern):
    layers = [synth.tq_layer(1024, 4096, 3, 256, seed=5500 + i) for i in range(20)]
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, nrows=128)


def test_tq3p_g64_int8_mixed_rows(tern):
    layers = [synth.tq_layer(n, 2048, 3, 64, seed=5600 + i) for i, n in enumerate([3200, 100, 9000, 33, 7000])]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=512)


@pytest.mark.parametrize("planes,group", [(3, 256), (2, 32), (4, 256)])
def test_tq_bf16_grouped(tern, planes, group):
    layers = [synth.tq_layer(1024, 4096, planes, group, seed=5700 + 10 * planes + i) for i in range(20)]
    (y32,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    (y16,), _ = run_grouped(tern, layers, tern.ACT_BF16, out=tern.OUT_BF16)
    for i, (lay, y, yb, x) in enumerate(zip(layers, y32, y16, xbits)):
        rows = sample_rows(lay.n, 128, i)
        w = oracle.dequantize("tq", lay.trits[:, rows], lay.group, scales=lay.scales[:, rows])
        check_bf16(y[rows], oracle.gemv_bf16(w, x)[0])
        assert np.array_equal(yb.view(np.uint16), synth.f32_to_bf16_bits(y))


def test_bf16_deterministic(tern):
    layers = [synth.tq_layer(n, 4096, 3, 256, seed=5800 + i) for i, n in enumerate([5000, 70, 9000, 6000])]
    runs, _ = run_grouped(tern, layers, tern.ACT_BF16, reps=3)
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def bt3_check(layers, ys, xbits, nrows, outs16=None):
    for i, (lay, y, x) in enumerate(zip(layers, ys, xbits)):
        rows = sample_rows(lay.n, nrows, i)
        w = oracle.dequantize("bt3", lay.trits[:, rows], 16, idx=lay.idx[rows], codebook=lay.codebook)
        check_bf16(y[rows], oracle.gemv_bf16(w, x)[0])
        if outs16 is not None:
            assert np.array_equal(outs16[i].view(np.uint16), synth.f32_to_bf16_bits(y))


def test_bt3_llama_q_x8(tern):
    # balanced ternary d = 3 in the one-CTA-per-SM kernel: 8 x 128 row tiles
    layers = [synth.bt3_layer(4096, 4096, seed=5900 + i) for i in range(8)]
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    (y16,), _ = run_grouped(tern, layers, tern.ACT_BF16, out=tern.OUT_BF16)
    bt3_check(layers, ys, xbits, 256, y16)


def test_bt3_down_long_k_x5(tern):
    # K = 14336: the largest activation image per problem
    layers = [synth.bt3_layer(4096, 14336, seed=5950 + i) for i in range(5)]
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    bt3_check(layers, ys, xbits, 128)


def test_bt3_ragged_mix(tern):
    # rows not multiples of 32, K not a multiple of 80 (padded last column),
    # problems much smaller than a CTA's share next to large ones
    ns = [70, 20000, 33, 1500, 9000]
    layers = [synth.bt3_layer(n, 1040, seed=6000 + i) for i, n in enumerate(ns)]
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    bt3_check(layers, ys, xbits, 1024)
    runs, _ = run_grouped(tern, layers, tern.ACT_BF16, reps=2)
    for a, b in zip(runs[0], runs[1]):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


# ------------------------------------------------- problems of different K
def test_bitnet_layer_set_one_launch(tern):
    # the BitNet-2B layer set's shapes in one launch: q,k,v,o,gate,up (K = 2560)
    # next to down (K = 6912); CTAs balance columns, images of both widths
    shapes = [(2560, 2560), (640, 2560), (640, 2560), (2560, 2560), (6912, 2560), (6912, 2560), (2560, 6912)]
    layers = [synth.bitnet_layer(n, k, 6100 + i) for i, (n, k) in enumerate(shapes * 4)]
    layers.sort(key=lambda L: L.k)
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, nrows=512, flags=tern.F_PDL)
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=512)


def test_mixed_k_interleaved_ragged(tern):
    # K changes from problem to problem, ragged K (scalar loads), CTAs span
    # problems of different widths
    spec = [(9000, 1000), (70, 6912), (20000, 256), (33, 2560), (5000, 6912), (12000, 64), (3000, 4000)]
    layers = [synth.bitnet_layer(n, k, 6200 + i) for i, (n, k) in enumerate(spec)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=1024)
    check_int8_group(tern, layers, tern.ACT_BF16_Q8, nrows=1024)


def test_mixed_k_tq_int8_and_bf16(tern):
    spec = [(14336, 4096), (4096, 14336), (1024, 4096), (4096, 14336), (14336, 4096)]
    layers = [synth.tq_layer(n, k, 3, 256, seed=6300 + i) for i, (n, k) in enumerate(spec)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=256)
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    for i, (lay, y, x) in enumerate(zip(layers, ys, xbits)):
        rows = sample_rows(lay.n, 128, i)
        w = oracle.dequantize("tq", lay.trits[:, rows], lay.group, scales=lay.scales[:, rows])
        check_bf16(y[rows], oracle.gemv_bf16(w, x)[0])


def test_mixed_k_bt3(tern):
    spec = [(9000, 4096), (4096, 14336), (30, 1040), (6000, 4096)]
    layers = [synth.bt3_layer(n, k, seed=6400 + i) for i, (n, k) in enumerate(spec)]
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    bt3_check(layers, ys, xbits, 256)


def test_mixed_k_small_launch_runs_per_k(tern):
    # too few tiles for the one-CTA-per-SM kernel: one row-group launch per run of equal K
    spec = [(300, 1024), (200, 1024), (100, 2048), (64, 1024)]
    layers = [synth.bitnet_layer(n, k, 6500 + i) for i, (n, k) in enumerate(spec)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=300)


@pytest.mark.parametrize("planes,group", [(1, 32), (1, 64), (2, 64), (2, 128), (3, 128), (4, 32), (4, 64)])
def test_tq_plane_group_variants_grouped(tern, planes, group):
    # the one-CTA-per-SM kernel for plane counts and group sizes beyond the pages' main configs
    layers = [synth.tq_layer(5000, 1024, planes, group, seed=6600 + 10 * planes + group + i) for i in range(4)]
    check_int8_group(tern, layers, tern.ACT_INT8, nrows=256)
    (ys,), xbits = run_grouped(tern, layers, tern.ACT_BF16)
    for i, (lay, y, x) in enumerate(zip(layers, ys, xbits)):
        rows = sample_rows(lay.n, 128, i)
        w = oracle.dequantize("tq", lay.trits[:, rows], lay.group, scales=lay.scales[:, rows])
        check_bf16(y[rows], oracle.gemv_bf16(w, x)[0])
