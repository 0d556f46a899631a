"""GPU parity of balanced ternary at depth 2 and 4 (the card's rule at one trit
fewer or more per weight) on the row-group kernel: bf16 activations, fp32
accumulation, within the bf16 tolerance of the oracle's fp64 result; bf16
output equal to the rounding of the same call's fp32 result."""
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


def run(tern, layer, xbits, out, use_ws=True):
    d, buf = tern.pack_layer(layer)
    y = torch.empty((1, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = torch.zeros(max(16, tern.workspace_size(d, 1)), dtype=torch.uint8, device="cuda") if use_ws else None
    tern.gemm_batched(d, dev(buf), 1, tern.ACT_BF16, dev(xbits.view(np.int16)), None, out, y, ws)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    return y.cpu().numpy()


def check(tern, layer, rows=None, use_ws=True):
    x = synth.draw_x_bf16(layer.seed, 1, layer.k)
    y32 = run(tern, layer, x, tern.OUT_F32, use_ws)
    y16 = run(tern, layer, x, tern.OUT_BF16, use_ws)
    r = slice(None) if rows is None else rows
    w = oracle.dequantize("bt3", layer.trits[:, r], 16, idx=layer.idx[r], codebook=layer.codebook)
    yref = oracle.gemv_bf16(w, x)[0]
    floor = 1e-2 * np.sqrt(np.mean(yref ** 2))
    err = np.abs(y32[0, r].astype(np.float64) - yref) / np.maximum(np.abs(yref), floor)
    assert err.max() <= BF16_TOL, f"max rel err {err.max():.3g}"
    assert np.array_equal(y16.view(np.uint16), synth.f32_to_bf16_bits(y32))


@pytest.mark.parametrize("depth", [2, 4])
@pytest.mark.parametrize("n,k", [(1, 16), (45, 96), (32, 160), (70, 4096), (300, 1040)])
def test_bt_depth_ragged(tern, depth, n, k):
    lay = synth.bt3_layer(n, k, seed=n * 5 + k + depth, depth=depth)
    check(tern, lay)
    check(tern, lay, use_ws=False)


@pytest.mark.parametrize("depth", [2, 4])
@pytest.mark.parametrize("shape", synth.LLAMA_8B_SHAPES, ids=[s[0] for s in synth.LLAMA_8B_SHAPES])
def test_bt_depth_llama_shapes(tern, depth, shape):
    name, n, k = shape
    lay = synth.bt3_layer(n, k, seed=500 + 10 * depth + [s[0] for s in synth.LLAMA_8B_SHAPES].index(name),
                          depth=depth)
    rows = np.sort(np.random.default_rng(depth).choice(n, min(n, 384), replace=False))
    check(tern, lay, rows=rows)


@pytest.mark.parametrize("depth", [2, 4])
def test_bt_depth_codebook_extremes(tern, depth):
    lay = synth.bt3_layer(64, 320, seed=78 + depth, depth=depth)
    lay.idx[:32] = 0
    lay.idx[32:] = 26
    check(tern, lay)


@pytest.mark.parametrize("depth", [2, 4])
def test_bt_depth_grouped(tern, depth):
    lays = [synth.bt3_layer(n, 1024, seed=95 + n + depth, depth=depth) for n in (64, 200, 33)]
    descs, packs, xs, ys, xbits = [], [], [], [], []
    for lay in lays:
        d, buf = tern.pack_layer(lay)
        descs.append(d)
        packs.append(dev(buf))
        xb = synth.draw_x_bf16(lay.seed, 1, lay.k)
        xbits.append(xb)
        xs.append(dev(xb.view(np.int16)))
        ys.append(torch.empty(lay.n, dtype=torch.float32, device="cuda"))
    tern.gemv_grouped(descs, packs, tern.ACT_BF16, xs, None, tern.OUT_F32, ys)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    for lay, y, xb in zip(lays, ys, xbits):
        w = oracle.dequantize("bt3", lay.trits, 16, idx=lay.idx, codebook=lay.codebook)
        yref = oracle.gemv_bf16(w, xb)[0]
        floor = 1e-2 * np.sqrt(np.mean(yref ** 2))
        err = np.abs(y.cpu().numpy().astype(np.float64) - yref) / np.maximum(np.abs(yref), floor)
        assert err.max() <= BF16_TOL
