"""GPU parity of several tokens with bf16 activations (a8 for the bf16 formats).

Balanced ternary of depth 2, 3 and 4 reads its weights once for up to eight
tokens (each column's levels decoded once, dotted with every token's image);
TQ planes with bf16 activations run one token per pass of the row-group
kernel. Every token's fp32 result is within the bf16 tolerance of the fp64
oracle, and its bf16 output is bf16_rn of the same call's fp32 result.
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


def run(tern, layer, x, out, use_ws=True):
    d, buf = tern.pack_layer(layer)
    m = x.shape[0]
    y = torch.empty((m, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = torch.zeros(max(16, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda") if use_ws else None
    tern.gemm_batched(d, dev(buf), m, tern.ACT_BF16, dev(x.view(np.int16)), None, out, y, ws)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    return y.cpu().numpy()


def check(tern, layer, m, rows=None, use_ws=True):
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    y32 = run(tern, layer, x, tern.OUT_F32, use_ws)
    y16 = run(tern, layer, x, tern.OUT_BF16, use_ws)
    r = slice(None) if rows is None else rows
    if layer.fmt == "bt3":
        w = oracle.dequantize("bt3", layer.trits[:, r], 16, idx=layer.idx[r], codebook=layer.codebook)
    else:
        w = oracle.dequantize("tq", layer.trits[:, r], layer.group, scales=layer.scales[:, r])
    yref = oracle.gemv_bf16(w, x)
    for t in range(m):
        floor = 1e-2 * np.sqrt(np.mean(yref[t] ** 2))
        err = np.abs(y32[t, r].astype(np.float64) - yref[t]) / np.maximum(np.abs(yref[t]), floor)
        assert err.max() <= BF16_TOL, (t, err.max())
    assert np.array_equal(y16.view(np.uint16), synth.f32_to_bf16_bits(y32))


@pytest.mark.parametrize("depth", [2, 3, 4])
@pytest.mark.parametrize("m", [2, 3, 5, 8, 11])
def test_bt_several_tokens(tern, depth, m):
    lay = synth.bt3_layer(96, 1040, seed=7 * m + depth, depth=depth)
    check(tern, lay, m)


@pytest.mark.parametrize("m", [2, 4, 8])
def test_bt3_several_tokens_llama_shapes(tern, m):
    rng = np.random.default_rng(m)
    for si, (name, n, k) in enumerate(synth.LLAMA_8B_SHAPES):
        if name not in ("q_proj", "k_proj", "down_proj"):
            continue
        lay = synth.bt3_layer(n, k, seed=300 + si, name=name)
        rows = np.sort(rng.choice(n, min(n, 256), replace=False))
        check(tern, lay, m, rows=rows)


def test_bt3_several_tokens_match_single_calls_closely(tern):
    # each token of a batched call against the same token alone (different kernels and
    # summation orders, both within the tolerance of the oracle: compared here to 1e-5)
    lay = synth.bt3_layer(512, 4096, seed=41)
    x = synth.draw_x_bf16(lay.seed, 4, lay.k)
    yb = run(tern, lay, x, tern.OUT_F32)
    for t in range(4):
        y1 = run(tern, lay, x[t:t + 1], tern.OUT_F32)
        scale = np.sqrt(np.mean(y1 ** 2))
        assert np.abs(yb[t] - y1[0]).max() <= 1e-5 * scale


@pytest.mark.parametrize("planes,group,m", [(3, 256, 2), (3, 256, 4), (2, 32, 3), (1, 64, 5)])
def test_tq_bf16_several_tokens(tern, planes, group, m):
    lay = synth.tq_layer(200, 1024, planes, group, seed=planes * 10 + m)
    check(tern, lay, m)


def test_tq3p_bf16_several_tokens_llama_gate(tern):
    name, n, k = synth.LLAMA_8B_SHAPES[4]
    lay = synth.tq_layer(n, k, 3, 256, seed=204, name=name)
    rows = np.sort(np.random.default_rng(2).choice(n, 256, replace=False))
    check(tern, lay, 3, rows=rows)
