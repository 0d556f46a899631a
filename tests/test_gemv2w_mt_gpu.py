"""GPU parity of batched decode with a few tokens (M = 2..15) on the
one-CTA-per-SM CUDA-core kernel: every packed word is decoded once for up to
eight tokens, and rows of tiles shared between warps are summed with
shared-memory int64 atomics. Calls without a workspace on layers with at least
half a row tile per SM (2,368 rows) take this path (with a workspace, a few
tokens go to the tensor cores). int8 activations (given, or quantised in the
kernel from bf16): bit-exact against the oracle's exact integer rule.
"""
import numpy as np
import pytest

import oracle
from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tern():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from packed_ternary_weight_b200 import tern as t
    return t


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(tern, layer, x, act, out, use_ws=False):
    """Batched call through the C ABI, twice (the second result must be identical)."""
    d, buf = tern.pack_layer(layer)
    m, k = x.shape
    pk = dev(buf)
    if act == tern.ACT_INT8:
        xq, sx = oracle.quantize_act(x)
        xin, sin = dev(xq), dev(sx)
    else:
        xin, sin = dev(x.view(np.int16)), None
    y = torch.empty((m, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = torch.zeros(max(256, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda") if use_ws else None
    tern.gemm_batched(d, pk, m, act, xin, sin, out, y, ws)
    torch.cuda.synchronize()
    y1 = y.cpu().numpy().copy()
    y.fill_(0)
    tern.gemm_batched(d, pk, m, act, xin, sin, out, y, ws)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().view(np.uint16), y1.view(np.uint16)), "second call differs"
    assert tern.device_error() == tern.OK
    return y1


def expect(layer, x, rows):
    xq, sx = oracle.quantize_act(x)
    if layer.fmt == "tq":
        return oracle.gemv_tq_int8(layer.trits[:, rows], layer.scales[:, rows], layer.group, xq, sx)
    return oracle.gemv_bitnet_int8(layer.trits[:, rows], xq, sx, layer.tensor_scale)


def check(tern, layer, m, act=None, out=None, rows=None, use_ws=False):
    act = tern.ACT_INT8 if act is None else act
    out = tern.OUT_F32 if out is None else out
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    y = run(tern, layer, x, act, out, use_ws)
    r = np.arange(layer.n) if rows is None else rows
    ref = expect(layer, x, r)
    got = y[:, r]
    if out == tern.OUT_BF16:
        want = oracle.round_bf16(ref).astype(np.float32).view(np.uint32) >> 16
        assert np.array_equal(got.view(np.uint16).astype(np.uint32), want), "bf16 output differs"
    else:
        bad = np.argwhere(got.view(np.uint32) != ref.view(np.uint32))
        assert bad.size == 0, f"{len(bad)} mismatches, first {bad[:4].tolist()}"


@pytest.mark.parametrize("m", [2, 3, 4, 5, 8, 9, 15])
def test_tq2p_g32_tokens_bit_exact(tern, m):
    check(tern, synth.tq_layer(5000, 1024, 2, 32, seed=700 + m), m)


@pytest.mark.parametrize("m", [2, 4, 7, 8, 11])
def test_bitnet_tokens_bit_exact(tern, m):
    check(tern, synth.bitnet_layer(6000, 2560, seed=720 + m), m)


@pytest.mark.parametrize("planes,group,m", [(1, 256, 4), (2, 256, 6), (3, 256, 4), (4, 256, 3), (4, 256, 8),
                                            (3, 64, 5)])
def test_tq_variants_tokens_bit_exact(tern, planes, group, m):
    check(tern, synth.tq_layer(4800, 1024, planes, group, seed=740 + 10 * planes + m), m)


@pytest.mark.parametrize("n,k,m", [(4801, 1000, 4), (2400, 4096, 3), (2368, 320, 6), (8191, 192, 8)])
def test_ragged_tokens_bit_exact(tern, n, k, m):
    check(tern, synth.bitnet_layer(n, k, seed=n + k), m)
    if k % 64 == 0:
        check(tern, synth.tq_layer(n, k, 2, 32, seed=n + k + 1), m)


def test_whole_tiles_in_one_warp(tern):
    # many short rows per SM: some warps' ranges hold whole tiles, which they
    # finish without the shared-memory sums
    check(tern, synth.bitnet_layer(131072, 64, seed=760), 4)
    check(tern, synth.tq_layer(65536, 128, 2, 32, seed=761), 5)


@pytest.mark.parametrize("m", [3, 6])
def test_fused_quant_tokens_bit_exact(tern, m):
    check(tern, synth.bitnet_layer(5000, 1024, seed=770 + m), m, act=tern.ACT_BF16_Q8)
    check(tern, synth.tq_layer(5000, 1024, 2, 32, seed=780 + m), m, act=tern.ACT_BF16_Q8)


def test_bf16_out(tern):
    check(tern, synth.tq_layer(5000, 1024, 2, 32, seed=790), 4, out=tern.OUT_BF16)
    check(tern, synth.bitnet_layer(5000, 2048, seed=791), 7, out=tern.OUT_BF16)


@pytest.mark.parametrize("shape", synth.PREFILL_SHAPES, ids=[s[0] for s in synth.PREFILL_SHAPES])
@pytest.mark.parametrize("m", [4, 8])
def test_prefill_shapes_tokens_bit_exact(tern, shape, m):
    name, n, k = shape
    lay = synth.tq_layer(n, k, 2, 32, seed=400 + [s[0] for s in synth.PREFILL_SHAPES].index(name))
    rows = np.unique(np.concatenate([np.random.default_rng(m).choice(n, 768, replace=False),
                                     [0, 31, 32, n - 33, n - 1]]))
    check(tern, lay, m, rows=rows)

