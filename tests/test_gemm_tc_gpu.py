"""GPU parity of the batched tensor-core path (m >= 16 tokens, tcgen05 kind::i8).

The int8 path is bit-exact: every output equals the oracle's exact group-scaled
sum (an integer count of 2^-24 rounded once to fp32, times the token scale),
or for the single plane the exact integer sum times the layer scale, then the
token scale. Inputs come from the seeded generators; expected values from the
oracle only. The full-size prefill layers are checked on sampled rows.
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


def run(tern, layer, x, act, out=1, repeat=True):
    """Batched GEMM through the C ABI; the workspace is used twice to check that
    the call leaves its counters and partial sums at zero."""
    d, buf = tern.pack_layer(layer)
    m, k = x.shape
    pk = dev(buf)
    if act == tern.ACT_INT8:
        xq, sx = oracle.quantize_act(x)
        xin, sin = dev(xq), dev(sx)
    else:
        xin, sin = dev(x.view(np.int16)), None
    y = torch.empty((m, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = torch.zeros(max(256, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda")
    tern.gemm_batched(d, pk, m, act, xin, sin, out, y, ws)
    torch.cuda.synchronize()
    y1 = y.cpu().numpy().copy()
    if repeat:
        y.fill_(0)
        tern.gemm_batched(d, pk, m, act, xin, sin, out, y, ws)
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy().view(np.uint16), y1.view(np.uint16)), "second call differs"
    assert tern.device_error() == tern.OK
    return y1


def expect(layer, x, rows=None):
    xq, sx = oracle.quantize_act(x)
    r = slice(None) if rows is None else rows
    if layer.fmt == "tq":
        return oracle.gemv_tq_int8(layer.trits[:, r], layer.scales[:, r], layer.group, xq, sx)
    return oracle.gemv_bitnet_int8(layer.trits[:, r], xq, sx, layer.tensor_scale)


def check(tern, layer, m, act=None, rows=None, out=None):
    act = tern.ACT_INT8 if act is None else act
    out = tern.OUT_F32 if out is None else out
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    y = run(tern, layer, x, act, out)
    ref = expect(layer, x, rows)
    got = y if rows is None else y[:, rows]
    if out == tern.OUT_BF16:
        want = oracle.round_bf16(ref).astype(np.float32).view(np.uint32) >> 16
        assert np.array_equal(got.view(np.uint16).astype(np.uint32), want), "bf16 output differs"
    else:
        bad = np.argwhere(got.view(np.uint32) != ref.view(np.uint32))
        assert bad.size == 0, f"{len(bad)} mismatches, first {bad[:4].tolist()}"


@pytest.mark.parametrize("m", [9, 12, 15, 16, 17, 33, 64, 100, 256])
def test_tq2p_g32_small_bit_exact(tern, m):
    # from 9 tokens a call with a workspace runs on the tensor cores (padded to 16)
    check(tern, synth.tq_layer(300, 1024, 2, 32, seed=60 + m), m)


@pytest.mark.parametrize("planes,group", [(1, 16), (2, 64), (3, 128), (4, 256), (3, 32), (4, 16)])
def test_tq_variants_bit_exact(tern, planes, group):
    check(tern, synth.tq_layer(200, 768, planes, group, seed=planes * 7 + group), 40)


@pytest.mark.parametrize("n,k,m", [(1, 64, 16), (129, 320, 31), (257, 512, 48), (640, 2560, 16)])
def test_tq_ragged_shapes(tern, n, k, m):
    check(tern, synth.tq_layer(n, k, 2, 32, seed=n + k), m)


@pytest.mark.parametrize("m", [16, 300, 513])
def test_more_tokens_than_one_launch(tern, m):
    # beyond 256 tokens the host issues one launch per block of 256
    check(tern, synth.tq_layer(160, 512, 2, 32, seed=m), m)


@pytest.mark.parametrize("shape", synth.PREFILL_SHAPES, ids=[s[0] for s in synth.PREFILL_SHAPES])
@pytest.mark.parametrize("m", [16, 64, 256])
def test_tq2p_prefill_shapes_bit_exact(tern, shape, m):
    name, n, k = shape
    lay = synth.tq_layer(n, k, 2, 32, seed=400 + [s[0] for s in synth.PREFILL_SHAPES].index(name))
    rows = np.sort(np.random.default_rng(m).choice(n, 384, replace=False))
    check(tern, lay, m, rows=rows)


@pytest.mark.parametrize("big,digits", [(1.0, 4), (100.0, 5), (30000.0, 6), (1e-5, 3)])
def test_scale_digit_counts(tern, big, digits):
    # one group of every row gets a large scale, so the packed header's digit
    # count (base-128 digits of the largest |s| / 2^-24) covers 3 to 6 digits
    lay = synth.tq_layer(130, 512, 2, 16, seed=int(big) % 97 + 11)
    s = lay.scales.astype(np.float32)
    s[0, :, 3] = big
    s[1, ::3, 7] = -big / 3
    lay.scales = s.astype(np.float16)
    d, buf = tern.pack_layer(lay)
    if big >= 1.0:
        assert oracle.parse_header(buf)["scale_digits"] == digits
    check(tern, lay, 24)


def test_negative_and_subnormal_scales(tern):
    lay = synth.tq_layer(96, 256, 3, 32, seed=5)
    s = lay.scales.astype(np.float32)
    s[1] = -s[1]
    s[2, :, ::2] = 3e-7                              # fp16 subnormals
    lay.scales = s.astype(np.float16)
    check(tern, lay, 20)


@pytest.mark.parametrize("n,k", [(512, 1024), (45, 100), (2560, 6912)])
def test_bitnet_batched_tc_bit_exact(tern, n, k):
    lay = synth.bitnet_layer(n, k, seed=n + 3)
    rows = None if n < 1000 else np.sort(np.random.default_rng(1).choice(n, 256, replace=False))
    check(tern, lay, 32, rows=rows)


def test_fused_quantisation_tc(tern):
    lay = synth.tq_layer(256, 2048, 2, 32, seed=9)
    check(tern, lay, 48, act=tern.ACT_BF16_Q8)
    check(tern, synth.bitnet_layer(300, 640, seed=10), 20, act=tern.ACT_BF16_Q8)


def test_bf16_output_tc(tern):
    check(tern, synth.tq_layer(200, 512, 2, 32, seed=12), 32, out=tern.OUT_BF16)


def test_zero_tokens_tc(tern):
    lay = synth.tq_layer(128, 256, 2, 32, seed=13)
    x = synth.draw_x_bf16(lay.seed, 20, lay.k)
    x[3] = 0
    x[19] = 0
    y = run(tern, lay, x, tern.ACT_INT8)
    assert not y[3].any() and not y[19].any()
    assert np.array_equal(y.view(np.uint32), expect(lay, x).view(np.uint32))


def test_deterministic_tc(tern):
    lay = synth.tq_layer(14336 // 4, 4096, 2, 32, seed=14)
    x = synth.draw_x_bf16(lay.seed, 64, lay.k)
    y1 = run(tern, lay, x, tern.ACT_INT8, repeat=False)
    y2 = run(tern, lay, x, tern.ACT_INT8, repeat=False)
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))


@pytest.mark.parametrize("planes,group,m", [(2, 64, 4), (1, 128, 2), (4, 32, 7)])
def test_few_tokens_without_cuda_core_kernel(tern, planes, group, m):
    # plane counts and group sizes the several-token CUDA-core kernel is not built for: with a
    # workspace they run on the tensor path, padded to 16 tokens
    check(tern, synth.tq_layer(300, 1024, planes, group, seed=6700 + planes * 10 + group), m)
