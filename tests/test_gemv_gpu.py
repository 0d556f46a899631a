"""GPU parity of the C-ABI kernels against the CPU oracle (B200, sm_100a).

int8 activations: bit-exact. bf16 activations: the fp32 result is within
1e-3 of the fp64 reference relative to max(|y_ref|, 1e-2 * rms(y_ref)); the
bf16 output is exactly bf16_rn of the same kernel's fp32 result. Inputs come
from the seeded generators; expected values from the oracle only.
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


def x_dev(xbits):
    return dev(np.ascontiguousarray(xbits).view(np.int16))


def run_int8(tern, layer, xbits, use_ws=True, out=1, pdl=False):
    """Quantise x on the GPU, run the GEMV/batched GEMV; returns (y, xq, sx)."""
    d, buf = tern.pack_layer(layer, flags=tern.F_PDL if pdl else 0)
    m, k = xbits.shape
    pk = dev(buf)
    xd = x_dev(xbits)
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    tern.quantize_act(xd, xq, sx)
    y = torch.empty((m, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = None
    if use_ws:
        ws = torch.zeros(max(16, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda")
    tern.gemm_batched(d, pk, m, tern.ACT_INT8, xq, sx, out, y, ws)
    torch.cuda.synchronize()
    y1 = y.cpu().numpy()
    if ws is not None:
        # the same workspace again: its arrival counters must have been reset
        y.fill_(0)
        tern.gemm_batched(d, pk, m, tern.ACT_INT8, xq, sx, out, y, ws)
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().numpy().view(np.uint32), y1.view(np.uint32))
    assert tern.device_error() == tern.OK
    return y1, xq.cpu().numpy(), sx.cpu().numpy()


def run_bf16(tern, layer, xbits, out, use_ws=True):
    d, buf = tern.pack_layer(layer)
    pk = dev(buf)
    xd = x_dev(xbits)
    m = xbits.shape[0]
    y = torch.empty((m, layer.n), dtype=torch.float32 if out == tern.OUT_F32 else torch.int16, device="cuda")
    ws = torch.zeros(max(16, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda") if use_ws else None
    tern.gemm_batched(d, pk, m, tern.ACT_BF16, xd, None, out, y, ws)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    return y.cpu().numpy()


def check_bf16(y32, yref):
    floor = 1e-2 * np.sqrt(np.mean(yref ** 2))
    err = np.abs(y32.astype(np.float64) - yref) / np.maximum(np.abs(yref), floor)
    assert err.max() <= BF16_TOL, f"max rel err {err.max():.3g}"
    return err.max()


# ---------------------------------------------------------------- quantiser
@pytest.mark.parametrize("m,k", [(1, 1024), (3, 2560), (5, 6912), (2, 7)])
def test_quantize_bit_exact(tern, m, k):
    x = synth.draw_x_bf16(77 + k, m, k)
    if m >= 3:
        x[1] = 0                                    # all-zero token
        x[2, :4] = synth.f32_to_bf16_bits(np.array([2.0, 1.0, -1.0, 0.5], np.float32))
        x[2, 4:] = 0                                # exact .5 ties after scaling
    xd = x_dev(x)
    xq = torch.empty((m, k), dtype=torch.int8, device="cuda")
    sx = torch.empty((m,), dtype=torch.float32, device="cuda")
    tern.quantize_act(xd, xq, sx)
    q_ref, s_ref = oracle.quantize_act(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_tiny_and_subnormal_tokens(tern):
    """Token 0: absmax 2^-126, below 127 / FLT_MAX, so 127 / absmax overflows to
    +inf; its non-zero values (one of them a bf16 subnormal) quantise to +-127 and
    its zeros to 0. Token 1: absmax 1 with bf16-subnormal values beside it, which
    quantise to 0. Checked against the oracle for the quantiser and for the GEMV
    that quantises inside the kernel."""
    a = np.float32(2.0 ** -126)
    sub = np.float32(2.0 ** -130)                   # bf16 subnormal
    t0 = [a, 0.0, -a / 4, sub, -sub, 0.0, a, -a] + [0.0] * 8
    t1 = [1.0, sub, -sub, 2.0 ** -127, 0.5, -0.25, 0.0, -1.0] + [0.0] * 8
    x = synth.f32_to_bf16_bits(np.array([t0, t1], np.float32))
    xq = torch.empty((2, 16), dtype=torch.int8, device="cuda")
    sx = torch.empty((2,), dtype=torch.float32, device="cuda")
    tern.quantize_act(x_dev(x), xq, sx)
    q_ref, s_ref = oracle.quantize_act(x)
    assert q_ref[0, :8].tolist() == [127, 0, -127, 127, -127, 0, 127, -127]
    assert q_ref[1, 1:4].tolist() == [0, 0, 0]
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    lay = synth.bitnet_layer(64, 16, seed=5)
    d, buf = tern.pack_layer(lay)
    y = torch.empty((2, lay.n), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, tern.workspace_size(d, 2)), dtype=torch.uint8, device="cuda")
    tern.gemm_batched(d, dev(buf), 2, tern.ACT_BF16_Q8, x_dev(x), None, tern.OUT_F32, y, ws)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    y_ref = oracle.gemv_bitnet_int8(lay.trits, q_ref, s_ref, lay.tensor_scale)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y_ref.view(np.uint32))
    for i in range(2):                              # one token at a time: the single-token kernels
        y1 = torch.empty((1, lay.n), dtype=torch.float32, device="cuda")
        tern.gemv(d, dev(buf), tern.ACT_BF16_Q8, x_dev(x[i:i + 1]), None, tern.OUT_F32, y1, ws)
        torch.cuda.synchronize()
        assert np.array_equal(y1.cpu().numpy()[0].view(np.uint32), y_ref[i].view(np.uint32))


# ---------------------------------------------------------- BitNet int8 path
def bitnet_check(tern, layer, m=1, **kw):
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    y, xq, sx = run_int8(tern, layer, x, **kw)
    q_ref, s_ref = oracle.quantize_act(x)
    assert np.array_equal(xq, q_ref) and np.array_equal(sx, s_ref)
    y_ref = oracle.gemv_bitnet_int8(layer.trits, q_ref, s_ref, layer.tensor_scale)
    assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32)), \
        f"mismatch at {np.argwhere(y != y_ref)[:5]}"


def test_single_gemv_512x1024_bit_exact(tern):
    bitnet_check(tern, synth.single_gemv_layer())
    bitnet_check(tern, synth.single_gemv_layer(), use_ws=False)


@pytest.mark.parametrize("shape", synth.BITNET_2B_SHAPES, ids=[s[0] for s in synth.BITNET_2B_SHAPES])
def test_bitnet_2b_layer_shapes_bit_exact(tern, shape):
    name, n, k = shape
    layer = synth.bitnet_layer(n, k, synth.bitnet_layer_set_seed(0, [s[0] for s in synth.BITNET_2B_SHAPES].index(name)))
    bitnet_check(tern, layer)
    bitnet_check(tern, layer, pdl=True)


@pytest.mark.parametrize("n,k", [(1, 1), (37, 100), (33, 64), (300, 1000), (31, 6912), (4097, 129)])
def test_bitnet_ragged_shapes(tern, n, k):
    lay = synth.bitnet_layer(n, k, seed=n * 7 + k)
    bitnet_check(tern, lay)
    bitnet_check(tern, lay, use_ws=False)


@pytest.mark.parametrize("m", [2, 4, 5, 16, 21])
def test_bitnet_batched_bit_exact(tern, m):
    bitnet_check(tern, synth.bitnet_layer(640, 2560, seed=9), m=m)


def test_bitnet_zero_activation(tern):
    lay = synth.bitnet_layer(96, 256, seed=4)
    x = np.zeros((1, 256), np.uint16)
    y, _, _ = run_int8(tern, lay, x)
    assert not y.any() and not np.signbit(y).any()


def test_bitnet_deterministic(tern):
    lay = synth.bitnet_layer(2560, 6912, seed=12)
    x = synth.draw_x_bf16(12, 1, 6912)
    y1, _, _ = run_int8(tern, lay, x)
    y2, _, _ = run_int8(tern, lay, x)
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))


# ------------------------------------------------------------- TQ int8 path
def tq_int8_check(tern, layer, m, rows=None):
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    y, xq, sx = run_int8(tern, layer, x)
    q_ref, s_ref = oracle.quantize_act(x)
    assert np.array_equal(xq, q_ref)
    r = slice(None) if rows is None else rows
    y_ref = oracle.gemv_tq_int8(layer.trits[:, r], layer.scales[:, r], layer.group, q_ref, s_ref)
    assert np.array_equal(y[:, r].view(np.uint32), y_ref.view(np.uint32))


@pytest.mark.parametrize("m", [1, 4, 16, 3])
def test_tq2p_g32_int8_bit_exact(tern, m):
    tq_int8_check(tern, synth.tq_layer(300, 1024, 2, 32, seed=40 + m), m)


@pytest.mark.parametrize("shape", synth.PREFILL_SHAPES, ids=[s[0] for s in synth.PREFILL_SHAPES])
@pytest.mark.parametrize("m", [1, 4])
def test_tq2p_prefill_shapes_gemv_bit_exact(tern, shape, m):
    name, n, k = shape
    lay = synth.tq_layer(n, k, 2, 32, seed=400 + [s[0] for s in synth.PREFILL_SHAPES].index(name))
    rows = np.sort(np.random.default_rng(0).choice(n, 512, replace=False))
    tq_int8_check(tern, lay, m, rows=rows)


def test_tq3p_g256_int8_bit_exact(tern):
    tq_int8_check(tern, synth.tq_layer(1024, 4096, 3, 256, seed=7), 1)


# ------------------------------------------------------------- TQ bf16 path
def tq_bf16_check(tern, layer, rows=None, use_ws=True):
    x = synth.draw_x_bf16(layer.seed, 1, layer.k)
    y32 = run_bf16(tern, layer, x, tern.OUT_F32, use_ws)
    y16 = run_bf16(tern, layer, x, tern.OUT_BF16, use_ws)
    r = slice(None) if rows is None else rows
    w = oracle.dequantize("tq", layer.trits[:, r], layer.group, scales=layer.scales[:, r])
    yref = oracle.gemv_bf16(w, x)[0]
    err = check_bf16(y32[0, r], yref)
    # bf16 output = round-to-nearest-even of the fp32 result of the same kernel
    assert np.array_equal(y16.view(np.uint16), synth.f32_to_bf16_bits(y32))
    return err


@pytest.mark.parametrize("shape", synth.LLAMA_8B_SHAPES, ids=[s[0] for s in synth.LLAMA_8B_SHAPES])
def test_tq3p_llama_shapes_bf16(tern, shape):
    name, n, k = shape
    lay = synth.tq_layer(n, k, 3, 256, seed=200 + [s[0] for s in synth.LLAMA_8B_SHAPES].index(name))
    rows = np.sort(np.random.default_rng(1).choice(n, min(n, 384), replace=False))
    tq_bf16_check(tern, lay, rows=rows)


TQ_VARIANTS = [(p, g) for p in (1, 2, 3, 4) for g in (32, 64, 128, 256)]


@pytest.mark.parametrize("planes,group", TQ_VARIANTS)
def test_tq_bf16_variants(tern, planes, group):
    # sasori's K = 1..4 planes at every group size it names (README, "K and g")
    lay = synth.tq_layer(200, 1024, planes, group, seed=planes * 100 + group)
    tq_bf16_check(tern, lay)
    tq_bf16_check(tern, lay, use_ws=False)


@pytest.mark.parametrize("planes,group", TQ_VARIANTS)
def test_tq_int8_variants(tern, planes, group):
    tq_int8_check(tern, synth.tq_layer(200, 1024, planes, group, seed=planes * 100 + group + 1), 1)


def test_tq_bf16_wide_dynamic_range(tern):
    lay = synth.tq_layer(64, 512, 3, 256, seed=3)
    x = synth.draw_x_bf16(3, 1, 512).copy()
    xf = synth.bf16_bits_to_f32(x)
    xf[0, :256] *= 1e-3                    # one group much smaller than the other
    xf[0, 300] = 40.0                      # one outlier
    x = synth.f32_to_bf16_bits(xf)
    y32 = run_bf16(tern, lay, x, tern.OUT_F32)
    yref = oracle.gemv_bf16(oracle.dequantize("tq", lay.trits, 256, scales=lay.scales), x)[0]
    check_bf16(y32[0], yref)


# ----------------------------------------- in-kernel per-token quantisation
def q8_check(tern, layer, m):
    x = synth.draw_x_bf16(layer.seed, m, layer.k)
    d, buf = tern.pack_layer(layer)
    pk = dev(buf)
    y = torch.empty((m, layer.n), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, tern.workspace_size(d, m)), dtype=torch.uint8, device="cuda")
    tern.gemm_batched(d, pk, m, tern.ACT_BF16_Q8, x_dev(x), None, tern.OUT_F32, y, ws)
    torch.cuda.synchronize()
    assert tern.device_error() == tern.OK
    q_ref, s_ref = oracle.quantize_act(x)
    if layer.fmt == "bitnet":
        y_ref = oracle.gemv_bitnet_int8(layer.trits, q_ref, s_ref, layer.tensor_scale)
    else:
        y_ref = oracle.gemv_tq_int8(layer.trits, layer.scales, layer.group, q_ref, s_ref)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), y_ref.view(np.uint32))


@pytest.mark.parametrize("shape", synth.BITNET_2B_SHAPES, ids=[s[0] for s in synth.BITNET_2B_SHAPES])
def test_bitnet_fused_quant_bit_exact(tern, shape):
    name, n, k = shape
    q8_check(tern, synth.bitnet_layer(n, k, 2000 + n + k), 1)


@pytest.mark.parametrize("m", [1, 3, 4, 6])
def test_fused_quant_batched_bit_exact(tern, m):
    q8_check(tern, synth.bitnet_layer(300, 1000, seed=m), m)
    q8_check(tern, synth.tq_layer(200, 1024, 2, 32, seed=m), m)
    if m == 1:  # several tokens: BitNet and TQ2P g32 only
        # groups of 64 and 128: a warp's 32 four-value words span two groups, or one
        q8_check(tern, synth.tq_layer(200, 1024, 3, 64, seed=10 + m), m)
        q8_check(tern, synth.tq_layer(150, 2048, 1, 128, seed=20 + m), m)


def test_single_gemv_fused_quant(tern):
    q8_check(tern, synth.single_gemv_layer(), 1)


# ------------------------------------------------------------ grouped launch
def test_grouped_qkv_matches_single(tern):
    descs, packs, xs, ys, refs = [], [], [], [], []
    for i, (name, n, k) in enumerate(synth.BITNET_2B_SHAPES[:3]):
        lay = synth.bitnet_layer(n, k, 3000 + i)
        d, buf = tern.pack_layer(lay)
        x = synth.draw_x_bf16(lay.seed, 1, k)
        q_ref, s_ref = oracle.quantize_act(x)
        refs.append(oracle.gemv_bitnet_int8(lay.trits, q_ref, s_ref, lay.tensor_scale)[0])
        descs.append(d)
        packs.append(dev(buf))
        xs.append(x_dev(x))
        ys.append(torch.empty(n, dtype=torch.float32, device="cuda"))
    tern.gemv_grouped(descs, packs, tern.ACT_BF16_Q8, xs, None, tern.OUT_F32, ys)
    torch.cuda.synchronize()
    for y, r in zip(ys, refs):
        assert np.array_equal(y.cpu().numpy().view(np.uint32), r.view(np.uint32))


def test_grouped_int8_and_bf16(tern):
    lays = [synth.tq_layer(n, 1024, 3, 256, seed=60 + n) for n in (96, 300, 33)]
    descs, packs, xs, xqs, sxs, ys, ys2 = [], [], [], [], [], [], []
    for lay in lays:
        d, buf = tern.pack_layer(lay)
        descs.append(d)
        packs.append(dev(buf))
        x = synth.draw_x_bf16(lay.seed, 1, lay.k)
        xs.append(x_dev(x))
        xq = torch.empty((1, lay.k), dtype=torch.int8, device="cuda")
        sx = torch.empty((1,), dtype=torch.float32, device="cuda")
        tern.quantize_act(xs[-1].view(1, -1), xq, sx)
        xqs.append(xq)
        sxs.append(sx)
        ys.append(torch.empty(lay.n, dtype=torch.float32, device="cuda"))
        ys2.append(torch.empty(lay.n, dtype=torch.float32, device="cuda"))
    tern.gemv_grouped(descs, packs, tern.ACT_INT8, xqs, sxs, tern.OUT_F32, ys)
    tern.gemv_grouped(descs, packs, tern.ACT_BF16, xs, None, tern.OUT_F32, ys2)
    torch.cuda.synchronize()
    for lay, y, y2, x, in zip(lays, ys, ys2, xs):
        xb = x.cpu().numpy().view(np.uint16)[None]
        q_ref, s_ref = oracle.quantize_act(xb)
        r = oracle.gemv_tq_int8(lay.trits, lay.scales, 256, q_ref, s_ref)[0]
        assert np.array_equal(y.cpu().numpy().view(np.uint32), r.view(np.uint32))
        yref = oracle.gemv_bf16(oracle.dequantize("tq", lay.trits, 256, scales=lay.scales), xb)[0]
        check_bf16(y2.cpu().numpy(), yref)


# ------------------------------------------- very long K: workspace reduction
def test_long_k_workspace_path(tern):
    lay = synth.tq_layer(64, 1 << 21, 1, 256, seed=8)
    d = tern.desc_of(lay)
    assert tern.workspace_size(d, 1) > 0
    tq_int8_check(tern, lay, 1, rows=np.arange(0, 64, 7))
    with pytest.raises(tern.TernError) as ei:       # no workspace -> refused
        y = torch.empty(64, dtype=torch.float32, device="cuda")
        xq = torch.zeros(lay.k, dtype=torch.int8, device="cuda")
        sx = torch.ones(1, dtype=torch.float32, device="cuda")
        tern.gemv(d, dev(tern.pack_layer(lay)[1]), tern.ACT_INT8, xq, sx, tern.OUT_F32, y, None)
    assert ei.value.code == tern.ENOSPACE


# ------------------------------------------------- balanced ternary d = 3
def bt3_check(tern, layer, rows=None, use_ws=True):
    x = synth.draw_x_bf16(layer.seed, 1, layer.k)
    y32 = run_bf16(tern, layer, x, tern.OUT_F32, use_ws)
    y16 = run_bf16(tern, layer, x, tern.OUT_BF16, use_ws)
    r = slice(None) if rows is None else rows
    w = oracle.dequantize("bt3", layer.trits[:, r], 16, idx=layer.idx[r], codebook=layer.codebook)
    yref = oracle.gemv_bf16(w, x)[0]
    check_bf16(y32[0, r], yref)
    assert np.array_equal(y16.view(np.uint16), synth.f32_to_bf16_bits(y32))


@pytest.mark.parametrize("shape", synth.LLAMA_8B_SHAPES, ids=[s[0] for s in synth.LLAMA_8B_SHAPES])
def test_bt3_llama_shapes(tern, shape):
    name, n, k = shape
    lay = synth.bt3_layer(n, k, seed=300 + [s[0] for s in synth.LLAMA_8B_SHAPES].index(name))
    rows = np.sort(np.random.default_rng(2).choice(n, min(n, 384), replace=False))
    bt3_check(tern, lay, rows=rows)


@pytest.mark.parametrize("n,k", [(1, 16), (45, 96), (32, 160), (70, 4096), (300, 1040)])
def test_bt3_ragged(tern, n, k):
    lay = synth.bt3_layer(n, k, seed=n * 3 + k)
    bt3_check(tern, lay)
    bt3_check(tern, lay, use_ws=False)


def test_bt3_codebook_extremes(tern):
    lay = synth.bt3_layer(64, 320, seed=77)
    lay.idx[:32] = 0
    lay.idx[32:] = 26
    bt3_check(tern, lay)


def test_bt3_grouped(tern):
    lays = [synth.bt3_layer(n, 1024, seed=90 + n) for n in (64, 200, 33)]
    descs, packs, xs, ys, xbits = [], [], [], [], []
    for lay in lays:
        d, buf = tern.pack_layer(lay)
        descs.append(d)
        packs.append(dev(buf))
        xb = synth.draw_x_bf16(lay.seed, 1, lay.k)
        xbits.append(xb)
        xs.append(x_dev(xb))
        ys.append(torch.empty(lay.n, dtype=torch.float32, device="cuda"))
    tern.gemv_grouped(descs, packs, tern.ACT_BF16, xs, None, tern.OUT_F32, ys)
    torch.cuda.synchronize()
    for lay, y, xb in zip(lays, ys, xbits):
        w = oracle.dequantize("bt3", lay.trits, 16, idx=lay.idx, codebook=lay.codebook)
        check_bf16(y.cpu().numpy(), oracle.gemv_bf16(w, xb)[0])
