"""tern_gemv_noalloc: the GEMV for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (code running inside an allocator or a
framework that owns all device memory), so they cannot hand tern_gemv a
workspace. tern_gemv_noalloc keeps its scratch in a fixed device array of the
library instead. This checks, through the C ABI, that two calls in a row give
the same result as tern_gemv with a caller workspace (bit-exact on the int8
path, the bf16 tolerance of the other GPU tests on the bf16 path), and that a
layer needing more than the fixed scratch is refused.

Kept in its own file, collected last, so a run that stops at the first failure
has already run every other test.
"""
import numpy as np
import pytest

from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tern():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from packed_ternary_weight_b200 import tern as t
    return t


def _run_both(tern, lay, act, x, xq=None, sx=None):
    """tern_gemv with a caller workspace, then tern_gemv_noalloc twice; returns the three outputs."""
    d, buf = tern.pack_layer(lay)
    need = tern.workspace_size(d, 1)
    assert 0 < need <= (1 << 20)                           # this layer uses the scratch
    pk = torch.from_numpy(buf).cuda()
    xin = xq if act == tern.ACT_INT8 else x
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y_ref = torch.empty(lay.n, dtype=torch.float32, device="cuda")
    tern.gemv(d, pk, act, xin, sx, tern.OUT_F32, y_ref, ws)
    outs = []
    for _ in range(2):
        y = torch.full((lay.n,), float("nan"), dtype=torch.float32, device="cuda")
        tern.gemv_noalloc(d, pk, act, xin, sx, tern.OUT_F32, y)
        torch.cuda.synchronize()
        outs.append(y)
    assert tern.device_error() == tern.OK
    return y_ref, outs


def test_noalloc_matches_gemv_int8_two_calls(tern):
    # a very long K splits beyond one thread-block cluster and needs the scratch
    lay = synth.tq_layer(64, 1 << 21, 1, 256, seed=5)
    x = torch.from_numpy(synth.draw_x_bf16(5, 1, lay.k).view(np.int16)).cuda()
    xq = torch.empty((1, lay.k), dtype=torch.int8, device="cuda")
    sx = torch.empty((1,), dtype=torch.float32, device="cuda")
    tern.quantize_act(x, xq, sx)
    y_ref, outs = _run_both(tern, lay, tern.ACT_INT8, x, xq, sx)
    for y in outs:
        assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32))


def test_noalloc_matches_gemv_bf16_two_calls(tern):
    lay = synth.tq_layer(64, 1 << 20, 1, 256, seed=6)
    x = torch.from_numpy(synth.draw_x_bf16(6, 1, lay.k).view(np.int16)).cuda()
    y_ref, outs = _run_both(tern, lay, tern.ACT_BF16, x)
    ref = y_ref.double()
    floor = 1e-2 * ref.pow(2).mean().sqrt()
    for y in outs:
        err = ((y.double() - ref).abs() / torch.maximum(ref.abs(), floor)).max().item()
        assert err <= 1e-3


def test_noalloc_rejects_layer_beyond_scratch(tern):
    d = tern.make_desc("tq", 16384, 1 << 20, 1, 16)        # K split 11 ways: 1.4 MB of partials
    assert tern.workspace_size(d, 1) > (1 << 20)
    y = torch.empty(16, dtype=torch.float32, device="cuda")
    x = torch.zeros(16, dtype=torch.int16, device="cuda")
    pk = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(tern.TernError) as ei:
        tern.gemv_noalloc(d, pk, tern.ACT_BF16, x, None, tern.OUT_F32, y)
    assert ei.value.code == tern.ENOSPACE
