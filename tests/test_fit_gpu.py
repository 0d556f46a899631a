"""GPU parity of the dense -> ternary fits (tern_fit_tq, tern_fit_bt) against oracle/fit.py.

The fits are integer decisions and fp16 scales taken from fp64 arithmetic in
a fixed order, so the GPU's trits, scales and codebook indices must equal the
oracle's exactly. The fitted weights then go through the packer and the GEMV
and are checked against the oracle's GEMV of the oracle's fit.
"""
import numpy as np
import pytest

import oracle
from oracle import fit
from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tern():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from packed_ternary_weight_b200 import tern as t
    return t


def weights(seed, n, k, heavy=False):
    g = np.random.default_rng(seed)
    w = g.standard_t(3, (n, k)) if heavy else g.standard_normal((n, k))
    return (w * 0.02).astype(np.float32)


def gpu_fit_tq(tern, w, planes, group):
    n, k = w.shape
    t = torch.empty((planes, n, k), dtype=torch.int8, device="cuda")
    s = torch.empty((planes, n, k // group), dtype=torch.int16, device="cuda")
    tern.fit_tq(torch.from_numpy(w).cuda(), planes, group, t, s)
    torch.cuda.synchronize()
    return t.cpu().numpy(), s.cpu().numpy().view(np.uint16)


def gpu_fit_bt(tern, w, depth):
    n, k = w.shape
    t = torch.empty((depth, n, k), dtype=torch.int8, device="cuda")
    ix = torch.empty((n, k // 16), dtype=torch.uint8, device="cuda")
    tern.fit_bt(torch.from_numpy(w).cuda(), depth, torch.from_numpy(synth.codebook27()).cuda(), t, ix)
    torch.cuda.synchronize()
    return t.cpu().numpy(), ix.cpu().numpy()


@pytest.mark.parametrize("planes,group", [(1, 256), (2, 32), (3, 256), (3, 64), (4, 128), (2, 16)])
def test_fit_tq_matches_oracle(tern, planes, group):
    w = weights(planes * 100 + group, 70, 512)
    w[3] = 0                                            # an all-zero row
    t, s = gpu_fit_tq(tern, w, planes, group)
    rt, rs = fit.fit_tq(w, planes, group)
    assert np.array_equal(t, rt)
    assert np.array_equal(s, rs.view(np.uint16))


@pytest.mark.parametrize("shape", [(128, 4096), (96, 14336)], ids=["rows_of_4096", "rows_of_14336"])
def test_fit_tq_llama_widths(tern, shape):
    w = weights(7, *shape, heavy=True)
    for planes, group in ((3, 256), (2, 32)):
        t, s = gpu_fit_tq(tern, w, planes, group)
        rt, rs = fit.fit_tq(w, planes, group)
        assert np.array_equal(t, rt) and np.array_equal(s, rs.view(np.uint16))


@pytest.mark.parametrize("depth", [2, 3, 4])
def test_fit_bt_matches_oracle(tern, depth):
    for seed, (n, k), heavy in ((1, (64, 256), False), (2, (48, 4096), True)):
        w = weights(seed * 10 + depth, n, k, heavy)
        w[0, :16] = 0                                   # an all-zero group
        t, ix = gpu_fit_bt(tern, w, depth)
        rt, rix = fit.fit_bt(w, synth.codebook27(), depth)
        assert np.array_equal(ix, rix)
        assert np.array_equal(t, rt)


def test_fitted_weights_through_pack_and_gemv(tern):
    # fit on the GPU -> pack on the host -> GEMV on the GPU, against the oracle's
    # GEMV of the oracle's fit (int8 activations: bit-exact)
    n, k = 300, 1024
    w = weights(21, n, k)
    t, s = gpu_fit_tq(tern, w, 3, 64)
    d = tern.make_desc("tq", n, k, 3, 64)
    buf = tern.pack(d, t, s.view(np.float16))
    x = synth.draw_x_bf16(21, 1, k)
    q, sx = oracle.quantize_act(x)
    y = torch.empty((1, n), dtype=torch.float32, device="cuda")
    tern.gemv(d, torch.from_numpy(buf).cuda(), tern.ACT_INT8, torch.from_numpy(q).cuda(), torch.from_numpy(sx).cuda(),
              tern.OUT_F32, y, torch.zeros(max(16, tern.workspace_size(d, 1)), dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    rt, rs = fit.fit_tq(w, 3, 64)
    ref = oracle.gemv_tq_int8(rt, rs, 64, q, sx)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))
