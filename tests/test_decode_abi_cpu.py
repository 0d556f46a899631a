"""Host-side checks of the decode-step and fit entry points (no GPU needed: every
case is refused before anything touches a device)."""
import ctypes

import numpy as np
import pytest

from packed_ternary_weight_b200 import tern


def model(**kw):
    a = dict(layers=2, hidden=256, inter=512, heads=4, kv_heads=2, head_dim=128, max_pos=8, eps=1e-5)
    a.update(kw)
    n = a["layers"] * 7
    ptrs = (ctypes.c_void_p * n)(*([0x1000] * n))
    m = tern.DecodeModelC(a["layers"], a["hidden"], a["inter"], a["heads"], a["kv_heads"], a["head_dim"],
                          a["max_pos"], a["eps"], ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p)),
                          0x2000, 0x3000, 0x4000, 0x5000)
    return m, ptrs


def step(m, pos=0, first=0, last=9, attn=None):
    return tern.lib.tern_decode_step(ctypes.byref(m), pos, ctypes.c_void_p(0x6000), ctypes.c_void_p(0x7000), first, last,
                                     attn, None, ctypes.c_void_p(0x8000), 1 << 20, None)


@pytest.mark.parametrize("bad", [dict(layers=0), dict(layers=65), dict(head_dim=64), dict(hidden=100),
                                 dict(inter=96), dict(heads=5, kv_heads=2), dict(heads=20, kv_heads=2),
                                 dict(kv_heads=17, heads=17), dict(hidden=20480), dict(max_pos=0),
                                 dict(eps=float("nan")), dict(eps=-1.0)])
def test_decode_model_refused(bad):
    m, keep = model(**bad)
    size = ctypes.c_size_t()
    assert tern.lib.tern_decode_workspace_size(ctypes.byref(m), ctypes.byref(size)) == tern.EINVAL
    assert step(m) == tern.EINVAL


def test_decode_stage_ranges_refused():
    m, keep = model()
    for kw in (dict(pos=-1), dict(pos=8), dict(first=3, last=2), dict(last=10), dict(first=1, last=2),
               dict(first=4, last=4), dict(first=2, last=4), dict(first=-1)):
        assert step(m, **kw) == tern.EINVAL, kw
    # starting at o_proj needs the attention output
    assert step(m, first=2, last=4, attn=None) == tern.EINVAL


def test_decode_missing_buffers_refused():
    m, keep = model()
    keep[3] = None                                     # a missing packed buffer
    assert step(m) == tern.EINVAL
    m2, keep2 = model()
    m2.d_gains = None
    assert step(m2) == tern.EINVAL


def test_rope_table_values_and_checks():
    t = tern.decode_rope_table(3, 128)
    assert t.shape == (3, 64, 2) and t.dtype == np.float32
    assert np.all(t[0, :, 0] == 1) and np.all(t[0, :, 1] == 0)
    assert t[1, 0, 0] == np.float32(np.cos(1.0)) and t[2, 0, 1] == np.float32(np.sin(2.0))
    out = np.empty(16, np.float32)
    for args in ((0, 128, 5e5), (4, 127, 5e5), (4, 128, 0.5)):
        assert tern.lib.tern_decode_rope_table(*args, out.ctypes.data_as(ctypes.c_void_p)) == tern.EINVAL


def test_fit_arguments_refused():
    p = ctypes.c_void_p(0x1000)
    for args in ((64, 256, 0, 64), (64, 256, 5, 64), (64, 256, 3, 48), (64, 250, 3, 64), (0, 256, 3, 64),
                 (64, 256, 3, 512)):
        assert tern.lib.tern_fit_tq(p, *args, p, p, None) == tern.EINVAL, args
    for args in ((64, 250, 3), (64, 256, 1), (64, 256, 5), (0, 256, 3)):
        assert tern.lib.tern_fit_bt(p, *args, p, p, p, None) == tern.EINVAL, args
