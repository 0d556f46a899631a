"""ctypes binding of libtern.so: argument marshalling only.

Every step of the computation runs in the library's CUDA kernels (or, for
packing, its host C++ code). Importing this module fails loudly if the shared
library has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtern.so")

OK, EINVAL, EFORMAT, EALIGN, ENOSPACE, EUNSUPPORTED, ECUDA, ETIMEOUT = range(8)
FMT = {"bitnet": 1, "tq": 2, "bt3": 3}
ACT_INT8, ACT_BF16, ACT_BF16_Q8 = 1, 2, 3
OUT_F32, OUT_BF16 = 1, 2
F_PDL = 1


class TernError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libtern.so not built ({_LIB_PATH}); run python -m packed_ternary_weight_b200.build")
    return ctypes.CDLL(_LIB_PATH)


lib = _load()


class Desc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("n", ctypes.c_int32), ("k", ctypes.c_int32),
                ("planes", ctypes.c_int32), ("group", ctypes.c_int32), ("tensor_scale", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


_vp, _sz = ctypes.c_void_p, ctypes.c_size_t
lib.tern_status_string.restype = ctypes.c_char_p
lib.tern_status_string.argtypes = [ctypes.c_int]
lib.tern_packed_size.argtypes = [ctypes.POINTER(Desc), ctypes.POINTER(_sz)]
lib.tern_pack.argtypes = [ctypes.POINTER(Desc), _vp, _vp, _vp, _vp, _vp, _sz, ctypes.POINTER(_sz)]
lib.tern_workspace_size.argtypes = [ctypes.POINTER(Desc), ctypes.c_int32, ctypes.POINTER(_sz)]
lib.tern_quantize_act.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp]
lib.tern_gemv.argtypes = [ctypes.POINTER(Desc), _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp, _vp, _sz, _vp]
lib.tern_gemm_batched.argtypes = [ctypes.POINTER(Desc), _vp, ctypes.c_int32, ctypes.c_int, _vp, _vp, ctypes.c_int,
                                  _vp, _vp, _sz, _vp]
lib.tern_device_error.argtypes = [_vp]
lib.tern_gemv_noalloc.argtypes = [ctypes.POINTER(Desc), _vp, ctypes.c_int, _vp, _vp, ctypes.c_int, _vp, _vp]
lib.tern_stream_read.argtypes = [_vp, _sz, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                 ctypes.c_int32, _vp, _vp]
lib.tern_gemv_grouped.argtypes = [ctypes.c_int32, ctypes.POINTER(Desc), ctypes.POINTER(_vp), ctypes.c_int,
                                  ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.c_int, ctypes.POINTER(_vp), _vp]
lib.tern_selftest_wait.argtypes = [ctypes.c_uint64, _vp]
lib.tern_fit_tq.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp]
lib.tern_fit_bt.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp, _vp]


class DecodeModelC(ctypes.Structure):
    _fields_ = [("layers", ctypes.c_int32), ("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("max_pos", ctypes.c_int32), ("eps", ctypes.c_float), ("packed", ctypes.POINTER(_vp)),
                ("d_gains", _vp), ("d_kcache", _vp), ("d_vcache", _vp), ("d_rope", _vp)]


lib.tern_decode_rope_table.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_double, _vp]
lib.tern_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeModelC), ctypes.POINTER(_sz)]
lib.tern_decode_step.argtypes = [ctypes.POINTER(DecodeModelC), ctypes.c_int32, _vp, _vp, ctypes.c_int32,
                                 ctypes.c_int32, _vp, _vp, _vp, _sz, _vp]
for _f in (lib.tern_decode_rope_table, lib.tern_decode_workspace_size, lib.tern_decode_step):
    _f.restype = ctypes.c_int
for _f in (lib.tern_selftest_wait, lib.tern_fit_tq, lib.tern_fit_bt, lib.tern_packed_size, lib.tern_pack, lib.tern_workspace_size, lib.tern_quantize_act, lib.tern_gemv,
           lib.tern_gemm_batched, lib.tern_device_error, lib.tern_gemv_noalloc, lib.tern_gemv_grouped,
           lib.tern_stream_read):
    _f.restype = ctypes.c_int


def status_string(code: int) -> str:
    return lib.tern_status_string(code).decode()


def _check(code: int, what: str):
    if code != OK:
        raise TernError(code, what)


def make_desc(fmt: str, n: int, k: int, planes: int = 1, group: int = 0, tensor_scale: float = 0.0,
              flags: int = 0) -> Desc:
    return Desc(FMT[fmt], n, k, planes, group, tensor_scale, flags)


def desc_of(layer, flags: int = 0) -> Desc:
    """Descriptor of a synth.Layer (or anything with the same fields)."""
    return make_desc(layer.fmt, layer.n, layer.k, layer.planes, layer.group, layer.tensor_scale, flags)


def packed_size(desc: Desc) -> int:
    out = _sz()
    _check(lib.tern_packed_size(ctypes.byref(desc), ctypes.byref(out)), "tern_packed_size")
    return out.value


def _ptr(a):
    if a is None:
        return None
    if hasattr(a, "data_ptr"):
        return ctypes.c_void_p(a.data_ptr())
    return a.ctypes.data_as(ctypes.c_void_p)


def pack(desc: Desc, trits, scales_fp16=None, scale_idx=None, codebook=None) -> np.ndarray:
    """Pack logical weights (host numpy arrays) into a uint8 numpy buffer."""
    t = np.ascontiguousarray(trits, dtype=np.int8)
    s = None if scales_fp16 is None else np.ascontiguousarray(scales_fp16, dtype=np.float16).view(np.uint16)
    i = None if scale_idx is None else np.ascontiguousarray(scale_idx, dtype=np.uint8)
    c = None if codebook is None else np.ascontiguousarray(codebook, dtype=np.float32)
    size = packed_size(desc)
    out = np.empty(size, dtype=np.uint8)
    used = _sz()
    _check(lib.tern_pack(ctypes.byref(desc), _ptr(t), _ptr(s), _ptr(i), _ptr(c), _ptr(out), size,
                         ctypes.byref(used)), "tern_pack")
    return out


def pack_layer(layer, flags: int = 0):
    d = desc_of(layer, flags)
    return d, pack(d, layer.trits, layer.scales, layer.idx, layer.codebook)


def workspace_size(desc: Desc, m: int = 1) -> int:
    out = _sz()
    _check(lib.tern_workspace_size(ctypes.byref(desc), m, ctypes.byref(out)), "tern_workspace_size")
    return out.value


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def quantize_act(x_bf16, xq, xscale, stream=None):
    """x_bf16: device tensor [m][k] of bf16 (or int16/uint16 bits); xq int8 [m][k]; xscale float [m]."""
    m, k = x_bf16.shape
    _check(lib.tern_quantize_act(_ptr(x_bf16), m, k, _ptr(xq), _ptr(xscale), _stream(stream)), "tern_quantize_act")


def gemm_batched(desc: Desc, packed, m: int, act: int, x, xscale, out: int, y, ws=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.tern_gemm_batched(ctypes.byref(desc), _ptr(packed), m, act, _ptr(x), _ptr(xscale), out, _ptr(y),
                                 _ptr(ws), ws_bytes, _stream(stream)), "tern_gemm_batched")


def gemv(desc: Desc, packed, act: int, x, xscale, out: int, y, ws=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.tern_gemv(ctypes.byref(desc), _ptr(packed), act, _ptr(x), _ptr(xscale), out, _ptr(y), _ptr(ws),
                         ws_bytes, _stream(stream)), "tern_gemv")


class Grouped:
    """Marshalled arguments of tern_gemv_grouped, built once and launched many times."""

    def __init__(self, descs, packed, act: int, xs, xscales, out: int, ys):
        n = len(descs)
        self.count = n
        self.act, self.out = act, out
        self.descs = (Desc * n)(*descs)
        self.packed = (_vp * n)(*[p.data_ptr() for p in packed])
        self.xs = (_vp * n)(*[x.data_ptr() for x in xs])
        self.xscales = None if xscales is None else (_vp * n)(*[s.data_ptr() for s in xscales])
        self.ys = (_vp * n)(*[y.data_ptr() for y in ys])

    def launch(self, stream=None):
        _check(lib.tern_gemv_grouped(self.count, self.descs, self.packed, self.act, self.xs, self.xscales, self.out,
                                     self.ys, _stream(stream)), "tern_gemv_grouped")


def gemv_grouped(descs, packed, act: int, xs, xscales, out: int, ys, stream=None):
    Grouped(descs, packed, act, xs, xscales, out, ys).launch(stream)


def gemv_noalloc(desc: Desc, packed, act: int, x, xscale, out: int, y, stream=None):
    """tern_gemv with the library's fixed device scratch instead of a caller workspace."""
    _check(lib.tern_gemv_noalloc(ctypes.byref(desc), _ptr(packed), act, _ptr(x), _ptr(xscale), out, _ptr(y),
                                 _stream(stream)), "tern_gemv_noalloc")


def stream_read(src, mode: int, chunk: int, depth: int, ctas_per_sm: int, warps: int, sink, stream=None):
    """Read-ceiling kernel: stream all of `src` once with the given access shape."""
    _check(lib.tern_stream_read(_ptr(src), src.numel() * src.element_size(), mode, chunk, depth, ctas_per_sm, warps,
                                _ptr(sink), _stream(stream)), "tern_stream_read")


def device_error(stream=None) -> int:
    return lib.tern_device_error(_stream(stream))


def selftest_wait(limit_ns: int, stream=None):
    """Enqueue the failure-detection self-test: a bounded wait that expires after limit_ns."""
    _check(lib.tern_selftest_wait(limit_ns, _stream(stream)), "tern_selftest_wait")


def decode_rope_table(max_pos: int, head_dim: int = 128, theta: float = 500000.0) -> np.ndarray:
    """cos/sin table [max_pos][head_dim/2][2] (fp32) computed by the library."""
    out = np.empty((max_pos, head_dim // 2, 2), dtype=np.float32)
    _check(lib.tern_decode_rope_table(max_pos, head_dim, theta, _ptr(out)), "tern_decode_rope_table")
    return out


class DecodeModel:
    """Marshalled tern_decode_model: device buffers are caller-owned tensors; the host array of
    packed-buffer pointers lives as long as this object."""

    def __init__(self, packed, gains, kcache, vcache, rope, hidden: int, inter: int, heads: int, kv_heads: int,
                 max_pos: int, eps: float = 1e-5, head_dim: int = 128):
        n = len(packed)
        assert n % 7 == 0
        self._keep = (packed, gains, kcache, vcache, rope)
        self._ptrs = (_vp * n)(*[p.data_ptr() for p in packed])
        self.c = DecodeModelC(n // 7, hidden, inter, heads, kv_heads, head_dim, max_pos, eps,
                              ctypes.cast(self._ptrs, ctypes.POINTER(_vp)), gains.data_ptr(), kcache.data_ptr(),
                              vcache.data_ptr(), rope.data_ptr())

    def workspace_size(self) -> int:
        out = _sz()
        _check(lib.tern_decode_workspace_size(ctypes.byref(self.c), ctypes.byref(out)), "tern_decode_workspace_size")
        return out.value

    def step(self, pos: int, h_in, h_out, ws, first: int = 0, last: int | None = None, attn_in=None, trace=None,
             stream=None):
        last = 5 * self.c.layers - 1 if last is None else last
        _check(lib.tern_decode_step(ctypes.byref(self.c), pos, _ptr(h_in), _ptr(h_out), first, last, _ptr(attn_in),
                                    _ptr(trace), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
               "tern_decode_step")


def fit_tq(w, planes: int, group: int, trits, scales, stream=None):
    """Fit fp32 device weights [n][k] into TQ planes: trits int8 [planes][n][k], scales fp16 [planes][n][k/group]."""
    n, k = w.shape
    _check(lib.tern_fit_tq(_ptr(w), n, k, planes, group, _ptr(trits), _ptr(scales), _stream(stream)), "tern_fit_tq")


def fit_bt(w, depth: int, codebook, trits, idx, stream=None):
    """Fit fp32 device weights [n][k] into balanced ternary: trits int8 [depth][n][k], idx uint8 [n][k/16]."""
    n, k = w.shape
    _check(lib.tern_fit_bt(_ptr(w), n, k, depth, _ptr(codebook), _ptr(trits), _ptr(idx), _stream(stream)),
           "tern_fit_bt")
