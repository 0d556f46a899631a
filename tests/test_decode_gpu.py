"""GPU parity of the persistent decode step (tern_decode_step) against the decode-layer oracle.

Exact where the arithmetic is fixed: the q/k/v projections after RoPE and the
cache entries (bit for bit), the o_proj and MLP halves of a layer from seeded
inputs (bit for bit), and whole multi-layer steps at position 0, where the
softmax weight of the only position is exactly 1 on both sides, so attention
returns the stored value. The attention over several positions runs in fp32
on the GPU against the oracle's fp64: its output is checked within a
tolerance derived from fp32 accumulation (below).
"""
import numpy as np
import pytest

from oracle import decode as dec
from packed_ternary_weight_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# fp32 attention against fp64: scores carry ~128 * 2^-24 relative error, the
# softmax and the weighted sum over n positions a few ulps more per term, so
# the result is within ~1e-5 of the head's largest |value| for the lengths here
ATTN_TOL = 2e-5
SMALL = dict(D=256, F=512, H=4, KVH=2)


@pytest.fixture(scope="module")
def tern():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from packed_ternary_weight_b200 import tern as t
    return t


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class Setup:
    def __init__(self, tern, m: synth.DecodeModel):
        self.m = m
        packed = []
        for lw in m.layers:
            for lay in lw:
                _, buf = tern.pack_layer(lay)
                packed.append(dev(buf))
        gains = dev(np.concatenate([np.concatenate(g) for g in m.gains]).astype(np.float32))
        self.kc = dev(m.kcache.view(np.int16))
        self.vc = dev(m.vcache.view(np.int16))
        rope = dev(tern.decode_rope_table(m.max_pos))
        self.model = tern.DecodeModel(packed, gains, self.kc, self.vc, rope, m.D, m.F, m.H, m.KVH, m.max_pos)
        self.ws = torch.zeros(self.model.workspace_size(), dtype=torch.uint8, device="cuda")
        self.trace = torch.full((len(m.layers), 2 * m.H * 128 + 2 * m.KVH * 128), float("nan"), device="cuda")

    def run(self, tern, h, first=0, last=None, attn=None, pos=None):
        pos = self.m.pos if pos is None else pos
        out = torch.full((self.m.D,), float("nan"), device="cuda")
        self.model.step(pos, dev(h), out, self.ws, first, last, None if attn is None else dev(attn), self.trace)
        torch.cuda.synchronize()
        assert tern.device_error() == tern.OK
        return out.cpu().numpy()

    def weights(self, li):
        return [(lay.trits, lay.tensor_scale) for lay in self.m.layers[li]]


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def check_attention(got, ref, H):
    g = got.reshape(H, 128).astype(np.float64)
    r = ref.reshape(H, 128).astype(np.float64)
    for h in range(H):
        err = np.abs(g[h] - r[h]).max() / max(np.abs(r[h]).max(), 1e-30)
        assert err <= ATTN_TOL, (h, err)


# --------------------------------------------------------------- exact halves
@pytest.mark.parametrize("shape", ["small", "bitnet2b"])
def test_mlp_half_bit_exact(tern, shape):
    kw = SMALL if shape == "small" else {}
    m = synth.decode_model(n_layers=1, pos=5, max_pos=8, seed=40, **kw)
    s = Setup(tern, m)
    h = synth.decode_attn_input(41, m.D)                   # seeded residual stream
    got = s.run(tern, h, first=3, last=4)
    ref = dec.decode_layer(h, s.weights(0), m.gains[0], m.kcache[0].copy(), m.vcache[0].copy(), m.pos,
                           dec.rope_cos_sin(m.pos), first=4, last=5)
    assert np.array_equal(bits(got), bits(ref))


@pytest.mark.parametrize("shape", ["small", "bitnet2b"])
def test_o_proj_and_mlp_bit_exact(tern, shape):
    kw = SMALL if shape == "small" else {}
    m = synth.decode_model(n_layers=1, pos=5, max_pos=8, seed=50, **kw)
    s = Setup(tern, m)
    h = m.h0
    attn = synth.decode_attn_input(51, m.H * 128)
    for last in (2, 3, 4):      # ends after o_proj, gate/up, down
        got = s.run(tern, h, first=2, last=last, attn=attn)
        ref = dec.decode_layer(h, s.weights(0), m.gains[0], m.kcache[0].copy(), m.vcache[0].copy(), m.pos,
                               dec.rope_cos_sin(m.pos), first=3, last=last + 1, attn_in=attn)
        assert np.array_equal(bits(got), bits(ref)), last


@pytest.mark.parametrize("shape,pos,max_pos", [("small", 9, 16), ("small", 300, 320), ("bitnet2b", 1023, 1024)])
def test_qkv_rope_cache_and_attention(tern, shape, pos, max_pos):
    kw = SMALL if shape == "small" else {}
    m = synth.decode_model(n_layers=1, pos=pos, max_pos=max_pos, seed=60, **kw)
    s = Setup(tern, m)
    got_h = s.run(tern, m.h0, first=0, last=1)
    assert np.array_equal(bits(got_h), bits(m.h0))           # no residual add in these stages
    kc, vc = m.kcache[0].copy(), m.vcache[0].copy()
    rec = {}
    dec.decode_layer(m.h0, s.weights(0), m.gains[0], kc, vc, pos, dec.rope_cos_sin(pos), last=2, rec=rec)
    tr = s.trace.cpu().numpy()[0]
    HQ, KQ = m.H * 128, m.KVH * 128
    assert np.array_equal(bits(tr[:HQ]), bits(rec["q_rope"]))
    assert np.array_equal(bits(tr[HQ:HQ + KQ]), bits(rec["k_rope"]))
    assert np.array_equal(bits(tr[HQ + KQ:HQ + 2 * KQ]), bits(rec["v"]))
    # the cache: position pos written (bf16 as the oracle stores it), every other position untouched
    assert np.array_equal(s.kc.cpu().numpy().view(np.uint16)[0], kc)
    assert np.array_equal(s.vc.cpu().numpy().view(np.uint16)[0], vc)
    check_attention(tr[HQ + 2 * KQ:], rec["attn"], m.H)


def test_attention_long_context_passes(tern):
    # one KV head: the 148 position ranges hold more than 64 cached positions each (several passes)
    m = synth.decode_model(D=256, F=256, H=2, KVH=1, n_layers=1, pos=12000, max_pos=12001, seed=70)
    s = Setup(tern, m)
    s.run(tern, m.h0, first=0, last=1)
    rec = {}
    dec.decode_layer(m.h0, s.weights(0), m.gains[0], m.kcache[0].copy(), m.vcache[0].copy(), m.pos,
                     dec.rope_cos_sin(m.pos), last=2, rec=rec)
    HQ, KQ = 2 * 128, 128
    check_attention(s.trace.cpu().numpy()[0][HQ + 2 * KQ:], rec["attn"], 2)


# ------------------------------------------------------------- whole steps
@pytest.mark.parametrize("shape,layers", [("small", 3), ("bitnet2b", 2)])
def test_full_step_position_zero_bit_exact(tern, shape, layers):
    kw = SMALL if shape == "small" else {}
    m = synth.decode_model(n_layers=layers, pos=0, max_pos=4, seed=80, **kw)
    s = Setup(tern, m)
    got = s.run(tern, m.h0)
    kc, vc = m.kcache.copy(), m.vcache.copy()
    recs = {}
    ref = dec.decode_step(m.h0, [s.weights(li) for li in range(layers)], m.gains, kc, vc, 0, dec.rope_cos_sin(0),
                          recs=recs)
    assert np.array_equal(bits(got), bits(ref))
    assert np.array_equal(s.kc.cpu().numpy().view(np.uint16), kc)
    assert np.array_equal(s.vc.cpu().numpy().view(np.uint16), vc)
    tr = s.trace.cpu().numpy()
    HQ, KQ = m.H * 128, m.KVH * 128
    for li in range(layers):
        assert np.array_equal(bits(tr[li, HQ + 2 * KQ:]), bits(recs[li]["attn"]))


def test_full_step_repeatable_and_workspace_reuse(tern):
    m = synth.decode_model(n_layers=2, pos=7, max_pos=8, seed=90, **SMALL)
    s = Setup(tern, m)
    a = s.run(tern, m.h0)
    b = s.run(tern, m.h0)
    assert np.array_equal(bits(a), bits(b))
    # a whole step equals its stages run as separate calls from the same state
    k0, v0 = s.kc.clone(), s.vc.clone()
    h1 = s.run(tern, m.h0, first=0, last=4)
    h2 = s.run(tern, h1, first=5, last=9)
    assert np.array_equal(bits(h2), bits(a))
    assert torch.equal(s.kc, k0) and torch.equal(s.vc, v0)   # the same keys and values rewritten


def test_full_step_several_positions_within_tolerance(tern):
    # pos > 0: the fp32 attention differs from the oracle's fp64 in the last bits, and the
    # next linear's int8 codes can flip where a value lies that close to a rounding
    # boundary; one such flip moves every output of that linear by s_w * s_x. The
    # residual stream stays within 1% (rms) of the oracle's after two layers.
    m = synth.decode_model(n_layers=2, pos=11, max_pos=12, seed=95, **SMALL)
    s = Setup(tern, m)
    got = s.run(tern, m.h0)
    ref = dec.decode_step(m.h0, [s.weights(li) for li in range(2)], m.gains, m.kcache.copy(), m.vcache.copy(),
                          m.pos, dec.rope_cos_sin(m.pos))
    rel = np.sqrt(np.mean((got.astype(np.float64) - ref) ** 2)) / np.sqrt(np.mean(ref.astype(np.float64) ** 2))
    assert rel <= 1e-2, rel
