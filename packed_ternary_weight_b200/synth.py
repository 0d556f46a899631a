"""Seeded synthetic inputs for the packed ternary-weight GEMV.

This module only draws random inputs; it contains none of the arithmetic of the
method (no packing, no decoding, no products, no quantisation). Both the CUDA
path (through the packer and the C-ABI) and the CPU oracle consume what it
returns, so the two never share code beyond these generators.

Recipe (the same for every workload):

* generator: ``numpy.random.Generator(PCG64(seed))``;
* trits: ``integers(0, 10)`` mapped {0,1,2} -> -1, {3,4,5,6} -> 0, {7,8,9} -> +1,
  so P(-1) = P(+1) = 0.3 and P(0) = 0.4 exactly (the single-ternary-GEMV
  workload's distribution, used for every format);
* TQ{K}P group scales: ``fp16_rn(|z| * 0.02 * 3**-p)`` with z ~ N(0,1) in fp64,
  drawn after the trits from the same generator, shape [P][N][K/g];
* balanced-ternary scale indices: ``integers(0, 27)`` per (row, group of 16),
  drawn after the trits;
* activations: a separate generator seeded ``seed + 1_000_000``,
  ``standard_normal(float32)`` rounded to bf16 (round to nearest even);
* the 27-entry codebook: ``float32(1e-4 * 10**(3 i / 26))``, i = 0..26
  (log-spaced, both ends included: 1e-4 and 1e-1).

Layer shapes are those of BitNet b1.58-2B (hidden 2560, FFN 6912, 20 query /
5 KV heads of 128, 30 layers) and Llama-3.1-8B (hidden 4096, FFN 14336, 8 KV
heads of 128).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

X_SEED_OFFSET = 1_000_000

# BitNet b1.58-2B projections, (name, N out, K in): QORA-LLM-2B page, "Architecture".
BITNET_2B_SHAPES = (
    ("q_proj", 2560, 2560),
    ("k_proj", 640, 2560),
    ("v_proj", 640, 2560),
    ("o_proj", 2560, 2560),
    ("gate_proj", 6912, 2560),
    ("up_proj", 6912, 2560),
    ("down_proj", 2560, 6912),
)
BITNET_2B_LAYERS = 30

# Llama-3.1-8B projections (hidden 4096, FFN 14336, GQA 32/8 x 128).
LLAMA_8B_SHAPES = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
LLAMA_8B_LAYERS = 32


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


_TRIT_OF_DRAW = np.array([-1, -1, -1, 0, 0, 0, 0, 1, 1, 1], dtype=np.int8)


def draw_trits(gen: np.random.Generator, shape) -> np.ndarray:
    """Trits in {-1, 0, +1} as int8 with P(-1)=P(+1)=0.3, P(0)=0.4."""
    u = gen.integers(0, 10, size=shape, dtype=np.int8)
    return _TRIT_OF_DRAW[u]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_x_bf16(seed: int, m: int, k: int) -> np.ndarray:
    """Activations [m][k] as bf16 bits (uint16), N(0,1) rounded to bf16."""
    g = rng(seed + X_SEED_OFFSET)
    return f32_to_bf16_bits(g.standard_normal((m, k), dtype=np.float32))


def draw_tq_scales(gen: np.random.Generator, planes: int, n: int, groups: int) -> np.ndarray:
    z = gen.standard_normal((planes, n, groups))  # fp64
    mag = np.abs(z) * 0.02 * (3.0 ** -np.arange(planes, dtype=np.float64))[:, None, None]
    return mag.astype(np.float16)


def codebook27() -> np.ndarray:
    i = np.arange(27, dtype=np.float64)
    return (1e-4 * 10.0 ** (3.0 * i / 26.0)).astype(np.float32)


@dataclass
class Layer:
    """Logical (unpacked) inputs of one packed ternary linear layer."""

    fmt: str                 # "bitnet" | "tq" | "bt3"
    n: int
    k: int
    planes: int              # P for bitnet/tq; the depth d for bt3
    group: int               # g along K; K for bitnet; 16 for bt3
    trits: np.ndarray        # int8 [P][N][K]
    tensor_scale: float = 0.0            # bitnet
    scales: np.ndarray | None = None     # tq: fp16 [P][N][K/g]
    idx: np.ndarray | None = None        # bt3: uint8 [N][K/16] in 0..26
    codebook: np.ndarray | None = None   # bt3: float32 [27]
    seed: int = 0
    name: str = ""
    extra: dict = field(default_factory=dict)


def bitnet_layer(n: int, k: int, seed: int, tensor_scale: float = 0.02, name: str = "") -> Layer:
    g = rng(seed)
    t = draw_trits(g, (1, n, k))
    return Layer("bitnet", n, k, 1, k, t, tensor_scale=float(np.float32(tensor_scale)), seed=seed, name=name)


def tq_layer(n: int, k: int, planes: int, group: int, seed: int, name: str = "") -> Layer:
    assert k % group == 0
    g = rng(seed)
    t = draw_trits(g, (planes, n, k))
    s = draw_tq_scales(g, planes, n, k // group)
    return Layer("tq", n, k, planes, group, t, scales=s, seed=seed, name=name)


def bt3_layer(n: int, k: int, seed: int, name: str = "", depth: int = 3) -> Layer:
    assert k % 16 == 0
    g = rng(seed)
    t = draw_trits(g, (depth, n, k))
    idx = g.integers(0, 27, size=(n, k // 16), dtype=np.uint8)
    return Layer("bt3", n, k, depth, 16, t, idx=idx, codebook=codebook27(), seed=seed, name=name)


# ---------------------------------------------------------------- workloads
def single_gemv_layer() -> Layer:
    """One BitNet-layout plane, 512 out x 1024 in, tensor scale 0.02, seed 0."""
    return bitnet_layer(512, 1024, seed=0, tensor_scale=0.02, name="single_512x1024")


def bitnet_layer_set_seed(layer: int, proj: int) -> int:
    """Seed of projection `proj` (q,k,v,o,gate,up,down = 0..6) of layer `layer`."""
    return 1000 + 7 * layer + proj


def bitnet_layer_set(layers: int = BITNET_2B_LAYERS):
    """BitNet b1.58-2B decode layer set: `layers` x 7 projections, distinct seeds."""
    for li in range(layers):
        for pi, (name, n, k) in enumerate(BITNET_2B_SHAPES):
            yield bitnet_layer(n, k, bitnet_layer_set_seed(li, pi), 0.02, name=f"L{li}.{name}")


def tq3p_llama_layers():
    """TQ3P (3 planes, g = 256) at Llama-3.1-8B shapes; seed 200 + shape index."""
    for si, (name, n, k) in enumerate(LLAMA_8B_SHAPES):
        yield tq_layer(n, k, 3, 256, seed=200 + si, name=name)


def bt3_llama_layers():
    """Balanced ternary depth 3, group 16, Llama-3.1-8B shapes; seed 300 + shape index."""
    for si, (name, n, k) in enumerate(LLAMA_8B_SHAPES):
        yield bt3_layer(n, k, seed=300 + si, name=name)


PREFILL_SHAPES = (("ffn_up", 14336, 4096), ("ffn_down", 4096, 14336))
PREFILL_TOKENS = (1, 2, 4, 8, 16, 64, 256)


def tq2p_prefill_layers():
    """TQ2P (2 planes, g = 32) prefill layers; seed 400 + shape index."""
    for si, (name, n, k) in enumerate(PREFILL_SHAPES):
        yield tq_layer(n, k, 2, 32, seed=400 + si, name=name)


# ------------------------------------------------------------ decode step
# Synthetic BitNet b1.58 decoder (no trained weights): per layer the seven
# projections of the layer set's recipe (seeds 1000 + 7 layer + projection
# by default), RMSNorm gains bf16(1 + 0.1 z), a KV cache prefix of bf16
# N(0,1) keys and values, and the residual stream of the token as bf16 N(0,1)
# values (standing in for an embedding row).
@dataclass
class DecodeModel:
    D: int
    F: int
    H: int
    KVH: int
    layers: list            # per layer: seven Layer objects (q, k, v, o, gate, up, down)
    gains: list             # per layer: four fp32 vectors (input D, attn_sub H*128, post D, ffn_sub F)
    kcache: np.ndarray      # bf16 bits [L][KVH][max_pos][128]
    vcache: np.ndarray
    h0: np.ndarray          # fp32 [D]
    pos: int
    max_pos: int


def decode_model(D: int = 2560, F: int = 6912, H: int = 20, KVH: int = 5, n_layers: int = 1, pos: int = 1023,
                 max_pos: int = 1024, seed: int = 1000, head_dim: int = 128) -> DecodeModel:
    """Seeded synthetic decoder inputs. Layer li, projection pi uses seed + 7 li + pi (with the
    default seed and BitNet-2B shapes these are the layer set's layers)."""
    shapes = [(H * head_dim, D), (KVH * head_dim, D), (KVH * head_dim, D), (D, H * head_dim), (F, D), (F, D),
              (D, F)]
    names = [nm for nm, _, _ in BITNET_2B_SHAPES]
    layers, gains = [], []
    for li in range(n_layers):
        layers.append([bitnet_layer(n, k, seed + 7 * li + pi, 0.02, name=f"L{li}.{names[pi]}")
                       for pi, (n, k) in enumerate(shapes)])
        g = rng(seed + 500_000 + li)
        gains.append([bf16_bits_to_f32(f32_to_bf16_bits((1.0 + 0.1 * g.standard_normal(n)).astype(np.float32)))
                      for n in (D, H * head_dim, D, F)])
    g = rng(seed + 600_000)
    kc = f32_to_bf16_bits(g.standard_normal((n_layers, KVH, max_pos, head_dim), dtype=np.float32))
    vc = f32_to_bf16_bits(g.standard_normal((n_layers, KVH, max_pos, head_dim), dtype=np.float32))
    h0 = bf16_bits_to_f32(f32_to_bf16_bits(g.standard_normal(D, dtype=np.float32)))
    return DecodeModel(D, F, H, KVH, layers, gains, kc, vc, h0, pos, max_pos)


def decode_attn_input(seed: int, n: int) -> np.ndarray:
    """A stand-in attention output (fp32 N(0,1)) for runs that start at o_proj."""
    return rng(seed + 700_000).standard_normal(n, dtype=np.float32)
