"""Seeded synthetic inputs for the trellis-coded quantized linear layer.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle.
It holds no arithmetic of the method: it only names the layer shapes and draws
the random arrays the method consumes as inputs (packed code words, +-1 sign
vectors, the HYB lookup table, activations).

Workloads (synthetic stand-ins for the Llama-2/3-shaped layers the QTIP
OpenReview discussion times and evaluates; no weights or datasets are used):

  tiny      m=n=256,            k=2, L=16, V=1, 1MAD,  alpha=1,    batch 1
  attn4096  m=n=4096,           k=2, L=16, V=1, 3INST, alpha=0.02, batch 1
  mlp_up    m=11008, n=4096,    k=3, L=16, V=2, HYB Q=9,  alpha=1, batch 1/4/8
  mlp_down  m=4096,  n=11008,   k=3, L=16, V=2, HYB Q=9,  alpha=1, batch 1/4/8
  large     m=28672, n=8192,    k=4, L=16, V=1, 1MAD,  alpha=0.01, batch 1/4/16
  halftcq   m=14336, n=4096, rows [0,7168) k=2 and [7168,14336) k=3,
            L=16, V=1, 3INST, alpha=1, batch 64/256
  qkv_fused m=12288, n=4096, three 4096-row parts at k=2, 3, 4, L=16, V=1, 3INST

Palette workloads (the Q-Palette page's fractional bitwidths and its VQ / NUQ
quantizers beside TCQ), all m=n=4096, batch 1/4/8:

  tcq2p5    k=2.5 (5 bits per 2-value step), L=16, V=2, HYB Q=9
  tcq2p75   rows [0,2048) at k=2.5 and [2048,4096) at k=3, L=16, V=2, HYB Q=9
            (the page's 2.75-bit example: a 2.5-bit and a 3-bit quantizer)
  vq2p5     k=2.5, L=5, V=2, table code: 32 codewords of 2 values
  nuq3      k=3, L=3, V=1, table code: 8 levels
  e8p2      k=2, L=16, V=8, the E8-lattice code: 2^16 codewords of 8 values

Distributions: code words are uniform uint32, signs uniform +-1 (int8), the
HYB table holds 2^Q x V standard normals rounded to fp16 (numpy's float16
cast), the table code's codebook 2^L x V standard normals rounded to fp16
(V = 1: sorted, as the levels of a scalar quantizer), activations x ~ N(0,1)
cast to fp16.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence, Tuple

import numpy as np

CODE_1MAD = 0
CODE_3INST = 1
CODE_HYB = 2
CODE_TABLE = 3
CODE_E8P = 4
CODE_NAMES = {CODE_1MAD: "1MAD", CODE_3INST: "3INST", CODE_HYB: "HYB", CODE_TABLE: "TABLE", CODE_E8P: "E8P"}

T_BLOCK = 256  # columns per independent trellis block (fixed by the format)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    m: int
    n: int
    k: float                    # bits per weight (uniform layers), a multiple of 1/2
    L: int
    V: int
    code: int
    alpha: float
    seed: int
    Q: int = 0                  # HYB table index bits
    m_top: Optional[int] = None  # half-TCQ: rows [0, m_top) at k_top, rest at k_bot
    k_top: Optional[float] = None
    k_bot: Optional[float] = None
    batches: Sequence[int] = (1,)
    row_split: Optional[Tuple[Tuple[int, int], ...]] = None  # ((rows, k), ...): layers fused along m

    @property
    def mixed(self) -> bool:
        return self.m_top is not None or self.row_split is not None

    def row_parts(self):
        """[(row0, rows, k)] in stream order."""
        if self.row_split is not None:
            out, r0 = [], 0
            for rows, k in self.row_split:
                out.append((r0, rows, k))
                r0 += rows
            assert r0 == self.m
            return out
        if self.m_top is not None:
            return [(0, self.m_top, self.k_top), (self.m_top, self.m - self.m_top, self.k_bot)]
        return [(0, self.m, self.k)]

    def part_kv(self):
        """Bits per trellis step (kV) of each row part, in stream order."""
        out = []
        for _, _, k in self.row_parts():
            kv2 = int(round(2 * k)) * self.V
            assert kv2 % 2 == 0 and abs(2 * k - round(2 * k)) < 1e-12, "k*V must be a whole number of bits"
            out.append(kv2 // 2)
        return out

    @property
    def fractional(self) -> bool:
        return any(kv % self.V for kv in self.part_kv())

    @property
    def n_words(self) -> int:
        bits = sum(rows * self.n * kv // self.V for (_, rows, _), kv in zip(self.row_parts(), self.part_kv()))
        assert bits % 32 == 0
        return bits // 32

    @property
    def stream_bytes(self) -> int:
        return self.n_words * 4

    @property
    def bits_per_weight(self) -> float:
        return self.n_words * 32 / (self.m * self.n)


WORKLOADS = {
    "tiny": LayerSpec("tiny", 256, 256, 2, 16, 1, CODE_1MAD, 1.0, seed=0, batches=(1,)),
    "attn4096": LayerSpec("attn4096", 4096, 4096, 2, 16, 1, CODE_3INST, 0.02, seed=1, batches=(1,)),
    "mlp_up": LayerSpec("mlp_up", 11008, 4096, 3, 16, 2, CODE_HYB, 1.0, seed=2, Q=9, batches=(1, 4, 8)),
    "mlp_down": LayerSpec("mlp_down", 4096, 11008, 3, 16, 2, CODE_HYB, 1.0, seed=2, Q=9, batches=(1, 4, 8)),
    "large": LayerSpec("large", 28672, 8192, 4, 16, 1, CODE_1MAD, 0.01, seed=3, batches=(1, 4, 16)),
    "halftcq": LayerSpec("halftcq", 14336, 4096, 0, 16, 1, CODE_3INST, 1.0, seed=4,
                         m_top=7168, k_top=2, k_bot=3, batches=(64, 256)),
    # Q, K and V projections of a 4096-wide attention block fused along m (they
    # read the same input), each with its own bitwidth: 2, 3 and 4 bits.
    "qkv_fused": LayerSpec("qkv_fused", 12288, 4096, 0, 16, 1, CODE_3INST, 0.02, seed=5,
                           row_split=((4096, 2), (4096, 3), (4096, 4)), batches=(1, 16)),
    "tcq2p5": LayerSpec("tcq2p5", 4096, 4096, 2.5, 16, 2, CODE_HYB, 1.0, seed=6, Q=9, batches=(1, 4, 8)),
    "tcq2p75": LayerSpec("tcq2p75", 4096, 4096, 0, 16, 2, CODE_HYB, 1.0, seed=7, Q=9,
                         m_top=2048, k_top=2.5, k_bot=3, batches=(1, 4, 8)),
    "vq2p5": LayerSpec("vq2p5", 4096, 4096, 2.5, 5, 2, CODE_TABLE, 1.0, seed=8, batches=(1, 4, 8)),
    "nuq3": LayerSpec("nuq3", 4096, 4096, 3, 3, 1, CODE_TABLE, 1.0, seed=9, batches=(1, 4, 8)),
    # the E8-lattice vector quantizer the trellis codes are compared with: 2 bits
    # per weight, 8 weights per 16-bit step, L = kV = 16 (plain VQ)
    "e8p2": LayerSpec("e8p2", 4096, 4096, 2, 16, 8, CODE_E8P, 0.02, seed=10, batches=(1, 4, 8)),
}

# The up and down projections of the MLP pair draw from one seeded stream
# (up first), so that the two layers of the pair are distinct.
_STREAM_ORDER = {"mlp_down": 1}


@dataclasses.dataclass
class LayerInputs:
    spec: LayerSpec
    codes: np.ndarray       # uint32 [n_words], canonical stream order
    s_in: np.ndarray        # int8 [n], +-1
    s_out: np.ndarray       # int8 [m], +-1
    lut: Optional[np.ndarray]  # float16 [2^Q, V] for HYB, [2^L, V] for the table code, else None


def _rng(seed, instance, stream=0):
    if instance == 0 and stream == 0:
        return np.random.default_rng(seed)
    return np.random.default_rng([seed, stream, instance])


def hyb_table(Q: int, V: int, seed: int) -> np.ndarray:
    """2^Q x V standard-normal entries rounded to fp16 (numpy's float16 cast)."""
    return np.random.default_rng(seed).standard_normal((1 << Q, V)).astype(np.float16)


def palette_table(L: int, V: int, seed: int) -> np.ndarray:
    """The table code's codebook: 2^L x V standard normals rounded to fp16;
    V = 1 sorted ascending (the levels of a non-uniform scalar quantizer)."""
    t = np.random.default_rng([seed, 31]).standard_normal((1 << L, V)).astype(np.float16)
    return np.sort(t, axis=0) if V == 1 else t


def make_layer(spec: LayerSpec, instance: int = 0) -> LayerInputs:
    """Draw the layer's code stream, signs and table.

    instance 0 is the canonical draw for the workload's seed; other instances
    are independent layers of the same shape (used to rotate through more
    bytes than the L2 cache holds when timing).
    """
    stream = _STREAM_ORDER.get(spec.name, 0)
    rng = _rng(spec.seed, instance, stream)
    codes = rng.integers(0, 2**32, size=spec.n_words, dtype=np.uint32)
    s_in = (2 * rng.integers(0, 2, size=spec.n) - 1).astype(np.int8)
    s_out = (2 * rng.integers(0, 2, size=spec.m) - 1).astype(np.int8)
    lut = None
    if spec.code == CODE_HYB:
        lut = hyb_table(spec.Q, spec.V, spec.seed + 1000 * instance)
    elif spec.code == CODE_TABLE:
        lut = palette_table(spec.L, spec.V, spec.seed + 1000 * instance)
    return LayerInputs(spec, codes, s_in, s_out, lut)


def make_x(spec: LayerSpec, batch: int, instance: int = 0) -> np.ndarray:
    """Activations x ~ N(0,1) in fp16, shape [batch, n]."""
    rng = np.random.default_rng([spec.seed, 77, batch, instance])
    return rng.standard_normal((batch, spec.n)).astype(np.float16)


def random_layer(m: int, n: int, k: float, L: int, V: int, code: int, seed: int,
                 alpha: float = 1.0, Q: int = 9, m_top=None, k_top=None, k_bot=None, row_split=None) -> LayerInputs:
    """A small seeded layer of any supported shape (tests of ragged/edge shapes); row_split
    ((rows, k), ...) makes a layer of several row parts (layers fused along m); k may be a
    half number of bits when V = 2."""
    uniform = m_top is None and row_split is None
    spec = LayerSpec(f"rand_{m}x{n}_k{k}", m, n, k if uniform else 0, L, V, code, alpha,
                     seed, Q=Q if code == CODE_HYB else 0, m_top=m_top, k_top=k_top, k_bot=k_bot,
                     row_split=tuple(tuple(r) for r in row_split) if row_split is not None else None)
    return make_layer(spec)
