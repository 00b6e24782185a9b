"""An E8-lattice codebook of 2^16 eight-dimensional entries (the E8P-style
vector quantizer the QTIP discussion compares the trellis codes with).

What the pages fix (QuIP# page: abstract, Fig. 2 and Fig. 3 captions; QTIP
discussion, "Inference speed analysis (W2)" and the reply comparing QTIP with
QuIP#): a 2-bit codebook of 65536 entries of dimension 8 built on the E8
lattice (the densest packing of unit balls in 8 dimensions), stored as a
table of 256 32-bit entries and decompressed with a few bit operations per
weight, read 8 weights at a time.  The construction itself is not on the
pages; the reading used here is built from textbook facts about E8 only:

  * E8 = D8 u (D8 + (1/2) 1), with D8 = {x in Z^8 : sum of x even}: a vector
    is in E8 when its coordinates are all integers or all half-odd-integers
    and their sum is even.
  * Shapes: the 256 vectors of (Z_{>=0} + 1/2)^8 (nonnegative half-odd
    coordinates) of smallest norm, ties broken by the vector 2T read
    lexicographically (smallest first).  2T has odd coordinates 1, 3 or 5,
    which fit four bits each: one 32-bit table word per shape.
  * Index: a 16-bit state s, a = s >> 8 picks the shape, bits 1..7 of s give
    the signs of coordinates 0..6 (bit i + 1 set = coordinate i negative), and
    bit 0 the shift h.
  * Codeword: x = sigma * T[a] + (h ? +1/4 : -1/4) 1, where the sign of
    coordinate 7 is chosen so that sum(sigma * T[a]) is even, i.e.
    sigma * T[a] lies in E8.  So every codeword is an E8 point shifted by
    +-1/4 along the all-ones vector; the set is closed under negation
    (negate the signs and flip h).

With L = kV = 16 and V = 8 each trellis step's own 16 bits are the index
(plain VQ, the QTIP discussion's ablation reply: L = kV turns the trellis
into k-bit, V-dimensional VQ), at k = 2 bits per weight.  Every value is a
multiple of 1/4 below 4 in magnitude: exact in fp16.
"""
from __future__ import annotations

import itertools

import numpy as np

SHIFT = 0.25
N_SHAPES = 256


def is_e8(x) -> np.ndarray:
    """Membership in E8 of each vector x[..., 8] (float64, exact halves)."""
    x = np.asarray(x, dtype=np.float64)
    twice = 2.0 * x
    if not np.all(twice == np.round(twice)):
        return np.zeros(x.shape[:-1], dtype=bool)
    t = np.round(twice).astype(np.int64)
    all_even = np.all(t % 2 == 0, axis=-1)
    all_odd = np.all(t % 2 != 0, axis=-1)
    total = np.sum(t, axis=-1)          # 2 * sum(x)
    return (all_even | all_odd) & (total % 4 == 0)


def shape_table() -> np.ndarray:
    """The 256 shapes T (float64 [256, 8], nonnegative half-odd coordinates),
    smallest norm first, ties by 2T in lexicographic order."""
    cands = sorted(itertools.product((1, 3, 5, 7), repeat=8), key=lambda n: (sum(v * v for v in n), n))
    return np.array(cands[:N_SHAPES], dtype=np.float64) / 2.0


_SHAPES = None


def _shapes() -> np.ndarray:
    global _SHAPES
    if _SHAPES is None:
        _SHAPES = shape_table()
    return _SHAPES


def codeword(state) -> np.ndarray:
    """The codeword of each 16-bit state: float64 [..., 8]."""
    s = np.asarray(state, dtype=np.int64)
    assert np.all((s >= 0) & (s < 1 << 16))
    T = _shapes()[s >> 8]                                    # [..., 8]
    neg = np.stack([(s >> (i + 1)) & 1 for i in range(7)], axis=-1)  # coordinates 0..6
    sigma7 = 1.0 - 2.0 * neg.astype(np.float64)
    partial = np.sum(sigma7 * T[..., :7], axis=-1) + T[..., 7]   # sum with coordinate 7 positive
    # 2 * partial is an integer; the sum must be even: flip coordinate 7 when it is odd
    odd = np.round(2.0 * partial).astype(np.int64) % 4 != 0
    sigma = np.concatenate([sigma7, np.where(odd, -1.0, 1.0)[..., None]], axis=-1)
    shift = np.where((s & 1) == 1, SHIFT, -SHIFT)
    return sigma * T + shift[..., None]


def e8p(state) -> np.ndarray:
    """Code values of each state, float64 [..., 8] (fp16-exact)."""
    return codeword(state)
