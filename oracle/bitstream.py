"""The packed code stream: bit order and layout.

Reading of the pages (the QTIP discussion prints only the bit string
"0010110" in "Figure 2 (Q4)" and never fixes how bits sit in memory):

  * The stream is an array of uint32 words read as one bit string, most
    significant bit first: bit p is bit (31 - p % 32) of word p // 32.
  * Each row of W_hat is cut into blocks of T = 256 consecutive columns.  A
    block is one independent trellis of S = T*k bits.  Block j of row r
    starts at bit rowbase(r) + j*S with rowbase(r) = r*n*k; for a half-TCQ
    layer (Q-Palette's mixed-bitwidth layer) rows [m_top, m) start at bit
    m_top*n*k_top + (r - m_top)*n*k_bot.
"""
from __future__ import annotations

import numpy as np

T = 256


def bit(words: np.ndarray, p) -> np.ndarray:
    """Bit p of the stream (vectorised over p)."""
    p = np.asarray(p, dtype=np.int64)
    return (words[p >> 5].astype(np.int64) >> (31 - (p & 31))) & 1


def field(words: np.ndarray, p, width: int) -> np.ndarray:
    """The width-bit integer whose most significant bit is stream bit p."""
    p = np.asarray(p, dtype=np.int64)
    out = np.zeros(p.shape, dtype=np.int64)
    for b in range(width):
        out = (out << 1) | bit(words, p + b)
    return out


def half_bits(k) -> int:
    """2k as an integer (k is a whole or half number of bits per weight)."""
    k2 = int(round(2 * k))
    assert k2 > 0 and abs(2 * k - k2) < 1e-12, "k must be a multiple of 1/2"
    return k2


def bits(k, weights: int) -> int:
    """Bits of `weights` weights at k bits each (a whole number)."""
    b2 = half_bits(k) * weights
    assert b2 % 2 == 0, "not a whole number of bits"
    return b2 // 2


def row_base_bits(r, n: int, parts):
    """(first bit, 2k) of each row r. parts = [(row0, rows, k)] in stream order."""
    r = np.asarray(r, dtype=np.int64)
    base = np.zeros(r.shape, dtype=np.int64)
    kk2 = np.zeros(r.shape, dtype=np.int64)
    offset = 0
    for row0, rows, k in parts:
        inside = (r >= row0) & (r < row0 + rows)
        base = np.where(inside, offset + (r - row0) * bits(k, n), base)
        kk2 = np.where(inside, half_bits(k), kk2)
        offset += rows * bits(k, n)
    return base, kk2


def bits_to_words(bitstring: str) -> np.ndarray:
    """'0101...' (length a multiple of 32) -> uint32 words, MSB first."""
    assert len(bitstring) % 32 == 0
    return np.array([int(bitstring[i:i + 32], 2) for i in range(0, len(bitstring), 32)], dtype=np.uint32)
