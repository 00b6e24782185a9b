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


def row_base_bits(r, n: int, parts) -> np.ndarray:
    """First bit of row r. parts = [(row0, rows, k)] in stream order."""
    r = np.asarray(r, dtype=np.int64)
    base = np.zeros(r.shape, dtype=np.int64)
    kk = np.zeros(r.shape, dtype=np.int64)
    offset = 0
    for row0, rows, k in parts:
        inside = (r >= row0) & (r < row0 + rows)
        base = np.where(inside, offset + (r - row0) * n * k, base)
        kk = np.where(inside, k, kk)
        offset += rows * n * k
    return base, kk


def bits_to_words(bitstring: str) -> np.ndarray:
    """'0101...' (length a multiple of 32) -> uint32 words, MSB first."""
    assert len(bitstring) % 32 == 0
    return np.array([int(bitstring[i:i + 32], 2) for i in range(0, len(bitstring), 32)], dtype=np.uint32)
