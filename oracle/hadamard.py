"""Dense normalised Walsh-Hadamard blocks and the random-sign Hadamard transform.

QuIP# page, Fig. 2: incoherence processing with a Randomized Hadamard
Transform (random signs, then a Hadamard transform).  QTIP discussion,
"Incoherence Processing (W2)": the RHT is fully invertible up to numerical
error.  The layer's weight is W = alpha diag(s_out) H_m^T W_hat H_n diag(s_in).

Reading for dimensions that are not powers of two (the pages are silent; the
workloads' "padded power-of-2 blocks"): H_d = I_{d/B} (x) H_B with B the
largest power of two dividing d, i.e. the transform acts on consecutive
blocks of B entries.  H_B is the normalised Sylvester matrix
H_B[i][j] = (-1)^popcount(i & j) / sqrt(B), which is symmetric, so H^T = H.
"""
from __future__ import annotations

import numpy as np


def block_size(d: int) -> int:
    """Largest power of two dividing d."""
    assert d > 0
    return d & -d


def dense(B: int, normalised: bool = True, rows=None) -> np.ndarray:
    """H_B (or the listed rows of it) from the closed form, float64."""
    assert B > 0 and B & (B - 1) == 0
    i = np.arange(B, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    j = np.arange(B, dtype=np.int64)
    parity = np.bitwise_count(i[:, None] & j[None, :]) & 1
    H = 1.0 - 2.0 * parity.astype(np.float64)
    return H / np.sqrt(B) if normalised else H


def apply_blockwise(v: np.ndarray, B: int) -> np.ndarray:
    """(I (x) H_B) applied along the last axis of v, in float64.

    Output entry i of a block is the sum over j of H_B[i][j] * v[j], accumulated
    in the order j = 0, 1, ..., B-1; column j of H_B is taken from the closed
    form (H_B is symmetric, so it is row j)."""
    v = np.asarray(v, dtype=np.float64)
    d = v.shape[-1]
    assert d % B == 0
    blocks = v.reshape(v.shape[:-1] + (d // B, B))
    out = np.zeros_like(blocks)
    for j in range(B):
        col = dense(B, rows=[j])[0]
        out += blocks[..., j:j + 1] * col
    return out.reshape(v.shape)


def rht(x: np.ndarray, signs: np.ndarray, B: int) -> np.ndarray:
    """H (diag(signs) x) blockwise along the last axis."""
    return apply_blockwise(np.asarray(x, dtype=np.float64) * np.asarray(signs, dtype=np.float64), B)
