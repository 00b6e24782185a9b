"""The bitshift trellis, walked state by state.

QTIP discussion, "Figure 2 (Q4)": a state is L bits; the last L-kV bits of a
state are the first L-kV bits of the next one, so only the kV-bit "delta" of
each step is stored.  The example given there: the bit string 0010110 with
L=2, kV=1 visits the states 00, 01, 10, 01, 11, 10.  "Ablations and fast
inference (W1 and W2)": L is the trellis size, k the bitrate, V the number of
weights per step; L = kV reduces the trellis to k-bit V-dimensional VQ.

Two forms are walked here:

  * walk_open(bits, L, kV): the form of the printed example.  The first state
    is the first L bits; each later step shifts in kV bits.
  * walk_tailbiting(chunks, prefix, L, kV): the form the stored layer uses
    (a reading; the pages do not say how a sequence starts).  A block of S
    bits holds exactly S/kV chunks, one per step; step t's state is the L-bit
    window ending at bit (t+1)*kV of the block, taken cyclically, so the first
    state borrows its high L-kV bits from the end of the same block.  This
    keeps the storage at exactly k bits per weight, which is what the "Bit
    Accounting (Q2)" answer counts (signs and codebook are the only overhead).

Each step asserts the bitshift property: the new state's high L-kV bits are
the old state's low L-kV bits.
"""
from __future__ import annotations

import numpy as np

from . import bitstream


def step(state, chunk, L: int, kV: int):
    """One trellis step: shift kV new bits into an L-bit state."""
    new = ((np.asarray(state, dtype=np.int64) << kV) | np.asarray(chunk, dtype=np.int64)) & ((1 << L) - 1)
    keep = L - kV
    assert np.all((new >> kV) == (np.asarray(state) & ((1 << keep) - 1))), "bitshift property violated"
    return new


def walk_open(bitstring: str, L: int, kV: int) -> list:
    """States visited by an open (non-cyclic) walk over a '0'/'1' string."""
    assert len(bitstring) >= L and (len(bitstring) - L) % kV == 0
    state = int(bitstring[:L], 2)
    states = [state]
    for p in range(L, len(bitstring), kV):
        state = int(step(state, int(bitstring[p:p + kV], 2), L, kV))
        states.append(state)
    return states


def walk_tailbiting(chunks: np.ndarray, prefix: np.ndarray, L: int, kV: int) -> np.ndarray:
    """Tail-biting walk of many blocks at once.

    chunks: int [blocks, steps], the kV-bit chunk of each step (MSB first).
    prefix: int [blocks], the last L-kV bits of each block.
    Returns the states, int [blocks, steps].
    """
    blocks, steps = chunks.shape
    states = np.empty((blocks, steps), dtype=np.int64)
    s = np.asarray(prefix, dtype=np.int64)
    for t in range(steps):
        s = step(s, chunks[:, t], L, kV)
        states[:, t] = s
    keep = L - kV
    assert np.all((s & ((1 << keep) - 1)) == (np.asarray(prefix) & ((1 << keep) - 1))), "tail-biting mismatch"
    return states


def block_states(words: np.ndarray, rows: np.ndarray, n: int, parts, L: int, V: int, blocks=None) -> np.ndarray:
    """States of every step of the given blocks (default: all) of the given rows.

    Returns int [len(rows), len(blocks), T/V].  Each row's k is taken from
    `parts` (half-TCQ layers carry two k values; k may be a half number of
    bits, e.g. 2.5 with V = 2 is a 5-bit step).
    """
    T = bitstream.T
    rows = np.asarray(rows, dtype=np.int64)
    base, kk2 = bitstream.row_base_bits(rows, n, parts)
    blocks = np.arange(n // T) if blocks is None else np.asarray(blocks, dtype=np.int64)
    nb = len(blocks)
    steps = T // V
    out = np.empty((len(rows), nb, steps), dtype=np.int64)
    for k2 in np.unique(kk2):
        k2 = int(k2)
        sel = np.nonzero(kk2 == k2)[0]
        assert (k2 * V) % 2 == 0, "a step must carry a whole number of bits"
        kV = k2 * V // 2
        S = T * k2 // 2
        assert L >= kV, "a state must hold at least one step's bits"
        # bit offset of every block start: [rows_sel, nb]
        bstart = base[sel][:, None] + blocks[None, :] * S
        bstart = bstart.reshape(-1)
        chunks = np.stack([bitstream.field(words, bstart + t * kV, kV) for t in range(steps)], axis=1)
        prefix = bitstream.field(words, bstart + S - (L - kV), L - kV) if L > kV else np.zeros_like(bstart)
        states = walk_tailbiting(chunks, prefix, L, kV)
        out[sel] = states.reshape(len(sel), nb, steps)
    return out
