"""Decode of W_hat and the forward pass of the quantized linear layer.

    y = alpha * diag(s_out) * H_m^T * W_hat * H_n * diag(s_in) * x

W_hat[r][j*T + t*V + e] is value e of the code applied to state t of block j
of row r (QTIP discussion: bitshift trellis, "Figure 2 (Q4)"; codes,
"Inference speed analysis (W2)"; reading of the element order: step t covers
the V consecutive columns t*V .. t*V+V-1 of its block).  Each value is rounded
once to fp16; the decoded matrix is the fp16 matrix the layer multiplies by.

Every step is a plain dense computation in float64: the trellis walk state by
state, the code on each state, the dense Hadamard blocks built explicitly, and
the contraction as a sum of products accumulated column by column.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from . import bitstream, codes, fp16, hadamard, trellis

T = bitstream.T


@dataclasses.dataclass
class Layer:
    m: int
    n: int
    parts: list          # [(row0, rows, k)] in stream order
    L: int
    V: int
    code: int
    words: np.ndarray    # uint32, canonical stream
    s_in: np.ndarray     # +-1, [n]
    s_out: np.ndarray    # +-1, [m]
    alpha: float
    lut: Optional[np.ndarray] = None  # float16 [2^Q, V]

    @classmethod
    def from_inputs(cls, li) -> "Layer":
        sp = li.spec
        return cls(sp.m, sp.n, sp.row_parts(), sp.L, sp.V, sp.code, li.codes, li.s_in, li.s_out,
                   sp.alpha, li.lut)

    @property
    def B_n(self) -> int:
        return hadamard.block_size(self.n)

    @property
    def B_m(self) -> int:
        return hadamard.block_size(self.m)

    # ---- decode -----------------------------------------------------------
    def decode_rows(self, rows, blocks=None) -> np.ndarray:
        """W_hat rows as float64 (fp16-exact values), [len(rows), n]; with
        `blocks`, only those 256-column blocks, [len(rows), len(blocks)*T]."""
        rows = np.asarray(rows, dtype=np.int64)
        states = trellis.block_states(self.words, rows, self.n, self.parts, self.L, self.V, blocks)
        vals = codes.evaluate(self.code, states, self.V, self.lut)  # [r, nb, steps, V]
        return vals.reshape(len(rows), -1)

    def decode_bits(self, rows) -> np.ndarray:
        """W_hat rows as fp16 bit patterns, uint16 [len(rows), n]."""
        return fp16.encode(self.decode_rows(rows))

    # ---- forward ----------------------------------------------------------
    def input_transform(self, x) -> np.ndarray:
        """x' = H_n diag(s_in) x, float64 [batch, n]; x is read exactly (fp16 -> float64)."""
        x64 = np.asarray(x).astype(np.float64)
        return hadamard.rht(x64, self.s_in, self.B_n)

    def contract(self, xp, rows) -> np.ndarray:
        """z = W_hat x' at the listed rows, float64 [batch, len(rows)]: entry
        (b, r) is the sum over columns c of W_hat[r][c] * x'[b][c], accumulated
        in the order c = 0, 1, ..., n-1."""
        return contract(self.decode_rows(rows), xp)

    def output_transform(self, z, rows) -> np.ndarray:
        """y = alpha * s_out * (H_m z) on whole output Hadamard blocks: `rows`
        lists the blocks' rows in order and z holds W_hat x' on them."""
        rows = np.asarray(rows, dtype=np.int64)
        assert len(rows) % self.B_m == 0 and np.all(rows[::self.B_m] % self.B_m == 0)
        yb = hadamard.apply_blockwise(z, self.B_m)  # H_m^T = H_m (symmetric)
        return self.alpha * self.s_out[rows].astype(np.float64) * yb

    def forward_blocks(self, x, out_blocks) -> dict:
        """y on whole output Hadamard blocks: {block index: float64 [batch, B_m]}."""
        xp = self.input_transform(x)
        Bm = self.B_m
        out = {}
        for b in out_blocks:
            rows = np.arange(b * Bm, (b + 1) * Bm)
            out[b] = self.output_transform(self.contract(xp, rows), rows)
        return out

    def forward(self, x) -> np.ndarray:
        """y = W x for every output, float64 [batch, m]."""
        blocks = self.forward_blocks(x, range(self.m // self.B_m))
        return np.concatenate([blocks[b] for b in range(self.m // self.B_m)], axis=1)

    def forward_rows(self, x, rows) -> np.ndarray:
        """y at the listed output rows, float64 [batch, len(rows)]."""
        rows = np.asarray(rows, dtype=np.int64)
        Bm = self.B_m
        blocks = self.forward_blocks(x, sorted(set((rows // Bm).tolist())))
        return np.stack([blocks[r // Bm][:, r % Bm] for r in rows], axis=1)


def contract(W, xp) -> np.ndarray:
    """z[b][r] = sum over c of W[r][c] * xp[b][c], float64, accumulated column by
    column in order (W: [rows, n], xp: [batch, n])."""
    W = np.asarray(W, dtype=np.float64)
    xp = np.asarray(xp, dtype=np.float64)
    Wt = np.ascontiguousarray(W.T)   # column c of W as a contiguous vector
    z = np.zeros((xp.shape[0], W.shape[0]))
    for c in range(W.shape[1]):
        z += xp[:, c:c + 1] * Wt[c]
    return z
