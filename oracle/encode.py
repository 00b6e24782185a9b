"""Trellis-coded quantization for the bitshift trellis: the bits of one block
whose tail-biting walk reproduces a source sequence with the least squared
error.  Test infrastructure (the oracle), like the rest of this package.

What the QTIP discussion fixes:
  * "Bitshift trellis" reply (around the 0010110 example): a block stores only
    the kV-bit delta of each step; a walk's states follow from its bits.
  * Reply to "Given a weight tensor, how do you actually find which words
    encode this value the best?" and "Why does TCQ work? (Q5)": encoding is a
    search over fixed-length walks on the trellis for the least distortion
    (trellis-coded quantization, with the RPTC theory behind it), and the
    "Table 1" replies: its distortion on an i.i.d. Gaussian source comes much
    closer to the rate-distortion limit than scalar or vector quantization.
The pages do not print the search.  Readings used here:
  * Objective: sum over the block's steps of the squared error between the
    source values and the code values of the step's state (all V values).
  * Tail-biting (the stream format): state t is the L-bit window ending at bit
    (t+1)kV of the block, cyclically, so the first state's high L-kV bits are
    the block's last L-kV bits (its "prefix").
  * encode_exact: the minimum over all tail-biting walks: one dynamic
    programme (Viterbi) per prefix, float64.  Feasible for small L only.
  * encode_two_pass: a search that stays affordable at L = 16.  Pass 1 runs
    the dynamic programme with a free first state and takes the prefix of its
    best final state; pass 2 runs it again with the first state's high bits
    and the last state's low bits both fixed to that prefix.  Every cost is
    float32 (difference, square, sum over the V values in order, then the
    addition to the path cost, each rounded to float32); ties go to the
    smallest state (final choice) and the smallest predecessor state.
"""
from __future__ import annotations

import numpy as np

from . import codes, trellis


def _predecessors(L: int, kV: int) -> np.ndarray:
    """pred[s, h]: the 2^kV states p whose low L-kV bits are s's high L-kV
    bits, ordered by p (h = p's top kV bits)."""
    s = np.arange(1 << L, dtype=np.int64)[:, None]
    h = np.arange(1 << kV, dtype=np.int64)[None, :]
    return (s >> kV) | (h << (L - kV))


def _step_costs(x: np.ndarray, values: np.ndarray, dtype) -> np.ndarray:
    """d[t, s] = sum_e (x[t, e] - values[s, e])^2 in the given precision."""
    x = x.astype(dtype)
    v = values.astype(dtype)
    d = np.zeros((x.shape[0], v.shape[0]), dtype=dtype)
    for e in range(x.shape[1]):
        diff = (x[:, e:e + 1] - v[None, :, e]).astype(dtype)
        d = (d + (diff * diff).astype(dtype)).astype(dtype)
    return d


def _viterbi(d: np.ndarray, pred: np.ndarray, L: int, kV: int, prefix, dtype):
    """Best walk over the steps of d [T, 2^L].  prefix None: free first state
    and free last state; else both ends tied to the prefix.  Returns (the last
    state, the path cost, the choice table [T, 2^L] of predecessor indices)."""
    T, S = d.shape
    keep = L - kV
    inf = np.array(np.inf, dtype=dtype)
    cost = d[0].copy()
    if prefix is not None:
        allowed = (np.arange(S, dtype=np.int64) >> kV) == prefix
        cost = np.where(allowed, cost, inf).astype(dtype)
    choice = np.zeros((T, S), dtype=np.int64)
    for t in range(1, T):
        cand = cost[pred]                       # [S, 2^kV]
        h = np.argmin(cand, axis=1)             # first minimum: the smallest predecessor
        cost = (cand[np.arange(S), h] + d[t]).astype(dtype)
        choice[t] = h
    if prefix is not None:
        ok = (np.arange(S, dtype=np.int64) & ((1 << keep) - 1)) == prefix
        cost = np.where(ok, cost, inf).astype(dtype)
    last = int(np.argmin(cost))                 # first minimum: the smallest state
    return last, cost[last], choice


def _backtrack(last: int, choice: np.ndarray, pred: np.ndarray) -> np.ndarray:
    T = choice.shape[0]
    states = np.empty(T, dtype=np.int64)
    s = last
    for t in range(T - 1, -1, -1):
        states[t] = s
        if t:
            s = int(pred[s, choice[t, s]])
    return states


def reconstruct(chunks: np.ndarray, L: int, kV: int, code: int, V: int, lut=None) -> np.ndarray:
    """Decoded values [T, V] of a block given its kV-bit chunks (the format's
    tail-biting walk, then the code)."""
    chunks = np.asarray(chunks, dtype=np.int64)
    T = chunks.shape[0]
    keep = L - kV
    # the block's last L-kV bits, from its last chunks
    bits = ((chunks[:, None] >> np.arange(kV - 1, -1, -1)[None, :]) & 1).reshape(-1)
    prefix = 0
    for b in bits[len(bits) - keep:] if keep else []:
        prefix = (prefix << 1) | int(b)
    states = trellis.walk_tailbiting(chunks[None, :], np.array([prefix]), L, kV)[0]
    return codes.evaluate(code, states, V, lut)


def _bits_per_step(k, V: int) -> int:
    """kV as an integer: k may be a half number of bits when V = 2."""
    kV = int(round(k * V))
    assert abs(k * V - kV) < 1e-12, "k*V must be a whole number of bits"
    return kV


def encode_exact(x, L: int, k, V: int, code: int, lut=None):
    """Minimum-squared-error tail-biting encoding of one block, float64.
    x: [T, V] source values (T steps).  Returns (chunks [T], squared error)."""
    x = np.asarray(x, dtype=np.float64).reshape(-1, V)
    kV = _bits_per_step(k, V)
    keep = L - kV
    pred = _predecessors(L, kV)
    values = codes.evaluate(code, np.arange(1 << L), V, lut)
    d = _step_costs(x, values, np.float64)
    best = None
    for p in range(1 << keep):
        last, cost, choice = _viterbi(d, pred, L, kV, p, np.float64)
        if best is None or cost < best[0]:
            best = (cost, _backtrack(last, choice, pred))
    states = best[1]
    return states & ((1 << kV) - 1), float(best[0])


def encode_two_pass(x, L: int, k, V: int, code: int, lut=None):
    """The two-pass tail-biting encoding (module docstring), float32 costs; the
    source is taken as float32.  Returns (chunks [T], squared error of the
    reconstruction against that source, in float64)."""
    x = np.asarray(x, dtype=np.float32).reshape(-1, V)
    kV = _bits_per_step(k, V)
    keep = L - kV
    pred = _predecessors(L, kV)
    values = codes.evaluate(code, np.arange(1 << L), V, lut)
    d = _step_costs(x, values, np.float32)
    last, _, _ = _viterbi(d, pred, L, kV, None, np.float32)
    prefix = last & ((1 << keep) - 1)
    last, _, choice = _viterbi(d, pred, L, kV, prefix, np.float32)
    states = _backtrack(last, choice, pred)
    chunks = states & ((1 << kV) - 1)
    err = float(np.sum((x.astype(np.float64) - reconstruct(chunks, L, kV, code, V, lut)) ** 2))
    return chunks, err
