"""Statistics of a code over all 2^L states (used by the code pins).

QTIP discussion, reply on computed codes: the codes are approximately
Gaussian for L >~ 10, and "a poorly designed computed code will have strong
correlations that result in unrepresentable neighboring values" because
neighbouring states in the bitshift trellis share L-kV bits (the FP8-cast
example).  Three measures of that dependence between the value of a state s
and the values of its successors s' = ((s << kV) | c) mod 2^L:

  * pearson:    linear correlation of (v(s), v(s')) over all s and all c.
  * mutual_information: in bits, of (v(s), v(s')) on a quantile grid.
  * successor_spread_ratio: the successors of s are the 2^kV states sharing
    their high L-kV bits.  For a random code the variance of the group means
    is Var(v)/2^kV, so Var(group means) * 2^kV / Var(v) is ~1; a code whose
    successors of a state crowd into one region of the value range (the FP8
    example) gives a ratio well above 1.
"""
from __future__ import annotations

import numpy as np


def moments(v):
    v = np.asarray(v, dtype=np.float64)
    m = v.mean()
    var = v.var()
    kurt = ((v - m) ** 4).mean() / var ** 2
    return float(m), float(var), float(kurt)


def successor_pairs(values: np.ndarray, L: int, kV: int):
    """(v(s), v(s')) for every state s and every kV-bit chunk c."""
    s = np.arange(1 << L, dtype=np.int64)
    c = np.arange(1 << kV, dtype=np.int64)
    s2 = ((s[:, None] << kV) | c[None, :]) & ((1 << L) - 1)
    return np.repeat(values, 1 << kV), values[s2.reshape(-1)]


def pearson(values, L, kV):
    a, b = successor_pairs(values, L, kV)
    return float(np.corrcoef(a, b)[0, 1])


def mutual_information(values, L, kV, bins=16):
    a, b = successor_pairs(values, L, kV)
    qa = np.quantile(a, np.linspace(0, 1, bins + 1)[1:-1])
    qb = np.quantile(b, np.linspace(0, 1, bins + 1)[1:-1])
    ia = np.searchsorted(qa, a, side="right")
    ib = np.searchsorted(qb, b, side="right")
    h = np.zeros((bins, bins))
    np.add.at(h, (ia, ib), 1.0)
    p = h / h.sum()
    pa = p.sum(1, keepdims=True)
    pb = p.sum(0, keepdims=True)
    nz = p > 0
    return float((p[nz] * np.log2(p[nz] / (pa @ pb)[nz])).sum())


def successor_spread_ratio(values, L, kV):
    v = np.asarray(values, dtype=np.float64)
    assert v.shape == (1 << L,)
    # states s' with the same high L-kV bits are consecutive integers
    groups = v.reshape(-1, 1 << kV)
    return float(groups.mean(axis=1).var() * (1 << kV) / v.var())


def normal_ks(values):
    """Kolmogorov-Smirnov distance of the empirical distribution to N(0,1)."""
    from math import erf, sqrt
    s = np.sort(np.asarray(values, dtype=np.float64))
    n = len(s)
    F = 0.5 * (1.0 + np.vectorize(erf)(s / sqrt(2.0)))
    return float(max(np.max(np.arange(1, n + 1) / n - F), np.max(F - np.arange(n) / n)))
