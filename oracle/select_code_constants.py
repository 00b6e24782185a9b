"""Record of how the multiply-add constants of the three codes were chosen.

The pages state properties of the codes but print no constants (QTIP
discussion: computed codes "do a good job of decorrelating the state ID from
the computed value", are "approximately Gaussian for large enough L", and
1MAD/3INST give "very similar coverage as a random Gaussian" at L = 16).
This script walks a seeded stream of candidate (A, B) pairs (A odd) and keeps,
for each code, the first pair that meets every threshold below at L = 16.
Its output is what oracle/codes.py holds; the CUDA sources carry their own
copy of the same numbers.

Thresholds (over all 2^16 states):
  1MAD, 3INST:  |mean| < 0.02, |var - 1| < 0.05, KS distance to N(0,1) < 0.03;
                for kV in 1..4: |pearson| < 0.05, mutual information < 0.05 bit,
                successor spread ratio < 1.5.
  HYB (Q = 9, with the seed-2 table, V = 1 and V = 2):
                every index used, max/min index count < 2, flip bit balanced
                within 1%, all 2^(Q+1) (index, flip) pairs reachable; for each
                value position and kV in 1..4 (V=1) or 2,4,6,8 (V=2): the same
                three neighbour thresholds.

Run:  python -m oracle.select_code_constants
"""
from __future__ import annotations

import numpy as np

from . import codes, stats

SEARCH_SEED = 20240607
L = 16


def _neighbour_ok(values, kVs):
    for kV in kVs:
        if abs(stats.pearson(values, L, kV)) >= 0.05:
            return False
        if stats.mutual_information(values, L, kV) >= 0.05:
            return False
        if stats.successor_spread_ratio(values, L, kV) >= 1.5:
            return False
    return True


def computed_code_ok(fn) -> bool:
    v = fn(np.arange(1 << L))
    m, var, _ = stats.moments(v)
    if abs(m) >= 0.02 or abs(var - 1) >= 0.05:
        return False
    if stats.normal_ks(v[::4]) >= 0.03:
        return False
    return _neighbour_ok(v, (1, 2, 3, 4))


def hyb_ok(Q=9) -> bool:
    s = np.arange(1 << L)
    idx, flip = codes.hyb_index(s, Q)
    cnt = np.bincount(idx, minlength=1 << Q)
    if cnt.min() == 0 or cnt.max() / cnt.min() >= 2:
        return False
    if abs(flip.mean() - 0.5) >= 0.01:
        return False
    if len(np.unique(idx * 2 + flip)) != 1 << (Q + 1):
        return False
    for V, kVs in ((1, (1, 2, 3, 4)), (2, (2, 4, 6, 8))):
        lut = np.random.default_rng(2).standard_normal((1 << Q, V)).astype(np.float16)
        vals = codes.hyb(s, lut)
        for e in range(V):
            if not _neighbour_ok(vals[:, e], kVs):
                return False
    return True


def search(max_tries=2000):
    rng = np.random.default_rng(SEARCH_SEED)
    chosen = {}
    for name, attr, test in (("1MAD", "1MAD", lambda: computed_code_ok(codes.one_mad)),
                             ("3INST", "3INST", lambda: computed_code_ok(codes.three_inst)),
                             ("HYB", "HYB", hyb_ok)):
        saved = (getattr(codes, f"A_{attr}"), getattr(codes, f"B_{attr}"))
        for tries in range(1, max_tries + 1):
            A = int(rng.integers(0, 2**32)) | 1
            B = int(rng.integers(0, 2**32))
            setattr(codes, f"A_{attr}", A)
            setattr(codes, f"B_{attr}", B)
            if test():
                chosen[name] = (A, B, tries)
                break
        setattr(codes, f"A_{attr}", saved[0])
        setattr(codes, f"B_{attr}", saved[1])
    return chosen


if __name__ == "__main__":
    for name, (A, B, tries) in search().items():
        print(f"{name}: A=0x{A:08X} B=0x{B:08X} (candidate {tries})")
