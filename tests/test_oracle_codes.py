"""Pins of the oracle's codes against the properties the pages state.

QTIP OpenReview discussion:
  * reply on computed codes: the codes are approximately Gaussian for
    L >~ 10 (experiments use L = 16), and must decorrelate a state from the
    states it can move to, unlike an FP8-cast code whose neighbouring values
    are strongly tied (the printed scatter script, L = 8, K = 4);
  * "Inference speed analysis" comment and "Bit Accounting (Q2)": HYB stores
    2^Q x V fp16 values (Q = 9, V = 2: 512 x 32-bit words, 2 KiB) and
    decompresses them to 1024 effective entries.
"""
import struct

import numpy as np
import pytest

from oracle import codes, fp16, stats

L = 16
S = np.arange(1 << L)


@pytest.mark.parametrize("fn", [codes.one_mad, codes.three_inst], ids=["1MAD", "3INST"])
def test_computed_code_is_close_to_standard_normal(fn):
    v = fn(S)
    mean, var, kurt = stats.moments(v)
    assert abs(mean) < 0.02
    assert abs(var - 1.0) < 0.05
    assert 2.4 < kurt < 3.6
    assert stats.normal_ks(v[::4]) < 0.03


@pytest.mark.parametrize("fn", [codes.one_mad, codes.three_inst], ids=["1MAD", "3INST"])
@pytest.mark.parametrize("kV", [1, 2, 3, 4])
def test_computed_code_decorrelates_neighbours(fn, kV):
    v = fn(S)
    assert abs(stats.pearson(v, L, kV)) < 0.05
    assert stats.mutual_information(v, L, kV) < 0.05
    assert stats.successor_spread_ratio(v, L, kV) < 1.5


@pytest.mark.parametrize("kV", [2, 4])
def test_fp8_cast_code_fails_the_neighbour_test(kV):
    """Negative control: casting the 8-bit state to FP8 e5m2 (the top byte of
    a binary16 pattern) ties a state's successors together."""
    v = fp16.decode_bits(np.arange(256) << 8)
    v = np.where(np.isfinite(v), v, 0.0)
    assert stats.successor_spread_ratio(v, 8, kV) > 3.0


def test_random_gaussian_code_passes_the_neighbour_test():
    """Positive control: a table of i.i.d. normals over 2^16 states."""
    v = np.random.default_rng(1).standard_normal(1 << L)
    for kV in (1, 2, 3, 4):
        assert stats.successor_spread_ratio(v, L, kV) < 1.5
        assert stats.mutual_information(v, L, kV) < 0.05


def test_1mad_is_an_irwin_hall_sum_of_four_bytes():
    """1MAD: the value is fp16(d * C1) with d + 510 a sum of four uniform
    bytes, so d lies in [-510, 510] and its histogram over all states follows
    the closed-form Irwin-Hall distribution of 4 bytes (mean 0, variance
    21845)."""
    v = codes.one_mad(S)
    d = np.rint(v / codes.C1).astype(np.int64)
    assert d.min() >= -510 and d.max() <= 510
    assert np.all(np.abs(v - d * codes.C1) <= np.abs(d * codes.C1) * 2.0 ** -11 + 1e-12)
    # closed form: ways to write u = d + 510 as a sum of 4 bytes
    one = np.ones(256)
    pmf = np.convolve(np.convolve(one, one), np.convolve(one, one)) / 256.0 ** 4
    emp = np.bincount(d + 510, minlength=1021) / len(d)
    assert 0.5 * np.abs(emp - pmf).sum() < 0.05
    assert abs(np.dot(np.arange(1021) - 510, pmf)) < 1e-9
    assert abs(np.dot((np.arange(1021) - 510.0) ** 2, pmf) - 21845.0) < 1e-6
    assert abs(codes.C1 - 1 / np.sqrt(21845)) < 2.0 ** -17


def test_3inst_halves_are_finite_and_bounded():
    x = codes.lcg(S, codes.A_3INST, codes.B_3INST).astype(np.int64)
    m = (x & codes.MASK_3INST) ^ codes.XOR_3INST
    for half in (m & 0xFFFF, m >> 16):
        h = fp16.decode_bits(half)
        assert np.all(np.isfinite(h)) and np.all(np.abs(h) < 2.0) and np.all(np.abs(h) >= 2.0 ** -7)
    v = codes.three_inst(S)
    assert np.all(np.abs(v) < 4.0)


def _scalar_reference(code, s, lut=None):
    """Scalar restatement with Python integers and struct's binary16 codec."""
    def f16(bits):
        return struct.unpack("<e", struct.pack("<H", bits & 0xFFFF))[0]

    def r16(val):
        return struct.unpack("<e", struct.pack("<e", val))[0]
    if code == "1MAD":
        x = (codes.A_1MAD * s + codes.B_1MAD) % 2**32
        d = sum((x >> (8 * i)) & 255 for i in range(4)) - 510
        return [r16(d * 443 / 65536)]
    if code == "3INST":
        x = (codes.A_3INST * s + codes.B_3INST) % 2**32
        m = (x & codes.MASK_3INST) ^ codes.XOR_3INST
        return [r16(f16(m) + f16(m >> 16))]
    x = (codes.A_HYB * s + codes.B_HYB) % 2**32
    entry = [float(e) for e in lut[x >> 23]]
    if (x >> 15) & 1:
        entry[0] = -entry[0]
    return entry


def test_vectorised_codes_match_a_scalar_restatement():
    lut = np.random.default_rng(2).standard_normal((512, 2)).astype(np.float16)
    picks = np.random.default_rng(3).integers(0, 1 << L, 300)
    picks = np.concatenate([picks, [0, 1, 0xFFFF, 0x8000]])
    for s in picks:
        s = int(s)
        assert [codes.one_mad(np.array([s]))[0]] == _scalar_reference("1MAD", s)
        assert [codes.three_inst(np.array([s]))[0]] == _scalar_reference("3INST", s)
        assert list(codes.hyb(np.array([s]), lut)[0]) == _scalar_reference("HYB", s, lut)


def test_hyb_table_decompresses_to_1024_entries():
    Q, V = 9, 2
    lut = np.random.default_rng(2).standard_normal((1 << Q, V)).astype(np.float16)
    assert lut.nbytes == 2048                       # 512 x 32-bit words = 2 KiB
    idx, flip = codes.hyb_index(S, Q)
    assert len(np.unique(idx * 2 + flip)) == 1024   # every (entry, sign) pair is reachable
    vals = codes.hyb(S, lut)
    assert len(np.unique(vals, axis=0)) == 1024
    # a degenerate table cannot exceed 2^(Q+1) distinct pairs either
    lut2 = np.zeros_like(lut)
    lut2[:, 0] = 1.0
    assert len(np.unique(codes.hyb(S, lut2), axis=0)) == 2


def test_hyb_flip_negates_first_value_only():
    lut = np.arange(1, 1 + 512 * 2, dtype=np.float64).reshape(512, 2).astype(np.float16)
    idx, flip = codes.hyb_index(S, 9)
    vals = codes.hyb(S, lut)
    base = lut.astype(np.float64)[idx]
    assert np.array_equal(vals[:, 1], base[:, 1])
    assert np.array_equal(vals[:, 0], np.where(flip == 1, -base[:, 0], base[:, 0]))
    assert 0.49 < flip.mean() < 0.51
