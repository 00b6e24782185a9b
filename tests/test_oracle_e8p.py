"""Pins of the oracle's E8-lattice codebook (QuIP# page, abstract and Fig. 3
caption: codebooks built on the E8 lattice, 2^16 entries of dimension 8 at 2
bits per weight; QTIP discussion, "Inference speed analysis (W2)").

Textbook facts about E8 used here: E8 = D8 u (D8 + 1/2), its vectors of
squared norm 2 number 240 (the kissing number: 112 of shape (+-1, +-1, 0^6)
and 128 of shape (+-1/2)^8 with an even number of minus signs) and those of
squared norm 4 number 2160 (the theta series 1 + 240 q + 2160 q^2 + ...)."""
import itertools
from math import comb

import numpy as np
import pytest

import workloads as wl
from oracle import bitstream, codes, e8p, qlinear


def _grid(values):
    return np.array(list(itertools.product(values, repeat=8)), dtype=np.float64)


@pytest.fixture(scope="module")
def candidates():
    # every integer vector with coordinates in [-2, 2] and every half-odd one
    # with coordinates in [-3/2, 3/2]: all E8 vectors of squared norm <= 4 lie here
    return np.concatenate([_grid((-2, -1, 0, 1, 2)), _grid((-1.5, -0.5, 0.5, 1.5))])


def test_membership_gives_the_first_shells_of_e8(candidates):
    inside = e8p.is_e8(candidates)
    norm2 = np.sum(candidates ** 2, axis=1)
    assert int(np.sum(inside & (norm2 == 0))) == 1
    assert int(np.sum(inside & (norm2 == 2))) == 240
    assert int(np.sum(inside & (norm2 == 4))) == 2160
    half = np.all(np.abs(candidates) == 0.5, axis=1)
    assert int(np.sum(inside & half)) == 128  # even number of minus signs


def test_membership_rejects_the_neighbours():
    assert e8p.is_e8(np.array([1, 1, 0, 0, 0, 0, 0, 0.0]))
    assert not e8p.is_e8(np.array([1, 0, 0, 0, 0, 0, 0, 0.0]))          # odd sum
    assert not e8p.is_e8(np.array([0.5] * 7 + [-0.5]))                   # odd sum of halves
    assert not e8p.is_e8(np.array([1, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5]))  # mixed cosets
    assert not e8p.is_e8(np.array([0.25] * 8))                           # not a half-integer


def test_shape_table_is_the_smallest_norm_half_integer_shapes():
    T = e8p.shape_table()
    n = np.round(2 * T).astype(int)
    assert T.shape == (256, 8) and len({tuple(r) for r in n}) == 256
    assert np.all(n % 2 == 1) and np.all(n > 0)
    # shells of squared norm 2, 4, ..., 10 are complete: j coordinates at 3/2 and
    # the rest at 1/2 (C(8, j)), plus one coordinate at 5/2 from norm 8 on
    shell = np.sum(T ** 2, axis=1)
    want = {2: 1, 4: comb(8, 1), 6: comb(8, 2), 8: comb(8, 3) + 8, 10: comb(8, 4) + 8 * 7}
    for norm, count in want.items():
        assert int(np.sum(shell == norm)) == count
    # the rest come from the squared-norm-12 shell (five 3/2, or one 5/2 and two
    # 3/2), the lexicographically smallest of 2T first
    rest = sum(want.values())
    shell12 = sorted([tuple(v) for v in itertools.permutations((3, 3, 3, 3, 3, 1, 1, 1))] +
                     [tuple(v) for v in itertools.permutations((5, 3, 3, 1, 1, 1, 1, 1))])
    shell12 = sorted(set(shell12))
    assert len(shell12) == comb(8, 5) + 8 * comb(7, 2)
    assert [tuple(r) for r in n[rest:]] == shell12[:256 - rest]
    assert np.all(np.diff(shell) >= 0)


def test_every_codeword_is_a_shifted_e8_point_and_the_set_is_symmetric():
    s = np.arange(1 << 16)
    cw = e8p.codeword(s)
    shift = np.where(s & 1, 0.25, -0.25)[:, None]
    assert np.all(e8p.is_e8(cw - shift))
    assert len(np.unique(cw, axis=0)) == 1 << 16
    as_set = {tuple(r) for r in cw}
    assert all(tuple(-r) in as_set for r in cw[::97])
    assert float(cw.mean()) == 0.0
    # shape 0 is (1/2)^8: with its sign patterns it gives E8's 128 minimal
    # half-integer vectors, once per shift
    d = cw - shift
    assert int(np.sum(np.sum(d ** 2, axis=1) == 2)) == 2 * 128


def test_values_are_exact_in_fp16():
    cw = e8p.codeword(np.arange(1 << 16))
    assert np.all(cw * 4 == np.round(cw * 4)) and np.max(np.abs(cw)) < 4
    assert np.array_equal(codes.evaluate(4, np.arange(8), 8), cw[:8])


def test_a_layer_with_the_e8_code_is_plain_vq_on_16_bit_steps():
    """With L = kV = 16 and V = 8, step t of a block is the codeword of the
    step's own 16 bits: columns 8t .. 8t+7."""
    li = wl.random_layer(16, 512, 2, 16, 8, wl.CODE_E8P, seed=5)
    layer = qlinear.Layer.from_inputs(li)
    rows = np.array([0, 7, 15])
    W = layer.decode_rows(rows)
    base, _ = bitstream.row_base_bits(rows, 512, layer.parts)
    for ri, r in enumerate(rows):
        for t in range(512 // 8):
            j, tt = divmod(t, 32)
            idx = int(bitstream.field(li.codes, base[ri] + j * 512 + tt * 16, 16))
            assert np.array_equal(W[ri, 8 * t:8 * t + 8], e8p.codeword(idx))
