"""Pins of the oracle's palette quantizers: fractional bitwidths and the table code.

Sources: the Q-Palette page (fractional-bit quantizers such as 2.5 and 3.75
bits; TCQ, VQ and NUQ in one palette; half-TCQ's 2.75 bits from a 2.5-bit and
a 3-bit quantizer) and the QTIP discussion's ablation reply (a trellis with
L = kV is plain k-bit, V-dimensional VQ).

Each check restates the layout from a plain bit string ("0"/"1" characters,
most significant bit of each word first) with its own offsets, independent of
oracle.bitstream's field arithmetic:
  * fractional rows: row r of a k-bit layer starts at bit r*n*k, block j at
    r*n*k + 256*k*j, and step t's state is the cyclic L-bit window ending at
    bit (t+1)*kV of its block, for half-integer k (odd kV at V = 2);
  * the table code with L = kV is a field lookup: step t's V values are the
    codebook row indexed by the step's own kV bits (VQ at V = 2, NUQ at V = 1);
  * a codebook filled with the HYB code's values on every state decodes
    exactly as HYB (the table code is HYB without its hash);
  * a layer of fractional parts is the stack of its single-part layers.
"""
import numpy as np
import pytest

import workloads as wl
from oracle import codes, hadamard, qlinear, trellis


def _bitstring(words):
    return "".join(f"{int(w):032b}" for w in words)


def _cyclic_window(bits, end, L):
    S = len(bits)
    return int("".join(bits[p % S] for p in range(end - L, end)), 2)


@pytest.mark.parametrize("L,k,V", [(16, 2.5, 2), (16, 1.5, 2), (16, 3.5, 2), (7, 3.5, 2), (5, 2.5, 2)])
def test_fractional_states_are_cyclic_windows(L, k, V):
    rng = np.random.default_rng(int(L * 10 + 2 * k))
    n, rows = 512, 3
    kV = int(round(k * V))
    row_bits = n * kV // V
    words = rng.integers(0, 2**32, size=rows * row_bits // 32, dtype=np.uint32)
    st = trellis.block_states(words, np.arange(rows), n, [(0, rows, k)], L, V)
    full = _bitstring(words)
    S = 256 * kV // V
    for r in range(rows):
        for j in range(n // 256):
            blk = full[r * row_bits + j * S: r * row_bits + (j + 1) * S]
            assert len(blk) == S
            for t in range(0, 256 // V, 5):
                assert st[r, j, t] == _cyclic_window(blk, (t + 1) * kV, L)


@pytest.mark.parametrize("kV,V", [(1, 1), (2, 1), (3, 1), (4, 1), (2, 2), (3, 2), (5, 2), (8, 2)])
def test_memoryless_table_code_is_a_field_lookup(kV, V):
    m, n = 16, 512
    li = wl.random_layer(m, n, kV / V, kV, V, wl.CODE_TABLE, seed=40 + kV * 3 + V)
    layer = qlinear.Layer.from_inputs(li)
    assert li.lut.shape == (1 << kV, V)
    book = li.lut.astype(np.float64)
    W = layer.decode_rows(np.arange(m))
    full = _bitstring(li.codes)
    row_bits = n * kV // V
    for r in (0, 7, 15):
        for col in range(0, n, 3):
            j, t, e = col // 256, (col % 256) // V, col % V
            p = r * row_bits + j * (256 * kV // V) + t * kV
            assert W[r, col] == book[int(full[p:p + kV], 2), e]


def test_nuq_levels_are_sorted_and_every_weight_is_a_level():
    li = wl.make_layer(wl.WORKLOADS["nuq3"])
    levels = li.lut[:, 0].astype(np.float64)
    assert len(levels) == 8 and np.all(np.diff(levels) >= 0)
    W = qlinear.Layer.from_inputs(li).decode_rows(np.arange(4))
    assert set(np.unique(W)).issubset(set(levels))


def test_table_filled_with_hyb_values_decodes_as_hyb():
    """HYB = hash, table lookup, sign flip; a 2^L codebook holding the HYB
    value of every L-bit state turns the table code into HYB."""
    L, V, k = 8, 2, 2.5
    li = wl.random_layer(16, 512, k, L, V, wl.CODE_HYB, seed=12, Q=6)
    hyb_layer = qlinear.Layer.from_inputs(li)
    book = codes.hyb(np.arange(1 << L), li.lut).astype(np.float16)
    assert np.array_equal(book.astype(np.float64), codes.hyb(np.arange(1 << L), li.lut))  # fp16-exact
    tab_layer = qlinear.Layer(16, 512, [(0, 16, k)], L, V, wl.CODE_TABLE, li.codes, li.s_in, li.s_out, 1.0, book)
    assert np.array_equal(tab_layer.decode_rows(np.arange(16)), hyb_layer.decode_rows(np.arange(16)))


def test_layer_of_fractional_parts_is_the_stack_of_its_parts():
    split = ((16, 2.5), (32, 3), (16, 1.5))
    V, n = 2, 512
    li = wl.random_layer(64, n, 0, 16, V, wl.CODE_HYB, 5, Q=9, row_split=split)
    layer = qlinear.Layer.from_inputs(li)
    W = layer.decode_rows(np.arange(64))
    off, r0 = 0, 0
    for rows, k in split:
        nw = int(rows * n * k) // 32
        single = qlinear.Layer(rows, n, [(0, rows, k)], 16, V, wl.CODE_HYB, li.codes[off:off + nw], li.s_in,
                               li.s_out[r0:r0 + rows], 1.0, li.lut)
        assert np.array_equal(W[r0:r0 + rows], single.decode_rows(np.arange(rows)))
        off += nw
        r0 += rows
    assert off == len(li.codes)
    assert li.spec.bits_per_weight == (16 * 2.5 + 32 * 3 + 16 * 1.5) / 64


def test_palette_bit_accounting():
    """Stream = m n k bits at the fractional bitwidths; the codebooks add
    under 0.001 bits per weight."""
    want = {"tcq2p5": 2.5, "tcq2p75": 2.75, "vq2p5": 2.5, "nuq3": 3.0}
    for name, bpw in want.items():
        sp = wl.WORKLOADS[name]
        assert sp.n_words * 32 == int(sp.m * sp.n * bpw)
        assert sp.bits_per_weight == bpw
        table_bits = ((1 << sp.Q) if sp.code == wl.CODE_HYB else (1 << sp.L)) * sp.V * 16
        assert table_bits / (sp.m * sp.n) < 0.001
    assert wl.WORKLOADS["tcq2p5"].part_kv() == [5]
    assert wl.WORKLOADS["tcq2p75"].part_kv() == [5, 6]


@pytest.mark.parametrize("k,L,V,code", [(2.5, 16, 2, wl.CODE_HYB), (2.5, 5, 2, wl.CODE_TABLE),
                                        (3, 3, 1, wl.CODE_TABLE), (1.5, 8, 2, wl.CODE_TABLE)])
def test_fractional_and_table_forward_equals_dense_weight(k, L, V, code):
    m, n = 32, 512
    li = wl.random_layer(m, n, k, L, V, code, seed=int(10 * k) + L, alpha=0.61)
    layer = qlinear.Layer.from_inputs(li)

    def kron_h(d):
        B = hadamard.block_size(d)
        H = np.array([[1.0]])
        while H.shape[0] < B:
            H = np.block([[H, H], [H, -H]])
        return np.kron(np.eye(d // B), H / np.sqrt(B))

    What = layer.decode_rows(np.arange(m))
    W = layer.alpha * (layer.s_out[:, None] * (kron_h(m) @ What @ kron_h(n))) * layer.s_in[None, :]
    x = np.random.default_rng(2).standard_normal((3, n)).astype(np.float16)
    assert np.allclose(layer.forward(x), x.astype(np.float64) @ W.T, rtol=1e-10, atol=1e-10)
