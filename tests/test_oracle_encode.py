"""Pins for the trellis-coded quantization oracle (oracle/encode.py).

- The exact tail-biting Viterbi is the true minimum: it equals brute force over
  every bit string of tiny blocks.
- The two-pass search is never better than the exact minimum.
- With L = kV (no memory, plain kV-bit V-dimensional VQ: "When L = KV, TCQ
  becomes K bit V dim VQ") both reduce to the nearest codeword at every step.
- The encoded chunks, packed MSB-first into a block of the stream format, decode
  through the layer oracle to the reconstruction the encoder scored.
- On an i.i.d. N(0,1) source the distortion lies between the Gaussian
  rate-distortion bound D(k) = 2^(-2k) and the optimal k-bit scalar (Lloyd-Max)
  quantizer's distortion (0.3634 for 1 bit, 0.1175 for 2 bits: textbook
  values), as the discussion's "Table 1" replies describe; a larger trellis
  does better ("Larger trellises improve quality").
- The two-pass search's costs follow its float32 rule."""
import itertools

import numpy as np
import pytest

import workloads as wl
from oracle import bitstream, codes, encode, qlinear

LLOYD_MAX = {1: 1.0 - 2.0 / np.pi, 2: 0.1175}


def _brute_force(x, L, k, V, code, lut=None):
    T = x.shape[0]
    kV = int(k * V)
    best = None
    for bits in itertools.product((0, 1), repeat=T * kV):
        chunks = np.array([int("".join(map(str, bits[t * kV:(t + 1) * kV])), 2) for t in range(T)])
        err = float(np.sum((x - encode.reconstruct(chunks, L, kV, code, V, lut)) ** 2))
        if best is None or err < best:
            best = err
    return best


def _lut(code, L, V, seed):
    if code == wl.CODE_HYB:
        return wl.hyb_table(4, V, seed)
    if code == wl.CODE_TABLE:
        return wl.palette_table(L, V, seed)
    return None


@pytest.mark.parametrize("L,k,V,code,T", [(4, 1, 1, wl.CODE_3INST, 8), (4, 2, 1, wl.CODE_1MAD, 4),
                                          (6, 1, 2, wl.CODE_HYB, 4), (5, 1, 1, wl.CODE_1MAD, 9),
                                          (5, 1.5, 2, wl.CODE_HYB, 4), (6, 1.5, 2, wl.CODE_TABLE, 4),
                                          (4, 1, 1, wl.CODE_TABLE, 7)])
def test_exact_viterbi_equals_brute_force(L, k, V, code, T):
    rng = np.random.default_rng(int(L * 100 + k * 10 + V + T))
    lut = _lut(code, L, V, 7)
    kV = int(k * V)
    for _ in range(3):
        x = rng.standard_normal((T, V))
        chunks, err = encode.encode_exact(x, L, k, V, code, lut)
        assert err == pytest.approx(_brute_force(x, L, k, V, code, lut), rel=1e-12, abs=1e-12)
        recon = encode.reconstruct(chunks, L, kV, code, V, lut)
        assert float(np.sum((x - recon) ** 2)) == pytest.approx(err, rel=1e-12, abs=1e-12)


def test_two_pass_is_never_better_than_the_exact_minimum():
    rng = np.random.default_rng(3)
    for L, k in [(6, 1), (6, 2), (8, 2)]:
        for _ in range(4):
            x = rng.standard_normal((32, 1))
            _, exact = encode.encode_exact(x, L, k, 1, wl.CODE_3INST)
            _, two = encode.encode_two_pass(x, L, k, 1, wl.CODE_3INST)
            assert two >= exact * (1 - 1e-6)


@pytest.mark.parametrize("k,V,code", [(2, 1, wl.CODE_3INST), (3, 1, wl.CODE_1MAD), (2, 2, wl.CODE_HYB),
                                      (2.5, 2, wl.CODE_TABLE), (3, 1, wl.CODE_TABLE)])
def test_memoryless_trellis_is_nearest_codeword_vq(k, V, code):
    """L = kV: every state is its own chunk, so both searches pick the nearest
    codeword at every step (VQ at V = 2, NUQ at V = 1 with the table code)."""
    L = int(k * V)
    lut = wl.hyb_table(4, V, 5) if code == wl.CODE_HYB else (wl.palette_table(L, V, 5) if code == wl.CODE_TABLE else None)
    rng = np.random.default_rng(int(2 * k) + V)
    x = rng.standard_normal((40, V))
    book = codes.evaluate(code, np.arange(1 << L), V, lut)                  # [2^L, V]
    nearest = np.argmin(((x[:, None, :] - book[None, :, :]) ** 2).sum(-1), axis=1)
    for enc in (encode.encode_exact, encode.encode_two_pass):
        chunks, _ = enc(x, L, k, V, code, lut)
        assert np.array_equal(chunks, nearest)


def test_encoded_block_decodes_through_the_layer_format():
    L, k, V, code = 16, 2, 1, wl.CODE_3INST
    rng = np.random.default_rng(11)
    x = rng.standard_normal((256, 1))                    # one 256-column block
    chunks, err = encode.encode_two_pass(x, L, k, V, code)
    bits = "".join(format(int(c), f"0{k * V}b") for c in chunks)
    words = bitstream.bits_to_words(bits)
    layer = qlinear.Layer(1, 256, [(0, 1, k)], L, V, code, words, np.ones(256, np.int8), np.ones(1, np.int8), 1.0)
    w = layer.decode_rows(np.arange(1))[0]
    assert np.array_equal(w, encode.reconstruct(chunks, L, k * V, code, V).reshape(-1))
    x32 = x[:, 0].astype(np.float32).astype(np.float64)  # the two-pass search takes the source as float32
    assert float(np.sum((x32 - w) ** 2)) == pytest.approx(err, rel=1e-12)


def test_fractional_block_decodes_through_the_layer_format():
    """A 2.5-bit block (V = 2, 5 bits per step) packed MSB-first decodes
    through the layer oracle to the reconstruction the encoder scored."""
    L, k, V, code = 12, 2.5, 2, wl.CODE_HYB
    lut = wl.hyb_table(9, V, 4)
    x = np.random.default_rng(13).standard_normal((128, 2))
    chunks, err = encode.encode_two_pass(x, L, k, V, code, lut)
    bits = "".join(format(int(c), "05b") for c in chunks)
    assert len(bits) == 640
    words = bitstream.bits_to_words(bits)
    layer = qlinear.Layer(1, 256, [(0, 1, k)], L, V, code, words, np.ones(256, np.int8), np.ones(1, np.int8), 1.0,
                          lut)
    w = layer.decode_rows(np.arange(1))[0]
    assert np.array_equal(w, encode.reconstruct(chunks, L, 5, code, V, lut).reshape(-1))
    x32 = x.astype(np.float32).astype(np.float64).reshape(-1)
    assert float(np.sum((x32 - w) ** 2)) == pytest.approx(err, rel=1e-12)


@pytest.mark.parametrize("k", [1, 2])
def test_gaussian_distortion_between_the_bound_and_scalar_quantization(k):
    rng = np.random.default_rng(20 + k)
    x = rng.standard_normal((4, 256, 1))
    mse = np.mean([encode.encode_two_pass(b, 12, k, 1, wl.CODE_3INST)[1] / b.size for b in x])
    assert 2.0 ** (-2 * k) < mse < LLOYD_MAX[k]


def test_larger_trellis_lowers_the_distortion():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 256, 1))
    mse = {L: np.mean([encode.encode_two_pass(b, L, 2, 1, wl.CODE_3INST)[1] / b.size for b in x]) for L in (8, 16)}
    assert mse[16] < mse[8]
    assert mse[16] > 2.0 ** -4


@pytest.mark.parametrize("k,levels,mse", [(1, [-0.7979, 0.7979], 1.0 - 2.0 / np.pi),
                                          (2, [-1.5104, -0.4528, 0.4528, 1.5104], 0.1175)])
def test_nuq_with_lloyd_max_levels_reaches_the_lloyd_max_distortion(k, levels, mse):
    """The palette's NUQ member (table code, L = kV, V = 1) with the optimal
    k-bit scalar quantizer's levels for N(0,1) as its codebook (textbook
    Lloyd-Max values, rounded to fp16) quantizes N(0,1) samples to its
    textbook distortion, within four standard errors of the sample mean."""
    book = np.array(levels, dtype=np.float16).reshape(-1, 1)
    x = np.random.default_rng(30 + k).standard_normal((400, 256, 1)).astype(np.float32)
    per_block = np.array([encode.encode_two_pass(b, k, k, 1, wl.CODE_TABLE, book)[1] / b.size for b in x])
    sem = per_block.std(ddof=1) / np.sqrt(len(per_block))
    assert abs(per_block.mean() - mse) < 4 * sem + 1e-3


def test_vq_with_a_product_codebook_is_per_dimension_scalar_quantization():
    """The palette's VQ member (table code, L = kV, V = 2) with the product of
    the 2-bit Lloyd-Max quantizer (first value of a pair) and the 1-bit one
    (second value) as its 8-pair codebook, 1.5 bits per weight: the nearest
    pair is the pair of per-dimension nearest levels, so the reconstruction
    matches per-dimension scalar quantization, and the distortion per weight
    is the mean of the two Lloyd-Max values.  The two coordinates use
    different level sets, so a pair read in the wrong order fails."""
    lv2 = np.array([-1.5104, -0.4528, 0.4528, 1.5104], dtype=np.float16)
    lv1 = np.array([-0.7979, 0.7979], dtype=np.float16)
    book = np.array([[a, b] for a in lv2 for b in lv1], dtype=np.float16)      # entry 2i + j = (lv2[i], lv1[j])
    x = np.random.default_rng(44).standard_normal((100, 128, 2)).astype(np.float32)
    same, per_block = 0, []
    for blk in x:
        chunks, err = encode.encode_two_pass(blk, 3, 1.5, 2, wl.CODE_TABLE, book)
        recon = encode.reconstruct(chunks, 3, 3, wl.CODE_TABLE, 2, book)
        xb = blk.astype(np.float64)
        n0 = lv2.astype(np.float64)[np.argmin(np.abs(xb[:, :1] - lv2.astype(np.float64)[None, :]), axis=1)]
        n1 = lv1.astype(np.float64)[np.argmin(np.abs(xb[:, 1:] - lv1.astype(np.float64)[None, :]), axis=1)]
        same += int(np.sum((recon[:, 0] == n0) & (recon[:, 1] == n1)))
        per_block.append(err / blk.size)
    assert same / (x.shape[0] * x.shape[1]) > 0.999
    per_block = np.array(per_block)
    want = (0.1175 + (1.0 - 2.0 / np.pi)) / 2
    assert abs(per_block.mean() - want) < 4 * per_block.std(ddof=1) / np.sqrt(len(per_block)) + 1e-3


def test_two_pass_costs_follow_the_float32_rule():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 2))
    values = rng.standard_normal((5, 2))
    d = encode._step_costs(x, values, np.float32)
    for t in range(3):
        for s in range(5):
            acc = np.float32(0)
            for e in range(2):
                diff = np.float32(np.float32(x[t, e]) - np.float32(values[s, e]))
                acc = np.float32(acc + np.float32(diff * diff))
            assert d[t, s] == acc
