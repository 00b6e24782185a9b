"""Pins of the oracle's binary16 arithmetic against numpy's float16 (a library
implementation of IEEE 754 binary16) and against the definition's edge cases."""
import numpy as np

from oracle import fp16


def test_decode_matches_numpy_on_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint16)
    ours = fp16.decode_bits(bits)
    ref = bits.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[np.isinf(ref)], ref[np.isinf(ref)])


def test_encode_inverts_decode():
    bits = np.arange(1 << 16, dtype=np.uint16)
    vals = fp16.decode_bits(bits)
    ok = np.isfinite(vals)
    assert np.array_equal(fp16.encode(vals[ok]), bits[ok])


def test_round_matches_numpy_random():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(200000) * 10.0 ** rng.integers(-9, 6, 200000),
        rng.uniform(-70000, 70000, 10000),
    ])
    ours = fp16.round_rne(v)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).astype(np.float64)
    assert np.array_equal(ours, ref)


def test_round_ties_to_even_and_overflow():
    bits = np.arange(0, 0x7BFF, dtype=np.uint16)       # consecutive finite positives
    lo = fp16.decode_bits(bits)
    hi = fp16.decode_bits(bits + 1)
    mid = (lo + hi) / 2                                # exact ties in float64
    got = fp16.round_rne(mid)
    even = np.where(bits % 2 == 0, lo, hi)
    assert np.array_equal(got, even)
    assert np.array_equal(got, mid.astype(np.float16).astype(np.float64))
    assert fp16.round_rne(65519.99) == 65504.0
    assert np.isinf(fp16.round_rne(65520.0))
    assert np.signbit(fp16.round_rne(-0.0))
    assert fp16.round_rne(2.0 ** -25) == 0.0            # tie between 0 and the smallest subnormal
    assert fp16.round_rne(3 * 2.0 ** -25) == 2.0 ** -23
