"""Pins of the oracle's bit order and bitshift-trellis walk.

Sources: QTIP OpenReview discussion, "Figure 2 (Q4)" (the worked example and
the shift property) and "Ablations and fast inference (W1 and W2)" (L = kV is
plain k-bit V-dimensional VQ; the bitshift trellis is parallel-decodable).
"""
import os

import numpy as np
import pytest

from oracle import bitstream, trellis

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bitshift_walk_example.txt")


def _golden():
    d = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = vals
    return d


def test_worked_example_open_walk():
    g = _golden()
    L, kV = int(g["L"][0]), int(g["kV"][0])
    states = trellis.walk_open(g["bits"][0], L, kV)
    assert states == [int(s, 2) for s in g["states"]]


def test_msb_first_bit_order():
    w = np.array([0x80000001, 0x40000000], dtype=np.uint32)
    assert bitstream.bit(w, 0) == 1 and bitstream.bit(w, 31) == 1 and bitstream.bit(w, 33) == 1
    assert [int(bitstream.bit(w, p)) for p in (1, 30, 32, 34)] == [0, 0, 0, 0]
    assert bitstream.field(w, 31, 3) == 0b101
    assert np.array_equal(bitstream.bits_to_words("1" + "0" * 30 + "1" + "01" + "0" * 30), w)


def _cyclic_window(bitstring, end, L):
    S = len(bitstring)
    return int("".join(bitstring[(p % S)] for p in range(end - L, end)), 2)


@pytest.mark.parametrize("L,k,V", [(16, 2, 1), (16, 3, 2), (16, 4, 1), (6, 1, 1), (6, 2, 1), (6, 3, 2), (8, 4, 2), (3, 3, 1)])
def test_tailbiting_states_are_cyclic_windows(L, k, V):
    """Every state equals the L-bit window ending at its step, read cyclically
    from the block's bit string (a random-access definition, independent of the
    sequential walk)."""
    rng = np.random.default_rng(L * 100 + k * 10 + V)
    n, rows = 512, 3
    words = rng.integers(0, 2**32, size=rows * n * k // 32, dtype=np.uint32)
    st = trellis.block_states(words, np.arange(rows), n, [(0, rows, k)], L, V)
    kV = k * V
    S = 256 * k
    full = "".join(f"{int(w):032b}" for w in words)
    for r in range(rows):
        for j in range(n // 256):
            blk = full[r * n * k + j * S: r * n * k + (j + 1) * S]
            for t in range(0, 256 // V, 7):
                assert st[r, j, t] == _cyclic_window(blk, (t + 1) * kV, L)


def test_L_equals_kV_is_plain_vq():
    """With L = kV each state is exactly its own chunk (k-bit V-dim VQ)."""
    rng = np.random.default_rng(5)
    k, V = 3, 2
    words = rng.integers(0, 2**32, size=2 * 256 * k // 32, dtype=np.uint32)
    st = trellis.block_states(words, np.arange(2), 256, [(0, 2, k)], k * V, V)
    for r in range(2):
        for t in range(256 // V):
            assert st[r, 0, t] == bitstream.field(words, r * 256 * k + t * k * V, k * V)


@pytest.mark.parametrize("L,kV", [(6, 1), (6, 2), (6, 3), (4, 2)])
def test_brute_force_tiny_trellis(L, kV):
    """Brute force over every state and every chunk of a tiny trellis: the
    successor keeps exactly L-kV bits, every state has 2^kV distinct
    successors, every state is reachable, and a walk over a de Bruijn string
    of order L visits every state once."""
    succ = {}
    for s in range(1 << L):
        nxt = set()
        for c in range(1 << kV):
            s2 = int(trellis.step(s, c, L, kV))
            assert s2 >> kV == s & ((1 << (L - kV)) - 1)
            nxt.add(s2)
        assert len(nxt) == 1 << kV
        succ[s] = nxt
    assert set().union(*succ.values()) == set(range(1 << L))
    if kV == 1:
        # de Bruijn sequence B(2, L) by the standard Lyndon-word construction
        a = [0] * (2 * L)
        seq = []

        def db(t, p):
            if t > L:
                if L % p == 0:
                    seq.extend(a[1:p + 1])
            else:
                a[t] = a[t - p]
                db(t + 1, p)
                for j in range(a[t - p] + 1, 2):
                    a[t] = j
                    db(t + 1, t)
        db(1, 1)
        s = "".join(map(str, seq))
        states = trellis.walk_open(s + s[:L - 1], L, 1)
        assert sorted(states) == list(range(1 << L))


def test_mixed_rows_start_after_top_part():
    """Half-TCQ layout: the bottom rows are a uniform layer of their own,
    starting right after the top rows' bits."""
    rng = np.random.default_rng(9)
    n, m_top, m_bot, k_top, k_bot = 512, 16, 16, 2, 3
    top = rng.integers(0, 2**32, size=m_top * n * k_top // 32, dtype=np.uint32)
    bot = rng.integers(0, 2**32, size=m_bot * n * k_bot // 32, dtype=np.uint32)
    words = np.concatenate([top, bot])
    parts = [(0, m_top, k_top), (m_top, m_bot, k_bot)]
    rows = np.array([0, 15, 16, 31])
    st = trellis.block_states(words, rows, n, parts, 16, 1)
    st_top = trellis.block_states(top, np.array([0, 15]), n, [(0, m_top, k_top)], 16, 1)
    st_bot = trellis.block_states(bot, np.array([0, 15]), n, [(0, m_bot, k_bot)], 16, 1)
    assert np.array_equal(st[:2], st_top) and np.array_equal(st[2:], st_bot)


def test_planted_shift_mistake_is_caught(monkeypatch):
    """A walk that shifts by one bit too few fails the worked example."""
    real = trellis.step

    def wrong(state, chunk, L, kV):
        return (np.asarray(state, dtype=np.int64) << max(kV - 1, 0) | np.asarray(chunk)) & ((1 << L) - 1)
    monkeypatch.setattr(trellis, "step", wrong)
    g = _golden()
    assert trellis.walk_open(g["bits"][0], 2, 1) != [int(s, 2) for s in g["states"]]
    monkeypatch.setattr(trellis, "step", real)


def test_planted_prefix_mistake_is_caught(monkeypatch):
    """A tail-biting walk that starts from zero instead of the block's last
    L-kV bits fails the walk's own end-of-block consistency check."""
    rng = np.random.default_rng(11)
    words = rng.integers(0, 2**32, size=256 * 2 // 32, dtype=np.uint32)
    real_field = bitstream.field

    def zero_prefix(w, p, width):
        if width == 14:
            return np.zeros(np.shape(p), dtype=np.int64)
        return real_field(w, p, width)
    monkeypatch.setattr(bitstream, "field", zero_prefix)
    with pytest.raises(AssertionError, match="tail-biting"):
        trellis.block_states(words, np.arange(1), 256, [(0, 1, 2)], 16, 1)
