"""The GPU trellis-coded quantizer (qlinear_encode) against the oracle's two-pass
search, through the C ABI: the same float32 rule, so the same bits.

Source blocks are i.i.d. N(0,1) float32 (the discussion's "Table 1" setting).
The encoded words also round-trip through a layer: qlinear_create on them and
qlinear_decode give the oracle's reconstruction of the chosen walks."""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import trellis_coded_matmul_b200 as tcm  # noqa: E402
import workloads as wl  # noqa: E402
from oracle import bitstream, encode, fp16 as ofp16  # noqa: E402

CASES = [
    # L, k, V, code, Q
    (10, 1, 1, wl.CODE_1MAD, 0),
    (12, 2, 1, wl.CODE_3INST, 0),
    (12, 2, 2, wl.CODE_HYB, 6),
    (14, 2, 1, wl.CODE_3INST, 0),
    (13, 3, 1, wl.CODE_HYB, 9),
    (13, 2, 1, wl.CODE_1MAD, 0),
    (14, 2, 2, wl.CODE_HYB, 9),
    # L = 15, 16: one CTA holds the group minima of the search whenever they fit
    (16, 2, 1, wl.CODE_3INST, 0),
    (15, 1, 1, wl.CODE_1MAD, 0),
    (16, 1, 2, wl.CODE_HYB, 9),
    (16, 3, 1, wl.CODE_HYB, 9),
    (16, 4, 1, wl.CODE_1MAD, 0),
    (15, 2, 1, wl.CODE_HYB, 9),
    (15, 3, 1, wl.CODE_3INST, 0),
    # L = 16 at one bit per step: the dynamic programme shared by a cluster of 4 CTAs
    (16, 1, 1, wl.CODE_HYB, 9),
    (16, 1, 1, wl.CODE_3INST, 0),
]


def _source(blocks, seed):
    return np.random.default_rng(seed).standard_normal((blocks, 256)).astype(np.float32)


def _oracle_words(x, L, k, V, code, lut):
    out = []
    for blk in x:
        chunks, _ = encode.encode_two_pass(blk.reshape(-1, V), L, k, V, code, lut)
        bits = "".join(format(int(c), f"0{k * V}b") for c in chunks)
        out.append(bitstream.bits_to_words(bits))
    return np.stack(out)


@pytest.mark.parametrize("L,k,V,code,Q", CASES, ids=lambda v: str(v))
def test_encode_matches_the_oracle_bit_for_bit(L, k, V, code, Q):
    lut_np = wl.hyb_table(Q, V, 3) if code == wl.CODE_HYB else None
    lut = torch.from_numpy(lut_np.copy()).cuda() if lut_np is not None else None
    x = _source(3, seed=L * 10 + k)
    words, err = tcm.qlinear_encode(code, L, k, V, torch.from_numpy(x).cuda(), Q=Q, lut=lut, with_error=True)
    torch.cuda.synchronize()
    ref = _oracle_words(x, L, k, V, code, lut_np)
    assert np.array_equal(words.cpu().numpy().view(np.uint32), ref)
    for b in range(3):
        chunks = np.array([int(c, 2) for c in (lambda s: [s[i:i + k * V] for i in range(0, len(s), k * V)])(
            "".join(format(int(w), "032b") for w in ref[b]))])
        recon = encode.reconstruct(chunks, L, k * V, code, V, lut_np).reshape(-1)
        assert float(err[b]) == pytest.approx(float(np.sum((x[b].astype(np.float64) - recon) ** 2)), rel=1e-4)


# bits per step (kv) instead of k: half-integer bitwidths and the palette's table code
CASES_KV = [
    # L, kv, V, code, Q
    (12, 5, 2, wl.CODE_HYB, 9),      # 2.5-bit TCQ, one CTA per block
    (16, 5, 2, wl.CODE_HYB, 9),      # 2.5-bit TCQ at L = 16
    (15, 7, 2, wl.CODE_HYB, 6),      # 3.5 bits
    (5, 5, 2, wl.CODE_TABLE, 0),     # 2.5-bit VQ: nearest codeword
    (3, 3, 1, wl.CODE_TABLE, 0),     # 3-bit NUQ: nearest level
    (8, 3, 2, wl.CODE_TABLE, 0),     # 1.5 bits, a trellis over a 256-entry codebook
]


def _table(code, L, V, Q, seed):
    if code == wl.CODE_HYB:
        return wl.hyb_table(Q, V, seed)
    if code == wl.CODE_TABLE:
        return wl.palette_table(L, V, seed)
    return None


def _oracle_words_kv(x, L, kv, V, code, lut):
    out = []
    for blk in x:
        chunks, _ = encode.encode_two_pass(blk.reshape(-1, V), L, kv / V, V, code, lut)
        out.append(bitstream.bits_to_words("".join(format(int(c), f"0{kv}b") for c in chunks)))
    return np.stack(out)


@pytest.mark.parametrize("L,kv,V,code,Q", CASES_KV, ids=lambda v: str(v))
def test_encode_kv_matches_the_oracle_bit_for_bit(L, kv, V, code, Q):
    lut_np = _table(code, L, V, Q, 8)
    lut = torch.from_numpy(lut_np.copy()).cuda() if lut_np is not None else None
    x = _source(3, seed=L * 10 + kv)
    words, err = tcm.qlinear_encode_kv(code, L, kv, V, torch.from_numpy(x).cuda(), Q=Q, lut=lut, with_error=True)
    torch.cuda.synchronize()
    ref = _oracle_words_kv(x, L, kv, V, code, lut_np)
    assert words.shape == (3, (256 // V) * kv // 32)
    assert np.array_equal(words.cpu().numpy().view(np.uint32), ref)


def test_fractional_vq_round_trips_through_a_layer():
    """2.5-bit VQ of a 32 x 512 source: the encoder's words, given to
    qlinear_create_kv, decode to the oracle's reconstruction, which is the
    nearest codeword of (nearly) every pair: with L = kV the search only adds
    per-step costs, so it departs from the nearest codeword only where two
    codewords' costs tie after rounding against the running path cost."""
    L, kv, V, code = 5, 5, 2, wl.CODE_TABLE
    m, n = 32, 512
    book = wl.palette_table(L, V, 9)
    lut = torch.from_numpy(book.copy()).cuda()
    x = _source(m * n // 256, seed=15).reshape(m, n)
    words = tcm.qlinear_encode_kv(code, L, kv, V, torch.from_numpy(x).cuda(), lut=lut)
    torch.cuda.synchronize()
    ones_n = torch.ones(n, dtype=torch.int8, device="cuda")
    ones_m = torch.ones(m, dtype=torch.int8, device="cuda")
    h = tcm.qlinear_create_kv(m, n, [m], [kv], L, V, code, words.reshape(-1), ones_n, ones_m, 1.0, lut=lut)
    w = tcm.qlinear_decode(h).cpu().numpy()
    ref = _oracle_words_kv(x.reshape(-1, 256), L, kv, V, code, book)
    recon = []
    for row in ref:
        bits = "".join(format(int(wd), "032b") for wd in row)
        chunks = np.array([int(bits[i:i + kv], 2) for i in range(0, len(bits), kv)])
        recon.append(encode.reconstruct(chunks, L, kv, code, V, book).reshape(-1))
    recon = np.concatenate(recon).reshape(m, n)
    assert np.array_equal(w.view(np.uint16), ofp16.encode(recon))
    cb = book.astype(np.float32)
    pairs = x.reshape(m, n // 2, 2)
    d = (pairs[:, :, None, 0] - cb[None, None, :, 0]) ** 2 + (pairs[:, :, None, 1] - cb[None, None, :, 1]) ** 2
    nearest = cb[np.argmin(d, axis=-1)].astype(np.float64)
    assert np.mean(np.all(w.astype(np.float64).reshape(m, n // 2, 2) == nearest, axis=-1)) > 0.999
    tcm.qlinear_destroy(h)


def test_encoded_words_round_trip_through_a_layer():
    L, k, V, code = 12, 2, 1, wl.CODE_1MAD
    m, n = 32, 512
    x = _source(m * n // 256, seed=5).reshape(m, n)
    words = tcm.qlinear_encode(code, L, k, V, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    codes = words.reshape(-1)
    ones = torch.ones(n, dtype=torch.int8, device="cuda")
    h = tcm.qlinear_create(m, n, k, L, V, code, codes, ones, torch.ones(m, dtype=torch.int8, device="cuda"), 1.0)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    ref = _oracle_words(x.reshape(-1, 256), L, k, V, code, None)
    recon = []
    for row in ref:
        bits = "".join(format(int(wd), "032b") for wd in row)
        chunks = np.array([int(bits[i:i + k * V], 2) for i in range(0, len(bits), k * V)])
        recon.append(encode.reconstruct(chunks, L, k * V, code, V).reshape(-1))
    recon = np.concatenate(recon).reshape(m, n)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ofp16.encode(recon))
    tcm.qlinear_destroy(h)


@pytest.mark.parametrize("k,blocks", [(2, 300), (1, 100)], ids=["one_cta", "cluster"])
def test_encoder_loops_over_more_blocks_than_workers(k, blocks):
    """More blocks at L = 16 than the CTAs (k = 2: one a block) or clusters
    (k = 1: four CTAs a block) that run at once, so each encodes several blocks
    in turn.  Block i repeats source block i % 3 (consecutive blocks of one
    worker differ), so every block must give the oracle's words for its source."""
    L, V, code = 16, 1, wl.CODE_3INST
    base = _source(3, seed=77 + k)
    pick = np.arange(blocks) % 3
    x = np.ascontiguousarray(base[pick])
    words = tcm.qlinear_encode(code, L, k, V, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    got = words.cpu().numpy().view(np.uint32)
    ref = _oracle_words(base, L, k, V, code, None)
    assert np.array_equal(got, ref[pick])


def test_encoder_scratch_reuse_leaves_results_unchanged():
    """The search's scratch comes from a memory pool that the library keeps
    between calls: a call after a smaller one (other sizes, dirty scratch)
    gives the same words and errors as the first call on the same source."""
    x = torch.from_numpy(_source(200, seed=91)).cuda()
    w1, e1 = tcm.qlinear_encode(wl.CODE_3INST, 16, 2, 1, x, with_error=True)
    tcm.qlinear_encode(wl.CODE_1MAD, 14, 1, 1, x[:7])
    w2, e2 = tcm.qlinear_encode(wl.CODE_3INST, 16, 2, 1, x, with_error=True)
    torch.cuda.synchronize()
    assert torch.equal(w1, w2) and torch.equal(e1, e2)


def test_gaussian_distortion_at_L16_beats_L14():
    """The discussion's setting (L = 16, k = 2): distortion between the Gaussian
    rate-distortion bound and the 2-bit Lloyd-Max quantizer, and below L = 14's
    on the same source ("larger trellises improve quality")."""
    x = torch.from_numpy(_source(128, seed=60)).cuda()
    mse = {}
    for L in (14, 16):
        _, err = tcm.qlinear_encode(wl.CODE_3INST, L, 2, 1, x, with_error=True)
        mse[L] = float(err.sum()) / x.numel()
    assert 2.0 ** -4 < mse[16] < mse[14] < 0.1175


@pytest.mark.parametrize("k", [1, 2])
def test_gaussian_distortion_at_L14(k):
    x = _source(64, seed=40 + k)
    xt = torch.from_numpy(x).cuda()
    tcm.qlinear_encode(wl.CODE_3INST, 14, k, 1, xt[:2])  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    _, err = tcm.qlinear_encode(wl.CODE_3INST, 14, k, 1, xt, with_error=True)
    secs = time.perf_counter() - t0
    mse = float(err.sum()) / x.size
    print(f"L=14 k={k}: mse {mse:.4f}, {x.shape[0] / secs:.0f} blocks/s")
    assert 2.0 ** (-2 * k) < mse < {1: 1.0 - 2.0 / np.pi, 2: 0.1175}[k]
