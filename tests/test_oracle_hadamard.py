"""Pins of the oracle's Hadamard blocks and random-sign transform.

QuIP# page, Fig. 2 (incoherence processing with a randomized Hadamard
transform) and the QTIP discussion, "Incoherence Processing (W2)" (the RHT is
fully invertible up to numerical error); textbook facts: the unnormalised
Sylvester matrix satisfies H H^T = B I, H_2 = [[1, 1], [1, -1]], and
H_2B = [[H_B, H_B], [H_B, -H_B]].
"""
import numpy as np
import pytest

from oracle import hadamard


def _sylvester(B):
    H = np.array([[1.0]])
    while H.shape[0] < B:
        H = np.block([[H, H], [H, -H]])
    return H


def test_h2_textbook():
    assert np.array_equal(hadamard.dense(2, normalised=False), np.array([[1.0, 1.0], [1.0, -1.0]]))


@pytest.mark.parametrize("B", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_closed_form_equals_sylvester_recursion(B):
    assert np.array_equal(hadamard.dense(B, normalised=False), _sylvester(B))


@pytest.mark.parametrize("B", [2, 4, 16, 128, 1024, 4096])
def test_orthogonality(B):
    H = hadamard.dense(B, normalised=False)
    assert np.array_equal(H @ H.T, B * np.eye(B))
    Hn = hadamard.dense(B)
    assert np.allclose(Hn @ Hn, np.eye(B), atol=1e-12)
    assert np.array_equal(H, H.T)


def test_orthogonality_spot_rows_8192():
    B = 8192
    rows = np.array([0, 1, 777, 4096, 8191])
    Hr = hadamard.dense(B, normalised=False, rows=rows)
    G = Hr @ Hr.T
    assert np.array_equal(G, B * np.eye(len(rows)))


def test_block_size():
    assert [hadamard.block_size(d) for d in (256, 4096, 8192, 11008, 28672, 14336, 7168, 48)] == \
        [256, 4096, 8192, 256, 4096, 2048, 1024, 16]


def test_blockwise_equals_kronecker_and_preserves_norm():
    rng = np.random.default_rng(0)
    B, nblk = 64, 3
    v = rng.standard_normal((4, B * nblk))
    s = rng.choice([-1, 1], size=B * nblk)
    ref = (np.kron(np.eye(nblk), _sylvester(B) / np.sqrt(B)) @ (v * s).T).T
    got = hadamard.rht(v, s, B)
    assert np.allclose(got, ref, atol=1e-12)
    assert np.allclose(np.linalg.norm(got, axis=1), np.linalg.norm(v, axis=1), rtol=1e-12)
    back = hadamard.apply_blockwise(got, B) * s    # H^-1 = H, then undo the signs
    assert np.allclose(back, v, atol=1e-12)


def test_blockwise_apply_equals_the_dense_product():
    """The ordered accumulation equals the dense matrix product (H_2048 built
    by the Sylvester recursion, not the closed form) on random input."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal((2, 4096))
    a = hadamard.apply_blockwise(v, 2048)
    H = _sylvester(2048) / np.sqrt(2048)
    b = np.concatenate([v[:, :2048] @ H.T, v[:, 2048:] @ H.T], axis=1)
    assert np.allclose(a, b, atol=1e-12)
