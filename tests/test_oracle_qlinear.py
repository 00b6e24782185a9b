"""Pins of the oracle's decode layout and forward pass.

The layer (workload definition and QuIP#/QTIP incoherence processing):
    y = alpha * diag(s_out) * H_m^T * W_hat * H_n * diag(s_in) * x
Checks: closed forms (linearity, the alpha scale, basis inputs), an
independent dense construction of W with Kronecker-built Hadamard matrices,
the element order inside a block, and the bit accounting of the QTIP
discussion, "Bit Accounting (Q2)".
"""
import numpy as np
import pytest

import workloads as wl
from oracle import bitstream, codes, hadamard, qlinear, trellis


def _layer(m, n, k, code, V=1, seed=0, alpha=1.0, **kw):
    li = wl.random_layer(m, n, k, 16, V, code, seed, alpha=alpha, **kw)
    return qlinear.Layer.from_inputs(li)


def _dense_W(layer):
    """W = alpha diag(s_out) H_m W_hat H_n diag(s_in), Hadamards by np.kron."""
    def kron_h(d):
        B = hadamard.block_size(d)
        H = np.array([[1.0]])
        while H.shape[0] < B:
            H = np.block([[H, H], [H, -H]])
        return np.kron(np.eye(d // B), H / np.sqrt(B))
    What = layer.decode_rows(np.arange(layer.m))
    return layer.alpha * (layer.s_out[:, None] * (kron_h(layer.m) @ What @ kron_h(layer.n))) * layer.s_in[None, :]


@pytest.mark.parametrize("m,n,k,code,V", [(256, 256, 2, wl.CODE_1MAD, 1), (48, 768, 3, wl.CODE_3INST, 1),
                                          (32, 512, 4, wl.CODE_HYB, 2), (16, 256, 1, wl.CODE_HYB, 1)])
def test_forward_equals_dense_weight(m, n, k, code, V):
    layer = _layer(m, n, k, code, V, seed=m + n, alpha=0.37)
    x = np.random.default_rng(1).standard_normal((3, n)).astype(np.float16)
    y = layer.forward(x)
    W = _dense_W(layer)
    ref = x.astype(np.float64) @ W.T
    assert np.allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_tiny_workload_closed_forms():
    li = wl.make_layer(wl.WORKLOADS["tiny"])
    layer = qlinear.Layer.from_inputs(li)
    rng = np.random.default_rng(2)
    x1 = rng.standard_normal((1, 256)).astype(np.float16).astype(np.float64)
    x2 = rng.standard_normal((1, 256)).astype(np.float16).astype(np.float64)
    y1, y2 = layer.forward(x1), layer.forward(x2)
    assert np.allclose(layer.forward(x1 + 2 * x2), y1 + 2 * y2, atol=1e-9)
    layer2 = qlinear.Layer.from_inputs(li)
    layer2.alpha = 3.0 * layer.alpha
    assert np.allclose(layer2.forward(x1), 3.0 * y1, atol=1e-12)
    # basis input e_i: y = alpha s_out (H_m W_hat (H_n column i)) s_in[i]
    i = 17
    e = np.zeros((1, 256))
    e[0, i] = 1.0
    What = layer.decode_rows(np.arange(256))
    Hn = hadamard.dense(256)
    ref = layer.alpha * layer.s_out * (hadamard.dense(256) @ (What @ Hn[:, i])) * layer.s_in[i]
    assert np.allclose(layer.forward(e)[0], ref, atol=1e-12)


def test_forward_rows_match_full_forward():
    layer = _layer(64, 512, 2, wl.CODE_3INST, seed=4)
    x = np.random.default_rng(3).standard_normal((2, 512)).astype(np.float16)
    rows = np.array([0, 5, 63, 17])
    assert np.allclose(layer.forward_rows(x, rows), layer.forward(x)[:, rows], atol=1e-12)


def test_element_order_inside_a_block():
    """Column j*T + t*V + e holds value e of the code on state t of block j."""
    layer = _layer(16, 512, 3, wl.CODE_HYB, V=2, seed=6)
    layer.lut = (np.arange(1024).reshape(512, 2) / 64.0 + 1.0).astype(np.float16)
    rows = np.array([3, 9])
    W = layer.decode_rows(rows)
    st = trellis.block_states(layer.words, rows, 512, layer.parts, 16, 2)
    for ri in range(2):
        for j in range(2):
            for t in (0, 1, 57, 127):
                vals = codes.hyb(np.array([st[ri, j, t]]), layer.lut)[0]
                assert W[ri, j * 256 + t * 2] == vals[0] and W[ri, j * 256 + t * 2 + 1] == vals[1]


def test_decode_is_fp16_exact():
    layer = _layer(32, 256, 2, wl.CODE_1MAD, seed=7)
    bits = layer.decode_bits(np.arange(32))
    assert bits.dtype == np.uint16
    assert np.array_equal(bits.view(np.float16).astype(np.float64), layer.decode_rows(np.arange(32)))


def test_bit_accounting():
    """Stream = m n k bits; signs = n + m bits; HYB table = 2^Q V 16 bits,
    under 0.01 extra bits per weight on the MLP-shaped layers."""
    for name in ("attn4096", "mlp_up", "mlp_down", "large", "halftcq"):
        sp = wl.WORKLOADS[name]
        assert sp.n_words * 32 == sum(r * sp.n * k for _, r, k in sp.row_parts())
        extra_bits = (sp.m + sp.n) + ((1 << sp.Q) * sp.V * 16 if sp.code == wl.CODE_HYB else 0)
        assert extra_bits / (sp.m * sp.n) < 0.01
    assert wl.WORKLOADS["halftcq"].bits_per_weight == 2.5
    assert (1 << 9) * 2 * 16 // 8 == 2048


def test_mixed_layer_decodes_each_part_with_its_own_k():
    li = wl.random_layer(32, 512, 0, 16, 1, wl.CODE_3INST, 3, m_top=16, k_top=2, k_bot=3)
    layer = qlinear.Layer.from_inputs(li)
    top_words = li.codes[: 16 * 512 * 2 // 32]
    bot_words = li.codes[16 * 512 * 2 // 32:]
    top = qlinear.Layer(16, 512, [(0, 16, 2)], 16, 1, wl.CODE_3INST, top_words, li.s_in, li.s_out[:16], 1.0)
    bot = qlinear.Layer(16, 512, [(0, 16, 3)], 16, 1, wl.CODE_3INST, bot_words, li.s_in, li.s_out[16:], 1.0)
    W = layer.decode_rows(np.arange(32))
    assert np.array_equal(W[:16], top.decode_rows(np.arange(16)))
    assert np.array_equal(W[16:], bot.decode_rows(np.arange(16)))


def test_layer_of_several_parts_is_the_stack_of_its_parts():
    """A layer fused along m from parts of different bitwidths: its weight rows
    are those of the single-part layers decoded from the consecutive
    sub-streams (each part's blocks keep their own tail-biting)."""
    split = ((16, 2), (32, 4), (16, 1))
    li = wl.random_layer(64, 512, 0, 16, 1, wl.CODE_1MAD, 5, row_split=split)
    layer = qlinear.Layer.from_inputs(li)
    W = layer.decode_rows(np.arange(64))
    off, r0 = 0, 0
    for rows, k in split:
        words = li.codes[off: off + rows * 512 * k // 32]
        single = qlinear.Layer(rows, 512, [(0, rows, k)], 16, 1, wl.CODE_1MAD, words, li.s_in,
                               li.s_out[r0:r0 + rows], 1.0)
        assert np.array_equal(W[r0:r0 + rows], single.decode_rows(np.arange(rows)))
        off += rows * 512 * k // 32
        r0 += rows
    assert off == len(li.codes) and li.spec.bits_per_weight == (16 * 2 + 32 * 4 + 16 * 1) / 64
