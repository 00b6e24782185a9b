"""Palette quantizers on the CUDA path against the float64 oracle, through the C ABI.

Half-integer bitwidths (V = 2 with an odd number kV of bits per step: 1.5, 2.5
and 3.5 bits per weight) and the table code (an explicit 2^L-entry codebook:
VQ at V = 2 and NUQ at V = 1 when L = kV, a trellis over the codebook when
L > kV), the Q-Palette page's fractional-bit TCQ / VQ / NUQ quantizers.
Decoded weights must be bit-exact; outputs within 2e-3 (decode-GEMV, batch
<= 8) or 5e-3 (tensor-core GEMM) of max|y_ref|."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import trellis_coded_matmul_b200 as tcm  # noqa: E402
import workloads as wl  # noqa: E402
from oracle import codes as ocodes, fp16 as ofp16, qlinear as oq  # noqa: E402
from gpu_util import TOL_GEMV, TOL_TC, make_handle, rel_err  # noqa: E402


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("L,V", [(1, 1), (3, 1), (9, 1), (5, 2), (9, 2)])
def test_eval_code_table_every_state_bit_exact(L, V):
    book = wl.palette_table(L, V, seed=L + 10 * V)
    lut = torch.from_numpy(book.copy()).cuda()
    states_np = np.concatenate([np.arange(1 << L), np.arange(1 << L) + (5 << L)])  # high bits are ignored
    states = torch.from_numpy(states_np.astype(np.int32)).cuda()
    got = tcm.qlinear_eval_code(wl.CODE_TABLE, L, V, states, lut=lut)
    torch.cuda.synchronize()
    ref = ofp16.encode(ocodes.table(states_np & ((1 << L) - 1), book))
    assert np.array_equal(_bits(got), ref)


PALETTE = [
    # m, n, k (bits per weight), L, V, code, extra
    (48, 512, 2.5, 16, 2, wl.CODE_HYB, {"Q": 9}),    # fractional TCQ
    (32, 768, 1.5, 16, 2, wl.CODE_HYB, {"Q": 6}),
    (32, 512, 3.5, 16, 2, wl.CODE_HYB, {"Q": 9}),
    (16, 256, 2.5, 11, 2, wl.CODE_HYB, {"Q": 9}),    # short state, odd kV
    (32, 512, 2.5, 5, 2, wl.CODE_TABLE, {}),         # 2.5-bit VQ (L = kV)
    (48, 512, 2, 4, 2, wl.CODE_TABLE, {}),           # 2-bit VQ
    (16, 256, 4, 8, 2, wl.CODE_TABLE, {}),           # 4-bit VQ: 256 codewords
    (32, 768, 3, 3, 1, wl.CODE_TABLE, {}),           # 3-bit NUQ
    (16, 256, 1, 1, 1, wl.CODE_TABLE, {}),           # 1-bit NUQ
    (32, 512, 4, 4, 1, wl.CODE_TABLE, {}),           # 4-bit NUQ
    (32, 512, 2, 8, 1, wl.CODE_TABLE, {}),           # trellis over a 256-entry codebook
    (32, 512, 3.5, 9, 2, wl.CODE_TABLE, {}),         # trellis over a 512-entry codebook, odd kV
]


def _ids(c):
    return f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_V{c[4]}_c{c[5]}"


def _layer(m, n, k, L, V, code, extra):
    return wl.random_layer(m, n, k, L, V, code, seed=2000 + m + n + int(2 * k) * 7 + L, alpha=0.5, **extra)


@pytest.mark.parametrize("case", PALETTE, ids=_ids)
def test_palette_decode_bit_exact(case):
    li = _layer(*case)
    h = make_handle(li)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(w), oq.Layer.from_inputs(li).decode_bits(np.arange(li.spec.m)))


@pytest.mark.parametrize("case", PALETTE, ids=_ids)
@pytest.mark.parametrize("batch", [1, 3, 8, 16, 40])
def test_palette_forward(case, batch):
    li = _layer(*case)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=5)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= (TOL_GEMV if batch <= 8 else TOL_TC)


@pytest.mark.parametrize("code,L", [(wl.CODE_HYB, 16), (wl.CODE_TABLE, 7)], ids=["HYB", "TABLE"])
@pytest.mark.parametrize("batch", [2, 24])
def test_fractional_parts(code, L, batch):
    split = ((16, 2.5), (32, 3), (16, 1.5), (16, 3.5))
    li = wl.random_layer(80, 512, 0, L, 2, code, seed=61 + L, alpha=0.5, Q=9, row_split=split)
    h = make_handle(li)
    info = tcm.qlinear_info(h)
    assert info["part_kv"] == [5, 6, 3, 7] and info["part_rows"] == [16, 32, 16, 16]
    assert info["stream_bytes"] * 8 == int(512 * (16 * 2.5 + 32 * 3 + 16 * 1.5 + 16 * 3.5))
    layer = oq.Layer.from_inputs(li)
    x = wl.make_x(li.spec, batch, instance=19)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    assert rel_err(y.cpu().numpy(), layer.forward(x)) <= (TOL_GEMV if batch <= 8 else TOL_TC)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(w), layer.decode_bits(np.arange(80)))


def test_fractional_create_rejects_bad_bitrates():
    li = _layer(*PALETTE[0])
    codes = torch.from_numpy(li.codes.view(np.int32).copy()).cuda()
    s_in = torch.from_numpy(li.s_in.copy()).cuda()
    s_out = torch.from_numpy(li.s_out.copy()).cuda()
    lut = torch.from_numpy(li.lut.copy()).cuda()
    for kv, L, want in [(1, 16, tcm.QL_E_UNSUPPORTED),   # k = 0.5
                        (9, 16, tcm.QL_E_UNSUPPORTED),   # k = 4.5
                        (5, 4, tcm.QL_E_UNSUPPORTED)]:   # L < kV
        with pytest.raises(tcm.QLinearError) as e:
            tcm.qlinear_create_kv(48, 512, [48], [kv], L, 2, wl.CODE_HYB, codes, s_in, s_out, 1.0, Q=9, lut=lut)
        assert e.value.status == want
    with pytest.raises(tcm.QLinearError) as e:  # a 2^10-entry codebook is over the limit
        tcm.qlinear_create_kv(48, 512, [48], [5], 10, 2, wl.CODE_TABLE, codes, s_in, s_out, 1.0, lut=lut)
    assert e.value.status == tcm.QL_E_UNSUPPORTED
