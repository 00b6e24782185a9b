"""The E8-lattice code (QL_CODE_E8P) on the GPU against the oracle: every one
of the 2^16 states bit-exact, decoded layers bit-exact, forwards within the
tolerance on both the decode-GEMV and the tensor-core path."""
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


def test_every_state_bit_exact():
    states = torch.arange(1 << 16, dtype=torch.int32, device="cuda")
    got = tcm.qlinear_eval_code(wl.CODE_E8P, 16, 8, states)
    torch.cuda.synchronize()
    ref = ofp16.encode(ocodes.evaluate(4, np.arange(1 << 16), 8))
    assert np.array_equal(_bits(got), ref)


@pytest.mark.parametrize("m,n", [(16, 256), (48, 768), (128, 1024)])
def test_decode_bit_exact(m, n):
    li = wl.random_layer(m, n, 2, 16, 8, wl.CODE_E8P, seed=50 + m, alpha=0.5)
    h = make_handle(li)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(w), oq.Layer.from_inputs(li).decode_bits(np.arange(m)))


@pytest.mark.parametrize("batch", [1, 3, 8, 16, 40])
def test_forward(batch):
    li = wl.random_layer(48, 768, 2, 16, 8, wl.CODE_E8P, seed=61, alpha=0.5)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=2)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= (TOL_GEMV if batch <= 8 else TOL_TC)


def test_create_rejects_other_shapes_of_the_code():
    li = wl.random_layer(16, 256, 2, 16, 8, wl.CODE_E8P, seed=62)
    codes = torch.from_numpy(li.codes.view(np.int32).copy()).cuda()
    s_in = torch.from_numpy(li.s_in.copy()).cuda()
    s_out = torch.from_numpy(li.s_out.copy()).cuda()
    for k, L, V in [(2, 16, 1), (2, 15, 8), (3, 16, 8)]:
        with pytest.raises(tcm.QLinearError):
            tcm.qlinear_create(16, 256, k, L, V, wl.CODE_E8P, codes, s_in, s_out, 1.0)
