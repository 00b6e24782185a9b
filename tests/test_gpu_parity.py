"""CUDA path against the float64 oracle, element by element, through the C ABI.

Decoded weights (qlinear_decode, qlinear_eval_code) must be bit-exact with the
oracle's fp16 rounding; layer outputs must satisfy
max|y - y_ref| <= tol * max|y_ref| with tol = 2e-3 for batch <= 8 (fp32
accumulation) and 5e-3 for the tensor-core path."""
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

L16 = 1 << 16


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


# ---------------------------------------------------------------- codes
@pytest.mark.parametrize("kind,fn", [(wl.CODE_1MAD, ocodes.one_mad), (wl.CODE_3INST, ocodes.three_inst)],
                         ids=["1MAD", "3INST"])
def test_eval_code_every_state_bit_exact(kind, fn):
    states = torch.arange(L16, dtype=torch.int32, device="cuda")
    got = tcm.qlinear_eval_code(kind, 16, 1, states)
    torch.cuda.synchronize()
    ref = ofp16.encode(fn(np.arange(L16)))
    assert np.array_equal(_bits(got)[:, 0], ref)


@pytest.mark.parametrize("V,Q", [(2, 9), (1, 9), (2, 6), (1, 4)])
def test_eval_code_hyb_every_state_bit_exact(V, Q):
    lut_np = wl.hyb_table(Q, V, 2)
    lut = torch.from_numpy(lut_np.copy()).cuda()
    states = torch.arange(L16, dtype=torch.int32, device="cuda")
    got = tcm.qlinear_eval_code(wl.CODE_HYB, 16, V, states, Q=Q, lut=lut)
    torch.cuda.synchronize()
    ref = ofp16.encode(ocodes.hyb(np.arange(L16), lut_np))
    assert np.array_equal(_bits(got), ref)


def test_eval_code_odd_count_and_small_L():
    states = torch.arange(0, 1001, dtype=torch.int32, device="cuda")
    got = tcm.qlinear_eval_code(wl.CODE_3INST, 10, 1, states)
    ref = ofp16.encode(ocodes.three_inst(np.arange(1001) & 1023))
    assert np.array_equal(_bits(got)[:, 0], ref)


# ---------------------------------------------------------------- decode
SMALL = [
    # m, n, k, L, V, code, extra
    (256, 256, 2, 16, 1, wl.CODE_1MAD, {}),
    (48, 768, 3, 16, 1, wl.CODE_3INST, {}),
    (32, 512, 4, 16, 1, wl.CODE_1MAD, {}),
    (16, 256, 1, 16, 1, wl.CODE_3INST, {}),
    (64, 512, 3, 16, 2, wl.CODE_HYB, {"Q": 9}),
    (32, 256, 1, 16, 2, wl.CODE_HYB, {"Q": 6}),
    (32, 1024, 2, 16, 1, wl.CODE_HYB, {"Q": 5}),
    (32, 512, 4, 16, 2, wl.CODE_HYB, {"Q": 9}),
    (16, 256, 2, 2, 1, wl.CODE_1MAD, {}),         # L = kV: plain VQ
    (16, 256, 2, 7, 1, wl.CODE_3INST, {}),        # short state
    (16, 256, 3, 6, 2, wl.CODE_HYB, {"Q": 9}),    # L = kV with V = 2
]


def _small_layer(m, n, k, L, V, code, extra, seed=0):
    return wl.random_layer(m, n, k, L, V, code, seed=1000 + m + n + k * 7 + L, alpha=0.5, **extra)


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_V{c[4]}_c{c[5]}")
def test_decode_small_bit_exact(case):
    li = _small_layer(*case)
    h = make_handle(li)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    ref = oq.Layer.from_inputs(li).decode_bits(np.arange(li.spec.m))
    assert np.array_equal(_bits(w), ref)


def test_decode_mixed_bit_exact():
    li = wl.random_layer(64, 512, 0, 16, 1, wl.CODE_3INST, 5, m_top=32, k_top=2, k_bot=3)
    h = make_handle(li)
    w = tcm.qlinear_decode(h)
    ref = oq.Layer.from_inputs(li).decode_bits(np.arange(64))
    assert np.array_equal(_bits(w), ref)


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_V{c[4]}_c{c[5]}")
@pytest.mark.parametrize("batch", [1, 3, 8])
def test_forward_small(case, batch):
    li = _small_layer(*case)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=3)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_GEMV


@pytest.mark.parametrize("batch", [9, 16, 33])
def test_forward_larger_batches(batch):
    li = _small_layer(*SMALL[1])
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=4)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_TC


def test_forward_fp16_output_and_zero_batch():
    li = _small_layer(*SMALL[0])
    h = make_handle(li)
    x = wl.make_x(li.spec, 2, instance=5)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda(), out_dtype=torch.float16)
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert y.dtype == torch.float16
    assert rel_err(y.float().cpu().numpy(), y_ref) <= TOL_GEMV + 2.0 ** -11
    empty = torch.empty((0, li.spec.n), dtype=torch.float16, device="cuda")
    assert tcm.qlinear_forward(h, empty).shape == (0, li.spec.m)


def test_forward_host_buffers():
    li = _small_layer(*SMALL[4])
    h = make_handle(li)
    x = torch.from_numpy(wl.make_x(li.spec, 4, instance=6)).pin_memory()
    y = tcm.qlinear_forward_host(h, x)
    assert not y.is_cuda
    y_ref = oq.Layer.from_inputs(li).forward(x.numpy())
    assert rel_err(y.numpy(), y_ref) <= TOL_GEMV


@pytest.mark.parametrize("case,batch,pinned", [(0, 1, True), (2, 2, False), (4, 72, True), (1, 6, True)],
                         ids=["1mad_b1_pinned", "1mad_b2_pageable", "hyb_b72_large_x", "3inst_b6_pinned"])
def test_forward_host_input_paths(case, batch, pinned):
    """qlinear_forward_host with pinned and pageable host buffers, x from 512 B
    to 72 KB (72 x 512 fp16), on the GEMV and tensor-core paths, against the
    oracle."""
    li = _small_layer(*SMALL[case])
    h = make_handle(li)
    x = torch.from_numpy(wl.make_x(li.spec, batch, instance=8))
    if pinned:
        x = x.pin_memory()
    y = tcm.qlinear_forward_host(h, x)
    tol = TOL_GEMV if batch <= 8 else TOL_TC
    assert rel_err(y.numpy(), oq.Layer.from_inputs(li).forward(x.numpy())) <= tol


def test_forward_mixed_small():
    li = wl.random_layer(64, 512, 0, 16, 1, wl.CODE_3INST, 5, m_top=32, k_top=2, k_bot=3)
    h = make_handle(li)
    for batch in (1, 8, 20):
        x = wl.make_x(li.spec, batch, instance=7)
        y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
        tol = TOL_GEMV if batch <= 8 else TOL_TC
        assert rel_err(y.cpu().numpy(), oq.Layer.from_inputs(li).forward(x)) <= tol


def test_bad_signs_are_rejected():
    li = _small_layer(*SMALL[0])
    li.s_in[5] = 0
    with pytest.raises(tcm.QLinearError) as e:
        make_handle(li)
    assert e.value.status == tcm.QL_E_ARG


def test_info_reports_the_bit_accounting():
    li = wl.make_layer(wl.WORKLOADS["mlp_up"])
    h = make_handle(li)
    info = tcm.qlinear_info(h)
    sp = li.spec
    assert info["stream_bytes"] == sp.m * sp.n * sp.k // 8
    assert info["sign_bytes"] * 8 >= sp.m + sp.n and info["sign_bytes"] * 8 < sp.m + sp.n + 64
    assert info["lut_bytes"] == 2048
    assert (info["B_n"], info["B_m"]) == (4096, 256)


def test_forward_in_cuda_graph_with_profiling():
    """forward is capturable in a CUDA graph after a first (allocating) call,
    replays give the oracle's result, and the profiling slots record the
    main kernel on every replay."""
    li = _small_layer(*SMALL[1])
    h = make_handle(li)
    tcm.qlinear_profile_enable(h, 4)
    xs = [torch.from_numpy(wl.make_x(li.spec, 2, instance=10 + i)).cuda() for i in range(3)]
    ys = [torch.zeros((2, li.spec.m), device="cuda") for _ in range(3)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        tcm.qlinear_forward(h, xs[0], ys[0])
    torch.cuda.synchronize()
    for y in ys:
        y.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for x, y in zip(xs, ys):
            tcm.qlinear_forward(h, x, y)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    ref = oq.Layer.from_inputs(li)
    for x, y in zip(xs, ys):
        assert rel_err(y.cpu().numpy(), ref.forward(x.cpu().numpy())) <= TOL_GEMV
    ms, slots = tcm.qlinear_profile_read(h)
    assert slots == 4 and ms > 0
    tcm.qlinear_profile_enable(h, 0)


# ---------------------------------------------------------------- largest Hadamard blocks
# B = 16384 and 32768 run the transforms with 1024-thread CTAs (16 and 32
# entries per thread); B_n = 32768 also takes the separate input-transform
# kernel at batch 1 (batch * n above the in-kernel limit).
@pytest.mark.parametrize("m,n", [(32768, 256), (16384, 256), (16, 32768)], ids=lambda v: str(v))
def test_forward_largest_hadamard_blocks(m, n):
    li = wl.random_layer(m, n, 2, 16, 1, wl.CODE_3INST, seed=7 + m + n, alpha=0.25)
    h = make_handle(li)
    x = wl.make_x(li.spec, 2, instance=9)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_GEMV


# ---------------------------------------------------------------- layers of several row parts
PARTS = [((32, 2), (48, 3), (16, 4)), ((16, 1), (16, 2), (32, 3), (16, 4), (16, 2)),
         ((16, 1), (16, 2), (16, 3), (16, 4), (32, 2), (16, 3), (16, 1), (16, 4))]  # the most parts: 8


@pytest.mark.parametrize("split", PARTS, ids=lambda v: "-".join(f"{r}k{k}" for r, k in v))
def test_parts_decode_bit_exact(split):
    m = sum(r for r, _ in split)
    li = wl.random_layer(m, 512, 0, 16, 1, wl.CODE_3INST, seed=21 + m, alpha=0.5, row_split=split)
    h = make_handle(li)
    assert tcm.qlinear_info(h)["nparts"] == len(split)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(w), oq.Layer.from_inputs(li).decode_bits(np.arange(m)))


@pytest.mark.parametrize("split", PARTS, ids=lambda v: "-".join(f"{r}k{k}" for r, k in v))
@pytest.mark.parametrize("batch", [1, 3, 16, 40])
def test_parts_forward(split, batch):
    m = sum(r for r, _ in split)
    li = wl.random_layer(m, 512, 0, 16, 1, wl.CODE_1MAD, seed=31 + m, alpha=0.5, row_split=split)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=11)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= (TOL_GEMV if batch <= 8 else TOL_TC)


# ---------------------------------------------------------------- tensor-core path over every small case
# (L < 16, L = kV, HYB V = 1 and 2, 1-4 bits, ragged row tiles) at two batch sizes
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_V{c[4]}_c{c[5]}")
@pytest.mark.parametrize("batch", [16, 40])
def test_forward_small_tensor_core_path(case, batch):
    li = _small_layer(*case)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=13)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    assert tcm.qlinear_info(h)["last_launches"] == 3  # input transform, GEMM, output transform
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_TC


# The GEMM's operand forms around their switch points: split A words (computed
# codes, padded batch <= 128) with x' twice along K, and the lean input
# transform of the operand tiles (batch >= 128), alone and together.
@pytest.mark.parametrize("case", [SMALL[0], SMALL[1], SMALL[2], SMALL[9]],
                         ids=lambda c: f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_c{c[5]}")
@pytest.mark.parametrize("batch", [112, 120, 128, 129, 200])
def test_forward_operand_form_boundaries(case, batch):
    li = _small_layer(*case)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=19)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= TOL_TC


@pytest.mark.parametrize("batch", [2, 24])
def test_parts_with_the_hyb_code(batch):
    split = ((16, 2), (32, 3), (16, 4))
    li = wl.random_layer(64, 512, 0, 16, 2, wl.CODE_HYB, seed=41, alpha=0.5, Q=9, row_split=split)
    h = make_handle(li)
    x = wl.make_x(li.spec, batch, instance=17)
    y = tcm.qlinear_forward(h, torch.from_numpy(x).cuda())
    y_ref = oq.Layer.from_inputs(li).forward(x)
    assert rel_err(y.cpu().numpy(), y_ref) <= (TOL_GEMV if batch <= 8 else TOL_TC)
    w = tcm.qlinear_decode(h)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(w), oq.Layer.from_inputs(li).decode_bits(np.arange(64)))


# ---------------------------------------------------------------- every output element written
@pytest.mark.parametrize("case", [SMALL[1], SMALL[4], SMALL[9]], ids=lambda c: f"{c[0]}x{c[1]}_k{c[2]}_L{c[3]}_V{c[4]}")
def test_outputs_are_fully_written_over_a_nan_sentinel(case):
    """y and W_hat buffers pre-filled with NaN come back without any NaN (the
    codes' values and the outputs are finite), on both forward paths; the
    fp16 output too."""
    li = _small_layer(*case)
    h = make_handle(li)
    for batch in (3, 16):
        x = torch.from_numpy(wl.make_x(li.spec, batch, instance=21)).cuda()
        for dtype in (torch.float32, torch.float16):
            y = torch.full((batch, li.spec.m), float("nan"), dtype=dtype, device="cuda")
            tcm.qlinear_forward(h, x, y)
            torch.cuda.synchronize()
            assert not torch.isnan(y).any()
    w = torch.full((li.spec.m, li.spec.n), float("nan"), dtype=torch.float16, device="cuda")
    tcm.qlinear_decode(h, w)
    torch.cuda.synchronize()
    assert not torch.isnan(w).any()
