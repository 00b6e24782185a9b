"""qlinear_forward_noalloc against qlinear_forward, through the C ABI.

The no-allocation entry point runs the same decode-GEMV kernels with its
scratch in one fixed array of the library's static device memory, shared by
all handles on the device.  Each case calls it twice in a row (the second call
finds the array as the first left it) and compares both results with the
allocating entry point; cases run on different handles one after another, so
each also starts from an array that another layer used.  The file is named to
be collected last: it must pass both after the other GPU tests and alone in a
fresh process, where its first call does the one-time set-up."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import trellis_coded_matmul_b200 as tcm  # noqa: E402
import workloads as wl  # noqa: E402
from oracle import qlinear as oq  # noqa: E402
from gpu_util import TOL_GEMV, make_handle, rel_err  # noqa: E402

# Both entry points accumulate z with fp32 atomics in a run-dependent order;
# the results agree to fp32 rounding of the sums, far inside the oracle bound.
TOL_SAME_KERNELS = 1e-5


def _noalloc_raw(h, x, y):
    """Call the C entry point directly and return its status."""
    ydt = tcm.QL_F16 if y.dtype == torch.float16 else tcm.QL_F32
    lib = tcm.raw_library()
    return lib.qlinear_forward_noalloc(h.ptr, ctypes.c_void_p(x.data_ptr()), x.shape[0],
                                       ctypes.c_void_p(y.data_ptr()), ydt, None)


def _same(y, y_ref):
    y = y.double().cpu().numpy()
    y_ref = y_ref.double().cpu().numpy()
    return float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))


CASES = [
    # name, batch, out dtype: the output transform in the GEMV's epilogue
    # (tiny) and in its own kernel, HYB V = 2, half-TCQ (two row parts), and
    # fp16 output.
    ("tiny", 1, torch.float32),
    ("attn4096", 1, torch.float32),
    ("attn4096", 8, torch.float32),
    ("mlp_up", 8, torch.float32),
    ("mlp_down", 4, torch.float16),
    ("halftcq", 3, torch.float32),
]


@pytest.mark.parametrize("name,batch,dtype", CASES, ids=[f"{c[0]}-b{c[1]}-{str(c[2])[6:]}" for c in CASES])
def test_noalloc_matches_forward_on_two_calls_in_a_row(name, batch, dtype):
    sp = wl.WORKLOADS[name]
    h = make_handle(wl.make_layer(sp))
    try:
        x = torch.from_numpy(wl.make_x(sp, batch)).cuda()
        y_ref = tcm.qlinear_forward(h, x, torch.empty((batch, sp.m), dtype=dtype, device="cuda"))
        for call in range(2):
            y = torch.full((batch, sp.m), float("nan"), dtype=dtype, device="cuda")
            assert _noalloc_raw(h, x, y) == tcm.QL_OK
            torch.cuda.synchronize()
            tol = TOL_SAME_KERNELS if dtype == torch.float32 else 2 ** -10
            assert _same(y, y_ref) <= tol, (call, _same(y, y_ref))
        assert tcm.qlinear_get_status(h) == tcm.QL_OK
        assert tcm.qlinear_info(h)["last_launches"] >= 1
    finally:
        tcm.qlinear_destroy(h)


def test_noalloc_against_the_oracle():
    sp = wl.WORKLOADS["tiny"]
    li = wl.make_layer(sp)
    h = make_handle(li)
    try:
        x_np = wl.make_x(sp, 2)
        x = torch.from_numpy(x_np).cuda()
        y = torch.empty((2, sp.m), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(h, x, y) == tcm.QL_OK
        torch.cuda.synchronize()
        y_ref = oq.Layer.from_inputs(li).forward(x_np.astype(np.float64))
        assert rel_err(y.cpu().numpy(), y_ref) <= TOL_GEMV
    finally:
        tcm.qlinear_destroy(h)


def _noalloc_bytes(m, n, V, B_m, batch):
    """Scratch of one call as the header states it: the output-block tickets,
    z and x'."""
    up = lambda b: (b + 255) // 256 * 256  # noqa: E731
    return up(4 * (m // B_m)) + up(4 * batch * m) + 4 * batch * n // (1 if V == 1 else 2)


def test_noalloc_scratch_limit_and_batch_limit():
    # m = 81920 (Hadamard blocks of 16384), n = 256: batch 6 needs
    # 256 + 6*81920*4 + 6*256*4 = 1972480 bytes of scratch (fits in 2 MiB),
    # batch 7 needs 2301184 (does not).
    m, n = 81920, 256
    li = wl.random_layer(m, n, 2, 16, 1, wl.CODE_3INST, seed=11, alpha=0.5)
    h = make_handle(li)
    try:
        limit = tcm.QL_NOALLOC_SCRATCH_BYTES
        assert _noalloc_bytes(m, n, 1, 16384, 6) <= limit < _noalloc_bytes(m, n, 1, 16384, 7)

        x6 = torch.from_numpy(wl.make_x(li.spec, 6)).cuda()
        y_ref = tcm.qlinear_forward(h, x6)
        y6 = torch.empty((6, m), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(h, x6, y6) == tcm.QL_OK
        torch.cuda.synchronize()
        assert _same(y6, y_ref) <= TOL_SAME_KERNELS

        x7 = torch.from_numpy(wl.make_x(li.spec, 7)).cuda()
        y7 = torch.zeros((7, m), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(h, x7, y7) == tcm.QL_E_SCRATCH
        x9 = torch.from_numpy(wl.make_x(li.spec, 9)).cuda()
        y9 = torch.zeros((9, m), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(h, x9, y9) == tcm.QL_E_UNSUPPORTED
        torch.cuda.synchronize()
        assert not y7.any() and not y9.any()  # rejected before any device work
        with pytest.raises(tcm.QLinearError, match="fixed scratch"):
            tcm.qlinear_forward_noalloc(h, x7, y7)

        # the array still works after the rejections, for a smaller layer
        sp = wl.WORKLOADS["tiny"]
        h2 = make_handle(wl.make_layer(sp))
        try:
            x = torch.from_numpy(wl.make_x(sp, 8)).cuda()
            y_ref2 = tcm.qlinear_forward(h2, x)
            y = torch.empty_like(y_ref2)
            tcm.qlinear_forward_noalloc(h2, x, y)
            torch.cuda.synchronize()
            assert _same(y, y_ref2) <= TOL_SAME_KERNELS
        finally:
            tcm.qlinear_destroy(h2)
    finally:
        tcm.qlinear_destroy(h)


def test_noalloc_allocates_no_device_memory():
    sp = wl.WORKLOADS["attn4096"]
    h = make_handle(wl.make_layer(sp))
    try:
        x = torch.from_numpy(wl.make_x(sp, 8)).cuda()
        y = torch.empty((8, sp.m), dtype=torch.float32, device="cuda")
        assert _noalloc_raw(h, x, y) == tcm.QL_OK  # set-up done on an earlier call or here
        torch.cuda.synchronize()
        scratch_before = tcm.qlinear_info(h)["scratch_bytes"]
        free_before, _ = torch.cuda.mem_get_info()
        for _ in range(3):
            assert _noalloc_raw(h, x, y) == tcm.QL_OK
        torch.cuda.synchronize()
        free_after, _ = torch.cuda.mem_get_info()
        assert tcm.qlinear_info(h)["scratch_bytes"] == scratch_before == 0
        assert free_after == free_before
    finally:
        tcm.qlinear_destroy(h)
