"""Expiry of the tensor-core GEMM's bounded waits, made to happen on purpose.

Every mbarrier wait of the GEMM's producer/consumer pipeline gives up after a
bounded number of suspending tries, records QL_E_TIMEOUT in the handle's
status word and lets the CTA drop its work and free its tensor memory.  The
test hook qlinear_test_stall shortens the limit and makes the x' producer
withhold one stage, so the waits run out: no fault, trap or unbounded wait is
involved.  The handle must then report the timeout, give the oracle's result
on the next forward, and hold no more device memory than before."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import trellis_coded_matmul_b200 as tcm  # noqa: E402
import workloads as wl  # noqa: E402
from oracle import qlinear as oq  # noqa: E402
from gpu_util import TOL_TC, make_handle, rel_err  # noqa: E402


def test_expired_waits_report_a_timeout_and_the_handle_recovers():
    li = wl.random_layer(256, 1024, 2, 16, 1, wl.CODE_3INST, seed=77, alpha=0.5)
    h = make_handle(li)
    try:
        x_np = wl.make_x(li.spec, 32, instance=5)
        x = torch.from_numpy(x_np).cuda()
        y = tcm.qlinear_forward(h, x)  # allocates the handle's scratch
        torch.cuda.synchronize()
        assert tcm.qlinear_get_status(h) == tcm.QL_OK
        free_before, _ = torch.cuda.mem_get_info()

        tcm.qlinear_test_stall(h, True, wait_tries=8)
        tcm.qlinear_forward(h, x, y)
        torch.cuda.synchronize()
        assert tcm.qlinear_get_status(h) == tcm.QL_E_TIMEOUT
        assert tcm.qlinear_get_status(h) == tcm.QL_OK  # the status word was read and cleared

        tcm.qlinear_test_stall(h, False)
        y2 = tcm.qlinear_forward(h, x)
        torch.cuda.synchronize()
        assert tcm.qlinear_get_status(h) == tcm.QL_OK
        assert rel_err(y2.cpu().numpy(), oq.Layer.from_inputs(li).forward(x_np)) <= TOL_TC
        free_after, _ = torch.cuda.mem_get_info()
        assert free_after == free_before
    finally:
        tcm.qlinear_destroy(h)


def test_stall_hook_rejects_bad_limits():
    li = wl.random_layer(32, 256, 2, 16, 1, wl.CODE_1MAD, seed=78)
    h = make_handle(li)
    try:
        for bad in (0, 4097):
            with pytest.raises(tcm.QLinearError) as e:
                tcm.qlinear_test_stall(h, True, wait_tries=bad)
            assert e.value.status == tcm.QL_E_ARG
        tcm.qlinear_test_stall(h, False, wait_tries=0)  # disabling takes any limit
    finally:
        tcm.qlinear_destroy(h)
