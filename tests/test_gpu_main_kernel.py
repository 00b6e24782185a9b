"""qlinear_launch_main_kernel: the forward's dominant kernel launched alone
(for timing) runs on the scratch of the last forward with the same batch,
and leaves the handle able to produce correct forwards afterwards."""
import numpy as np
import pytest
import torch

import trellis_coded_matmul_b200 as tcm
import workloads as wl
from gpu_util import make_handle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,batch", [("tiny", 1), ("attn4096", 1), ("attn4096", 8), ("halftcq", 64)])
def test_main_kernel_alone_then_forward_is_unchanged(name, batch):
    sp = wl.WORKLOADS[name]
    h = make_handle(wl.make_layer(sp))
    x = torch.from_numpy(wl.make_x(sp, batch)).cuda()
    y0 = tcm.qlinear_forward(h, x)
    with pytest.raises(tcm.QLinearError):
        tcm.qlinear_launch_main_kernel(h, batch + 1, None)  # not the last forward's batch
    y = torch.empty_like(y0)
    for _ in range(3):
        tcm.qlinear_launch_main_kernel(h, batch, x, y)
    torch.cuda.synchronize()
    assert tcm.qlinear_info(h)["last_launches"] == 1
    y1 = tcm.qlinear_forward(h, x)
    torch.cuda.synchronize()
    # the accumulation order of the fp32 sums may differ between runs
    tol = 1e-4 * float(y0.abs().max())
    assert torch.allclose(y0, y1, rtol=1e-4, atol=tol)


def test_main_kernel_needs_a_forward_first():
    sp = wl.WORKLOADS["tiny"]
    h = make_handle(wl.make_layer(sp))
    with pytest.raises(tcm.QLinearError):
        tcm.qlinear_launch_main_kernel(h, 1, None)
