"""Full-size layers against the float64 oracle on every weight and every output.

For each workload at every batch it is benchmarked at, the whole decoded
matrix (qlinear_decode) must be bit-exact with the oracle's fp16 rounding of
each code value, and every output of qlinear_forward must satisfy
max|y - y_ref| <= tol * max|y_ref| (tol = 2e-3 on the decode-GEMV path at
batch <= 8, 5e-3 on the tensor-core path).  The oracle decodes the matrix in
row blocks in spawned worker processes and forms z = W_hat x' on each block;
the output transform then runs over whole Hadamard blocks of z."""
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle_pool  # noqa: E402
import trellis_coded_matmul_b200 as tcm  # noqa: E402
import workloads as wl  # noqa: E402
from oracle import qlinear as oq  # noqa: E402
from gpu_util import TOL_GEMV, TOL_TC, make_handle, rel_err  # noqa: E402

# workload -> batches: the benchmark configurations (the five layer shapes of
# the workload list with their batches), the fused QKV layer, and the palette
# layers at batch <= 8 plus one tensor-core batch
FULL = {
    "tiny": (1,),
    "attn4096": (1,),
    "mlp_up": (1, 4, 8),
    "mlp_down": (1, 4, 8),
    "large": (1, 4, 16),
    "halftcq": (64, 256),
    "qkv_fused": (1, 16),
    "tcq2p5": (1, 4, 8, 64),
    "tcq2p75": (1, 4, 8, 64),
    "vq2p5": (1, 4, 8, 64),
    "nuq3": (1, 4, 8, 64),
    "e8p2": (1, 4, 8, 64),
}
CHUNK_WEIGHTS = 1 << 21  # weights per oracle task


@pytest.fixture(scope="module")
def pool():
    workers = max(1, min(16, os.cpu_count() or 1))
    with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        yield ex


def _first_mismatch(got, ref, r0):
    r, c = np.argwhere(got != ref)[0]
    return f"W_hat[{r0 + r}][{c}]: got 0x{got[r, c]:04x}, oracle 0x{ref[r, c]:04x}"


@pytest.mark.parametrize("name", list(FULL))
def test_full_layer_every_weight_and_every_output(name, pool):
    sp = wl.WORKLOADS[name]
    batches = FULL[name]
    li = wl.make_layer(sp)
    h = make_handle(li)
    w = tcm.qlinear_decode(h)
    ys = {b: tcm.qlinear_forward(h, torch.from_numpy(wl.make_x(sp, b)).cuda()) for b in batches}
    torch.cuda.synchronize()
    assert tcm.qlinear_get_status(h) == tcm.QL_OK

    rows_per = max(16, CHUNK_WEIGHTS // sp.n)
    starts = list(range(0, sp.m, rows_per))
    futs = [pool.submit(oracle_pool.rows_chunk, name, r0, min(sp.m, r0 + rows_per), batches) for r0 in starts]
    z = {b: np.empty((b, sp.m)) for b in batches}
    for r0, f in zip(starts, futs):
        r1 = min(sp.m, r0 + rows_per)
        bits, zs = f.result()
        got = w[r0:r1].cpu().numpy().view(np.uint16)
        assert np.array_equal(got, bits), _first_mismatch(got, bits, r0)
        for b in batches:
            z[b][:, r0:r1] = zs[b]
    layer = oq.Layer.from_inputs(li)
    for b in batches:
        y_ref = layer.output_transform(z[b], np.arange(sp.m))
        err = rel_err(ys[b].cpu().numpy(), y_ref)
        assert err <= (TOL_GEMV if b <= 8 else TOL_TC), f"batch {b}: max err / max|y| = {err:.3e}"
