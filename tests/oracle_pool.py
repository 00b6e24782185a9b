"""Oracle work for the full-size parity tests, run in worker processes.

The full-size layers hold up to 235M weights; the oracle decodes them row
block by row block in float64 in spawned worker processes (a spawned worker
shares nothing with the parent's CUDA context).  Each call regenerates the
layer from its seeded workload, so only names and row ranges cross the
process boundary.  Nothing here is arithmetic of its own: every value comes
from `oracle/`.
"""
from __future__ import annotations

import functools
import os

os.environ.setdefault("OMP_NUM_THREADS", "1")
os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402
from oracle import fp16, qlinear  # noqa: E402


@functools.lru_cache(maxsize=2)
def _layer(name: str) -> qlinear.Layer:
    return qlinear.Layer.from_inputs(wl.make_layer(wl.WORKLOADS[name]))


@functools.lru_cache(maxsize=8)
def _xp(name: str, batch: int) -> np.ndarray:
    return _layer(name).input_transform(wl.make_x(wl.WORKLOADS[name], batch))


def rows_chunk(name: str, r0: int, r1: int, batches) -> tuple:
    """Rows [r0, r1) of the workload's layer: W_hat as fp16 bit patterns
    (uint16 [rows, n]) and z = W_hat x' on those rows for each batch
    ({batch: float64 [batch, rows]})."""
    layer = _layer(name)
    W = layer.decode_rows(np.arange(r0, r1))
    return fp16.encode(W), {b: qlinear.contract(W, _xp(name, b)) for b in batches}
