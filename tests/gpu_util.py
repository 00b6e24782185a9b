"""Helpers for the GPU parity tests: move seeded inputs to the device and build
handles through the C ABI (via the thin binding)."""
import numpy as np
import torch

import trellis_coded_matmul_b200 as tcm
import workloads as wl

# Tolerances of the layer output against the float64 oracle (relative to the
# largest |y_ref| of the compared entries): fp32 accumulation on the GEMV
# path, fp16-input products accumulated in fp32 by the tensor-core GEMM path.
TOL_GEMV = 2e-3
TOL_TC = 5e-3


def to_dev(li: wl.LayerInputs):
    codes = torch.from_numpy(li.codes.view(np.int32).copy()).cuda()
    s_in = torch.from_numpy(li.s_in.copy()).cuda()
    s_out = torch.from_numpy(li.s_out.copy()).cuda()
    lut = torch.from_numpy(li.lut.copy()).cuda() if li.lut is not None else None
    return codes, s_in, s_out, lut


def make_handle(li: wl.LayerInputs):
    sp = li.spec
    codes, s_in, s_out, lut = to_dev(li)
    if sp.fractional:  # a half-integer bitwidth: parts given as bits per trellis step
        return tcm.qlinear_create_kv(sp.m, sp.n, [r for _, r, _ in sp.row_parts()], sp.part_kv(), sp.L, sp.V,
                                     sp.code, codes, s_in, s_out, sp.alpha, Q=sp.Q, lut=lut)
    if sp.row_split is not None:
        return tcm.qlinear_create_parts(sp.m, sp.n, [r for r, _ in sp.row_split], [k for _, k in sp.row_split],
                                        sp.L, sp.V, sp.code, codes, s_in, s_out, sp.alpha, Q=sp.Q, lut=lut)
    if sp.mixed:
        return tcm.qlinear_create_mixed(sp.m, sp.n, sp.m_top, sp.k_top, sp.k_bot, sp.L, sp.V, sp.code, codes,
                                        s_in, s_out, sp.alpha, Q=sp.Q, lut=lut)
    return tcm.qlinear_create(sp.m, sp.n, sp.k, sp.L, sp.V, sp.code, codes, s_in, s_out, sp.alpha, Q=sp.Q, lut=lut)


def rel_err(y, y_ref):
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))
