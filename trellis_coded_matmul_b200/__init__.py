"""Python binding of libqlinear.so (include/qlinear.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module turns
torch tensors into pointers and status codes into exceptions.  It has no
fallback: if libqlinear.so is missing the import fails, and every call needs
CUDA tensors on the device the handle was created on.

    import trellis_coded_matmul_b200 as tcm
    h = tcm.qlinear_create(m, n, k, L, V, tcm.QL_CODE_3INST, codes, s_in, s_out, alpha)
    y = tcm.qlinear_forward(h, x)            # x: cuda fp16 [batch, n] -> y fp32 [batch, m]
    tcm.qlinear_destroy(h)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlinear.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python trellis_coded_matmul_b200/build.py`")
_lib = ctypes.CDLL(_LIB_PATH)

QL_OK = 0
QL_E_ARG = -1
QL_E_UNSUPPORTED = -2
QL_E_CUDA = -3
QL_E_OOM = -4
QL_E_TIMEOUT = -5
QL_E_DEVICE = -6
QL_E_SCRATCH = -7
QL_NOALLOC_SCRATCH_BYTES = 2 * 1024 * 1024
QL_CODE_1MAD = 0
QL_CODE_3INST = 1
QL_CODE_HYB = 2
QL_CODE_TABLE = 3
QL_CODE_E8P = 4
QL_F32 = 0
QL_F16 = 1

# Every function include/qlinear.h declares (checked by the CPU tests).
ABI_SYMBOLS = ("qlinear_create", "qlinear_create_mixed", "qlinear_create_parts", "qlinear_create_kv",
               "qlinear_forward", "qlinear_forward_host",
               "qlinear_decode", "qlinear_eval_code", "qlinear_get_status", "qlinear_info",
               "qlinear_destroy", "qlinear_strerror", "qlinear_profile_enable", "qlinear_profile_read",
               "qlinear_forward_noalloc", "qlinear_encode", "qlinear_encode_kv", "qlinear_test_stall",
               "qlinear_launch_main_kernel")


class ql_code_t(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("Q", ctypes.c_int), ("lut", ctypes.c_void_p)]


class ql_info_t(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int) for f in ("m", "n", "L", "V", "code", "Q", "k_top", "k_bot", "m_top", "B_n", "B_m")] + \
               [(f, ctypes.c_size_t) for f in ("stream_bytes", "sign_bytes", "lut_bytes", "scratch_bytes")] + \
               [("last_launches", ctypes.c_int), ("nparts", ctypes.c_int),
                ("part_rows", ctypes.c_int * 8), ("part_kv", ctypes.c_int * 8)]


_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_lib.qlinear_create.argtypes = [ctypes.POINTER(_vp), _i, _i, _i, _i, _i, ql_code_t, _vp, _sz, _vp, _vp, _f]
_lib.qlinear_create_mixed.argtypes = [ctypes.POINTER(_vp), _i, _i, _i, _i, _i, _i, _i, ql_code_t, _vp, _sz, _vp,
                                      _vp, _f]
_lib.qlinear_create_parts.argtypes = [ctypes.POINTER(_vp), _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i), _i, _i,
                                      ql_code_t, _vp, _sz, _vp, _vp, _f]
_lib.qlinear_create_kv.argtypes = [ctypes.POINTER(_vp), _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i), _i, _i,
                                   ql_code_t, _vp, _sz, _vp, _vp, _f]
_lib.qlinear_forward.argtypes = [_vp, _vp, _i, _vp, _i, _vp]
_lib.qlinear_forward_host.argtypes = [_vp, _vp, _i, _vp, _i, _vp]
_lib.qlinear_forward_noalloc.argtypes = [_vp, _vp, _i, _vp, _i, _vp]
_lib.qlinear_launch_main_kernel.argtypes = [_vp, _vp, _i, _vp, _i, _vp]
_lib.qlinear_encode.argtypes = [ql_code_t, _i, _i, _i, _vp, _i, _vp, _vp, _vp]
_lib.qlinear_encode_kv.argtypes = [ql_code_t, _i, _i, _i, _vp, _i, _vp, _vp, _vp]
_lib.qlinear_decode.argtypes = [_vp, _vp, _vp]
_lib.qlinear_eval_code.argtypes = [ql_code_t, _i, _i, _vp, _i, _vp, _vp]
_lib.qlinear_get_status.argtypes = [_vp]
_lib.qlinear_test_stall.argtypes = [_vp, _i, _i]
_lib.qlinear_info.argtypes = [_vp, ctypes.POINTER(ql_info_t)]
_lib.qlinear_destroy.argtypes = [_vp]
_lib.qlinear_strerror.argtypes = [_i]
_lib.qlinear_profile_enable.argtypes = [_vp, _i]
_lib.qlinear_profile_read.argtypes = [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i)]
_lib.qlinear_strerror.restype = ctypes.c_char_p
for _name in ABI_SYMBOLS:
    if _name != "qlinear_strerror":
        getattr(_lib, _name).restype = _i


class QLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {qlinear_strerror(status)} ({status})")
        self.status = status


def qlinear_strerror(status: int) -> str:
    return _lib.qlinear_strerror(status).decode()


def _check(status: int, where: str) -> None:
    if status != QL_OK:
        raise QLinearError(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cuda(t, name, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} must have dtype {dtype}")
    return t


class QLinearHandle:
    """Owns a qlinear_t; destroyed explicitly or when garbage-collected."""

    def __init__(self, ptr: int, m: int, n: int):
        self.ptr = ptr
        self.m = m
        self.n = n

    def __del__(self):
        if getattr(self, "ptr", None):
            try:
                _lib.qlinear_destroy(self.ptr)
            except Exception:
                pass
            self.ptr = None


def _code(kind: int, Q: int = 0, lut=None) -> ql_code_t:
    if lut is not None:
        import torch
        _cuda(lut, "lut", torch.float16)
    return ql_code_t(kind, Q, _ptr(lut))


def qlinear_create(m, n, k, L, V, kind, codes, s_in, s_out, alpha, Q=0, lut=None) -> QLinearHandle:
    """codes: CUDA uint32/int32 [m*n*k/32]; s_in, s_out: CUDA int8 +-1; lut: CUDA fp16
    [2^Q, V] (HYB) or [2^L, V] (the table code's codebook)."""
    import torch
    _cuda(codes, "codes", (torch.int32, torch.uint32))
    _cuda(s_in, "s_in", torch.int8)
    _cuda(s_out, "s_out", torch.int8)
    out = _vp()
    _check(_lib.qlinear_create(ctypes.byref(out), m, n, k, L, V, _code(kind, Q, lut), _ptr(codes), codes.numel(),
                               _ptr(s_in), _ptr(s_out), float(alpha)), "qlinear_create")
    return QLinearHandle(out.value, m, n)


def qlinear_create_mixed(m, n, m_top, k_top, k_bot, L, V, kind, codes, s_in, s_out, alpha, Q=0,
                         lut=None) -> QLinearHandle:
    import torch
    _cuda(codes, "codes", (torch.int32, torch.uint32))
    _cuda(s_in, "s_in", torch.int8)
    _cuda(s_out, "s_out", torch.int8)
    out = _vp()
    _check(_lib.qlinear_create_mixed(ctypes.byref(out), m, n, m_top, k_top, k_bot, L, V, _code(kind, Q, lut),
                                     _ptr(codes), codes.numel(), _ptr(s_in), _ptr(s_out), float(alpha)),
           "qlinear_create_mixed")
    return QLinearHandle(out.value, m, n)


def qlinear_create_parts(m, n, part_rows, part_k, L, V, kind, codes, s_in, s_out, alpha, Q=0,
                         lut=None) -> QLinearHandle:
    """A layer of several row parts (layers fused along m), part i at part_k[i] bits."""
    import torch
    _cuda(codes, "codes", (torch.int32, torch.uint32))
    _cuda(s_in, "s_in", torch.int8)
    _cuda(s_out, "s_out", torch.int8)
    if len(part_rows) != len(part_k):
        raise ValueError("part_rows and part_k must have the same length")
    rows = (ctypes.c_int * max(1, len(part_rows)))(*part_rows)
    ks = (ctypes.c_int * max(1, len(part_k)))(*part_k)
    out = _vp()
    _check(_lib.qlinear_create_parts(ctypes.byref(out), m, n, len(part_rows), rows, ks, L, V, _code(kind, Q, lut),
                                     _ptr(codes), codes.numel(), _ptr(s_in), _ptr(s_out), float(alpha)),
           "qlinear_create_parts")
    return QLinearHandle(out.value, m, n)


def qlinear_create_kv(m, n, part_rows, part_kv, L, V, kind, codes, s_in, s_out, alpha, Q=0,
                      lut=None) -> QLinearHandle:
    """A layer of row parts whose bitrates are given as bits per trellis step:
    part i at part_kv[i] / V bits per weight (a half number when V = 2 and
    part_kv[i] is odd, e.g. 5 bits per step = 2.5 bits per weight)."""
    import torch
    _cuda(codes, "codes", (torch.int32, torch.uint32))
    _cuda(s_in, "s_in", torch.int8)
    _cuda(s_out, "s_out", torch.int8)
    if len(part_rows) != len(part_kv):
        raise ValueError("part_rows and part_kv must have the same length")
    rows = (ctypes.c_int * max(1, len(part_rows)))(*part_rows)
    kvs = (ctypes.c_int * max(1, len(part_kv)))(*part_kv)
    out = _vp()
    _check(_lib.qlinear_create_kv(ctypes.byref(out), m, n, len(part_rows), rows, kvs, L, V, _code(kind, Q, lut),
                                  _ptr(codes), codes.numel(), _ptr(s_in), _ptr(s_out), float(alpha)),
           "qlinear_create_kv")
    return QLinearHandle(out.value, m, n)


def qlinear_forward(h: QLinearHandle, x, y=None, out_dtype=None, stream=None):
    """x: CUDA fp16 [batch, n] -> y [batch, m] (fp32 unless out_dtype/y says fp16)."""
    import torch
    _cuda(x, "x", torch.float16)
    batch = x.shape[0] if x.dim() == 2 else 0
    if x.dim() != 2 or x.shape[1] != h.n:
        raise ValueError("x must be [batch, n]")
    if y is None:
        y = torch.empty((batch, h.m), dtype=out_dtype or torch.float32, device=x.device)
    _cuda(y, "y", (torch.float32, torch.float16))
    if tuple(y.shape) != (batch, h.m):
        raise ValueError("y must be [batch, m]")
    ydt = QL_F16 if y.dtype == torch.float16 else QL_F32
    _check(_lib.qlinear_forward(h.ptr, _ptr(x), batch, _ptr(y), ydt, _stream(stream)), "qlinear_forward")
    return y


def qlinear_launch_main_kernel(h: QLinearHandle, batch: int, x=None, y=None, stream=None) -> None:
    """Launch the dominant kernel of a forward with this batch alone, on the
    scratch the handle's last forward (same batch) left (for timing; see the
    C header).  x: the forward's CUDA fp16 [batch, n] input, read where the
    decode-GEMV computes x' itself.  y: CUDA fp32/fp16 [batch, m], written
    only where the decode-GEMV transforms its own output."""
    import torch
    xp = None
    if x is not None:
        _cuda(x, "x", torch.float16)
        if tuple(x.shape) != (batch, h.n):
            raise ValueError("x must be [batch, n]")
        xp = _ptr(x)
    yp, ydt = None, QL_F32
    if y is not None:
        _cuda(y, "y", (torch.float32, torch.float16))
        if tuple(y.shape) != (batch, h.m):
            raise ValueError("y must be [batch, m]")
        yp, ydt = _ptr(y), (QL_F16 if y.dtype == torch.float16 else QL_F32)
    _check(_lib.qlinear_launch_main_kernel(h.ptr, xp, batch, yp, ydt, _stream(stream)), "qlinear_launch_main_kernel")


def qlinear_forward_host(h: QLinearHandle, x, y=None, out_dtype=None, stream=None):
    """x: CPU fp16 [batch, n] (pinned for asynchronous copies) -> y CPU [batch, m]; returns when y is ready."""
    import torch
    if x.is_cuda or x.dtype != torch.float16 or not x.is_contiguous() or x.dim() != 2 or x.shape[1] != h.n:
        raise ValueError("x must be a contiguous CPU fp16 tensor [batch, n]")
    batch = x.shape[0]
    if y is None:
        y = torch.empty((batch, h.m), dtype=out_dtype or torch.float32, pin_memory=x.is_pinned())
    if y.is_cuda or tuple(y.shape) != (batch, h.m) or y.dtype not in (torch.float32, torch.float16):
        raise ValueError("y must be a CPU fp32/fp16 tensor [batch, m]")
    ydt = QL_F16 if y.dtype == torch.float16 else QL_F32
    _check(_lib.qlinear_forward_host(h.ptr, _ptr(x), batch, _ptr(y), ydt, _stream(stream)), "qlinear_forward_host")
    return y


def qlinear_forward_noalloc(h: QLinearHandle, x, y, stream=None):
    """As qlinear_forward for batch <= 8, with the library's fixed scratch array
    instead of allocated scratch; the caller provides y (CUDA fp32/fp16 [batch, m])."""
    import torch
    _cuda(x, "x", torch.float16)
    if x.dim() != 2 or x.shape[1] != h.n:
        raise ValueError("x must be [batch, n]")
    _cuda(y, "y", (torch.float32, torch.float16))
    if tuple(y.shape) != (x.shape[0], h.m):
        raise ValueError("y must be [batch, m]")
    ydt = QL_F16 if y.dtype == torch.float16 else QL_F32
    _check(_lib.qlinear_forward_noalloc(h.ptr, _ptr(x), x.shape[0], _ptr(y), ydt, _stream(stream)),
           "qlinear_forward_noalloc")
    return y


def qlinear_encode(kind, L, k, V, x, Q=0, lut=None, with_error=False, stream=None):
    """Trellis-coded quantization of x (CUDA float32, [..., 256*j] rows whose
    length is a multiple of 256): the stream-format words (int32 [blocks, 8k])
    and, with with_error, each block's squared reconstruction error."""
    import torch
    _cuda(x, "x", torch.float32)
    if x.numel() % 256:
        raise ValueError("x must hold whole blocks of 256 values")
    blocks = x.numel() // 256
    words = torch.empty((blocks, 8 * k), dtype=torch.int32, device=x.device)
    err = torch.empty(blocks, dtype=torch.float32, device=x.device) if with_error else None
    _check(_lib.qlinear_encode(_code(kind, Q, lut), L, k, V, _ptr(x), blocks, _ptr(words),
                               _ptr(err) if err is not None else None, _stream(stream)), "qlinear_encode")
    return (words, err) if with_error else words


def qlinear_encode_kv(kind, L, kv, V, x, Q=0, lut=None, with_error=False, stream=None):
    """As qlinear_encode with kv bits per trellis step (odd kv with V = 2: a
    half-integer bitwidth): words int32 [blocks, (256 // V) * kv // 32]."""
    import torch
    _cuda(x, "x", torch.float32)
    if x.numel() % 256:
        raise ValueError("x must hold whole blocks of 256 values")
    if V not in (1, 2):
        raise ValueError("V must be 1 or 2")
    blocks = x.numel() // 256
    words = torch.empty((blocks, (256 // V) * kv // 32), dtype=torch.int32, device=x.device)
    err = torch.empty(blocks, dtype=torch.float32, device=x.device) if with_error else None
    _check(_lib.qlinear_encode_kv(_code(kind, Q, lut), L, kv, V, _ptr(x), blocks, _ptr(words),
                                  _ptr(err) if err is not None else None, _stream(stream)), "qlinear_encode_kv")
    return (words, err) if with_error else words


def qlinear_decode(h: QLinearHandle, w_hat=None, stream=None):
    """W_hat as CUDA fp16 [m, n] (code values before alpha, signs and transforms)."""
    import torch
    if w_hat is None:
        w_hat = torch.empty((h.m, h.n), dtype=torch.float16, device="cuda")
    _cuda(w_hat, "w_hat", torch.float16)
    _check(_lib.qlinear_decode(h.ptr, _ptr(w_hat), _stream(stream)), "qlinear_decode")
    return w_hat


def qlinear_eval_code(kind, L, V, states, Q=0, lut=None, out=None, stream=None):
    """states: CUDA uint32/int32 [count] -> fp16 [count, V]."""
    import torch
    _cuda(states, "states", (torch.int32, torch.uint32))
    if out is None:
        out = torch.empty((states.numel(), V), dtype=torch.float16, device=states.device)
    _check(_lib.qlinear_eval_code(_code(kind, Q, lut), L, V, _ptr(states), states.numel(), _ptr(out),
                                  _stream(stream)), "qlinear_eval_code")
    return out


def qlinear_get_status(h: QLinearHandle) -> int:
    return _lib.qlinear_get_status(h.ptr)


def qlinear_test_stall(h: QLinearHandle, enable: bool, wait_tries: int = 8) -> None:
    """Test hook: make the handle's tensor-core GEMM withhold its first stage so
    that its bounded waits expire after `wait_tries` tries (see the header)."""
    _check(_lib.qlinear_test_stall(h.ptr, int(bool(enable)), wait_tries), "qlinear_test_stall")


def qlinear_info(h: QLinearHandle) -> dict:
    info = ql_info_t()
    _check(_lib.qlinear_info(h.ptr, ctypes.byref(info)), "qlinear_info")
    d = {f: getattr(info, f) for f, _ in ql_info_t._fields_}
    for f in ("part_rows", "part_kv"):
        d[f] = list(d[f])[: info.nparts]
    return d


def qlinear_destroy(h: QLinearHandle) -> None:
    if h.ptr:
        _check(_lib.qlinear_destroy(h.ptr), "qlinear_destroy")
        h.ptr = None


def qlinear_profile_enable(h: QLinearHandle, capacity: int) -> None:
    _check(_lib.qlinear_profile_enable(h.ptr, capacity), "qlinear_profile_enable")


def qlinear_profile_read(h: QLinearHandle):
    """(summed milliseconds of the recorded main-kernel launches, number of recorded slots)."""
    ms, n = ctypes.c_double(), ctypes.c_int()
    _check(_lib.qlinear_profile_read(h.ptr, ctypes.byref(ms), ctypes.byref(n)), "qlinear_profile_read")
    return ms.value, n.value


def lib_path() -> str:
    return _LIB_PATH


def raw_library():
    """The ctypes handle of libqlinear.so (for tests that call the ABI directly)."""
    return _lib
