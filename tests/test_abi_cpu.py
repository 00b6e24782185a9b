"""The C ABI without a GPU: the library builds for sm_100a, loads, exports every
function include/qlinear.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tcm():
    from trellis_coded_matmul_b200 import build
    build.build()
    import trellis_coded_matmul_b200 as tcm
    return tcm


def _declared():
    text = open(os.path.join(ROOT, "include", "qlinear.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlinear_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = _declared()
    for n in ("qlinear_create", "qlinear_create_mixed", "qlinear_forward", "qlinear_decode",
              "qlinear_eval_code", "qlinear_get_status", "qlinear_destroy", "qlinear_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(tcm):
    lib = ctypes.CDLL(tcm.lib_path())
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(tcm.ABI_SYMBOLS) | {n for n in _declared() if n not in tcm.ABI_SYMBOLS}
    assert sorted(tcm.ABI_SYMBOLS) == _declared()


def test_strerror(tcm):
    assert tcm.qlinear_strerror(0) == "ok"
    assert tcm.qlinear_strerror(tcm.QL_E_ARG) == "invalid argument"
    assert tcm.qlinear_strerror(12345) == "unknown status"


def _create(lib, tcm, m=256, n=256, k=2, L=16, V=1, kind=0, Q=0, n_words=None, alpha=1.0, out=True):
    h = ctypes.c_void_p()
    code = tcm.ql_code_t(kind, Q, None)
    nw = m * n * k // 32 if n_words is None else n_words
    return lib.qlinear_create(ctypes.byref(h) if out else None, m, n, k, L, V, code, None, nw, None, None, alpha)


def test_create_rejects_bad_arguments_on_the_host(tcm):
    lib = tcm.raw_library()
    assert _create(lib, tcm, out=False) == tcm.QL_E_ARG
    assert _create(lib, tcm, m=0) == tcm.QL_E_ARG
    assert _create(lib, tcm, n=100) == tcm.QL_E_UNSUPPORTED          # n not a multiple of 256
    assert _create(lib, tcm, m=40) == tcm.QL_E_UNSUPPORTED           # m not a multiple of 16
    assert _create(lib, tcm, k=5) == tcm.QL_E_UNSUPPORTED
    assert _create(lib, tcm, L=17) == tcm.QL_E_UNSUPPORTED
    assert _create(lib, tcm, L=1, k=2) == tcm.QL_E_UNSUPPORTED       # L < kV
    assert _create(lib, tcm, V=2, kind=tcm.QL_CODE_1MAD) == tcm.QL_E_UNSUPPORTED
    assert _create(lib, tcm, kind=7) == tcm.QL_E_ARG
    assert _create(lib, tcm, n_words=7) == tcm.QL_E_ARG
    assert _create(lib, tcm, alpha=float("nan")) == tcm.QL_E_ARG
    assert _create(lib, tcm, m=65536 * 2, n=256) == tcm.QL_E_UNSUPPORTED  # Hadamard block > 32768
    # well-formed sizes but host (non-device) pointers
    assert _create(lib, tcm) == tcm.QL_E_ARG


def test_other_entry_points_reject_null_handles(tcm):
    lib = tcm.raw_library()
    assert lib.qlinear_forward(None, None, 1, None, 0, None) == tcm.QL_E_ARG
    assert lib.qlinear_forward_host(None, None, 1, None, 0, None) == tcm.QL_E_ARG
    assert lib.qlinear_decode(None, None, None) == tcm.QL_E_ARG
    assert lib.qlinear_get_status(None) == tcm.QL_E_ARG
    assert lib.qlinear_destroy(None) == tcm.QL_E_ARG
    assert lib.qlinear_info(None, None) == tcm.QL_E_ARG
    code = tcm.ql_code_t(0, 0, None)
    assert lib.qlinear_eval_code(code, 17, 1, None, 4, None, None) == tcm.QL_E_ARG
    assert lib.qlinear_eval_code(tcm.ql_code_t(1, 0, None), 16, 2, None, 4, None, None) == tcm.QL_E_UNSUPPORTED
    mixed = lib.qlinear_create_mixed
    h = ctypes.c_void_p()
    assert mixed(ctypes.byref(h), 64, 256, 64, 2, 3, 16, 1, code, None, 0, None, None, 1.0) == tcm.QL_E_ARG


def test_forward_noalloc_rejects_bad_arguments_on_the_host(tcm):
    lib = tcm.raw_library()
    assert lib.qlinear_forward_noalloc(None, None, 1, None, tcm.QL_F32, None) == tcm.QL_E_ARG
    assert tcm.qlinear_strerror(tcm.QL_E_SCRATCH).startswith("request exceeds the fixed scratch")
    header = open(os.path.join(ROOT, "include", "qlinear.h")).read()
    assert re.search(r"#define QL_NOALLOC_SCRATCH_BYTES \(2 \* 1024 \* 1024\)", header)
    assert tcm.QL_NOALLOC_SCRATCH_BYTES == 2 * 1024 * 1024



def test_create_parts_rejects_bad_arguments_on_the_host(tcm):
    lib = tcm.raw_library()
    code = tcm.ql_code_t(0, 0, None)

    def create(rows, ks, m=None, n=256, n_words=None):
        h = ctypes.c_void_p()
        m = sum(rows) if m is None else m
        nw = sum(r * n * k for r, k in zip(rows, ks)) // 32 if n_words is None else n_words
        r = (ctypes.c_int * max(1, len(rows)))(*rows)
        k = (ctypes.c_int * max(1, len(ks)))(*ks)
        return lib.qlinear_create_parts(ctypes.byref(h), m, n, len(rows), r, k, 16, 1, code, None, nw, None, None, 1.0)

    assert create([], []) == tcm.QL_E_ARG                          # no parts
    assert create([16] * 9, [2] * 9) == tcm.QL_E_ARG               # more than 8 parts
    assert create([16, 24], [2, 3]) == tcm.QL_E_UNSUPPORTED        # m = 40: not a multiple of 16
    assert create([16, 16], [2, 3], m=48) == tcm.QL_E_ARG          # parts do not add up to m
    assert create([16, 8, 8], [2, 3, 3]) == tcm.QL_E_ARG           # part rows not a multiple of 16
    assert create([16, 16], [2, 5]) == tcm.QL_E_UNSUPPORTED        # k out of range
    assert create([16, 16], [2, 3], n_words=7) == tcm.QL_E_ARG     # wrong stream length
    assert create([16, 16], [2, 3]) == tcm.QL_E_ARG                # valid shape, null device pointers


def test_create_kv_rejects_bad_arguments_on_the_host(tcm):
    """Bitrates as bits per trellis step: V <= kv <= 4V (1 to 4 bits per
    weight, half numbers with V = 2), L >= kv; the stream holds rows * (n / V)
    * kv bits per part; the table code's codebook has at most 2^9 entries."""
    lib = tcm.raw_library()

    def create(rows, kvs, V=2, L=16, kind=tcm.QL_CODE_HYB, Q=9, n=256, n_words=None):
        h = ctypes.c_void_p()
        nw = sum(r * (n // V) * kv for r, kv in zip(rows, kvs)) // 32 if n_words is None else n_words
        r = (ctypes.c_int * max(1, len(rows)))(*rows)
        k = (ctypes.c_int * max(1, len(kvs)))(*kvs)
        code = tcm.ql_code_t(kind, Q, None)
        return lib.qlinear_create_kv(ctypes.byref(h), sum(rows), n, len(rows), r, k, L, V, code, None, nw, None,
                                     None, 1.0)

    assert create([16], [1]) == tcm.QL_E_UNSUPPORTED               # 0.5 bits per weight
    assert create([16], [9]) == tcm.QL_E_UNSUPPORTED               # 4.5 bits per weight
    assert create([16], [5], L=4) == tcm.QL_E_UNSUPPORTED          # L < kV
    assert create([16], [5], V=3) == tcm.QL_E_ARG                  # V is 1 or 2
    assert create([16], [5], n_words=41) == tcm.QL_E_ARG           # 16 rows * 128 steps * 5 bits = 320 words
    assert create([16], [5], n_words=320) == tcm.QL_E_ARG          # right length, null device pointers
    assert create([16], [5], L=10, kind=tcm.QL_CODE_TABLE) == tcm.QL_E_UNSUPPORTED  # 2^10-entry codebook
    assert create([16], [5], L=5, kind=tcm.QL_CODE_TABLE) == tcm.QL_E_ARG           # valid, null pointers
    assert create([16], [3], V=1, kind=tcm.QL_CODE_1MAD) == tcm.QL_E_ARG            # 3 bits, V = 1
    assert create([16, 16], [5, 6], n_words=320 + 384) == tcm.QL_E_ARG              # 2.5 + 3 bits


def test_encode_rejects_bad_arguments_on_the_host(tcm):
    lib = tcm.raw_library()
    code = tcm.ql_code_t(1, 0, None)
    assert lib.qlinear_encode(code, 12, 2, 1, None, -1, None, None, None) == tcm.QL_E_ARG
    assert lib.qlinear_encode(code, 17, 2, 1, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # L > 16
    assert lib.qlinear_encode(code, 12, 5, 1, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # k > 4
    assert lib.qlinear_encode(code, 3, 2, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED   # L < kV
    assert lib.qlinear_encode(code, 12, 2, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # 3INST: V = 1
    assert lib.qlinear_encode(code, 12, 2, 1, None, 0, None, None, None) == tcm.QL_OK             # nothing to do
    assert lib.qlinear_encode(code, 12, 2, 1, None, 4, None, None, None) == tcm.QL_E_ARG          # null pointers
    hyb = tcm.ql_code_t(tcm.QL_CODE_HYB, 9, None)
    enc_kv = lib.qlinear_encode_kv
    assert enc_kv(hyb, 12, 5, 2, None, 4, None, None, None) == tcm.QL_E_ARG      # 2.5 bits: valid, null pointers
    assert enc_kv(hyb, 12, 1, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # 0.5 bits
    assert enc_kv(hyb, 12, 9, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # more than 8 bits per step
    assert enc_kv(hyb, 4, 5, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED   # L < kV
    assert enc_kv(code, 12, 3, 2, None, 4, None, None, None) == tcm.QL_E_UNSUPPORTED  # 3INST: V = 1


def test_info_struct_layout_matches_the_header(tcm, tmp_path):
    """The binding's ctypes mirror of ql_info_t has the C struct's size and
    field offsets (compiled from include/qlinear.h with the host compiler)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = [f for f, _ in tcm.ql_info_t._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"qlinear.h\"\nint main(void) {\n"
                   "  printf(\"%zu\\n\", sizeof(ql_info_t));\n"
                   + "".join(f"  printf(\"%zu\\n\", offsetof(ql_info_t, {f}));\n" for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()]
    assert out[0] == ctypes.sizeof(tcm.ql_info_t)
    assert out[1:] == [getattr(tcm.ql_info_t, f).offset for f in fields]
    code = tmp_path / "code.c"
    code.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"qlinear.h\"\nint main(void) {\n"
                    "  printf(\"%zu %zu %zu %zu\\n\", sizeof(ql_code_t), offsetof(ql_code_t, kind),"
                    " offsetof(ql_code_t, Q), offsetof(ql_code_t, lut));\n  return 0;\n}\n")
    exe2 = tmp_path / "code"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(code), "-o", str(exe2)], check=True)
    got = [int(v) for v in subprocess.run([str(exe2)], check=True, capture_output=True, text=True).stdout.split()]
    assert got == [ctypes.sizeof(tcm.ql_code_t), tcm.ql_code_t.kind.offset, tcm.ql_code_t.Q.offset,
                   tcm.ql_code_t.lut.offset]


def test_host_validation_never_accepts_null_buffers(tcm):
    """Random shapes, bitrates, codes and stream lengths with null device
    buffers: every create entry point rejects them on the host with QL_E_ARG
    or QL_E_UNSUPPORTED (never QL_OK, never a crash), whatever else is wrong."""
    hyp = pytest.importorskip("hypothesis")
    st = pytest.importorskip("hypothesis.strategies")
    lib = tcm.raw_library()
    bad = {tcm.QL_E_ARG, tcm.QL_E_UNSUPPORTED}

    @hyp.settings(max_examples=400, deadline=None, derandomize=True)
    @hyp.given(m=st.integers(-16, 1 << 20), n=st.integers(-256, 1 << 20), k=st.integers(-1, 6),
               L=st.integers(-1, 18), V=st.integers(0, 3), kind=st.integers(-1, 4), Q=st.integers(-1, 11),
               nparts=st.integers(0, 9), kv=st.lists(st.integers(-1, 10), min_size=9, max_size=9),
               rows=st.lists(st.integers(-16, 4096), min_size=9, max_size=9), exact=st.booleans())
    def check(m, n, k, L, V, kind, Q, nparts, kv, rows, exact):
        code = tcm.ql_code_t(kind, Q, None)
        h = ctypes.c_void_p()
        nw = (m * n * max(k, 0)) // 32 if exact and m > 0 and n > 0 else 7
        assert lib.qlinear_create(ctypes.byref(h), m, n, k, L, V, code, None, max(nw, 0), None, None, 1.0) in bad
        r = (ctypes.c_int * 9)(*rows)
        kvs = (ctypes.c_int * 9)(*kv)
        tot = sum(max(x, 0) * max(n, 0) // max(V, 1) * max(y, 0) for x, y in zip(rows[:nparts], kv[:nparts])) // 32
        nw2 = tot if exact else 7
        assert lib.qlinear_create_kv(ctypes.byref(h), sum(rows[:nparts]), n, nparts, r, kvs, L, V, code, None,
                                     max(nw2, 0), None, None, 1.0) in bad
        assert lib.qlinear_create_parts(ctypes.byref(h), sum(rows[:nparts]), n, nparts, r, kvs, L, V, code, None,
                                        max(nw2, 0), None, None, 1.0) in bad
        assert h.value is None

    check()


def test_encode_and_eval_validation_never_accept_null_buffers(tcm):
    """Random encoder and code-evaluation arguments with null device buffers:
    rejected on the host (QL_E_ARG / QL_E_UNSUPPORTED), or QL_OK only when
    there is nothing to do (zero blocks or states) and the arguments are valid."""
    hyp = pytest.importorskip("hypothesis")
    st = pytest.importorskip("hypothesis.strategies")
    lib = tcm.raw_library()
    rejected = {tcm.QL_E_ARG, tcm.QL_E_UNSUPPORTED}

    @hyp.settings(max_examples=400, deadline=None, derandomize=True)
    @hyp.given(L=st.integers(-1, 18), kv=st.integers(-1, 10), k=st.integers(-1, 6), V=st.integers(0, 3),
               kind=st.integers(-1, 4), Q=st.integers(-1, 11), count=st.integers(-2, 5))
    def check(L, kv, k, V, kind, Q, count):
        code = tcm.ql_code_t(kind, Q, None)
        for rc in (lib.qlinear_encode_kv(code, L, kv, V, None, count, None, None, None),
                   lib.qlinear_encode(code, L, k, V, None, count, None, None, None),
                   lib.qlinear_eval_code(code, L, V, None, count, None, None)):
            assert rc in rejected or (rc == tcm.QL_OK and count == 0)

    check()
