"""Host-side checks of the C ABI: the library builds/loads on a machine without a
GPU, exports every function the header declares, and its host-only logic
(level table, byte sizes, argument validation) agrees with the oracle.  No
compute call reaches a GPU here."""
import ctypes

import numpy as np
import pytest

from bit_nf4_quantized_19_b200 import _abi, build
from oracle import nf4 as onf4


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def test_every_declared_symbol_is_exported(L):
    names = _abi.header_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
        assert n in _abi.SIGNATURES, f"binding lacks {n}"
    assert set(_abi.SIGNATURES) == set(names)


def test_version_and_status_strings(L):
    assert L.qlora_version() >= 100
    for code in range(9):
        s = L.qlora_status_string(code)
        assert s and s != b"unknown status"
    assert L.qlora_status_string(99) == b"unknown status"


def test_level_table_bit_identical_to_oracle(L):
    """The library builds its table with its own inverse-CDF code (Newton on
    erfc); the oracle uses scipy's ndtri.  Both must give the same fp32 bits."""
    buf = (ctypes.c_float * 16)()
    L.qlora_nf4_levels(buf)
    lib_levels = np.frombuffer(buf, dtype=np.float32).copy()
    assert np.array_equal(lib_levels.view(np.uint32), onf4.nf4_levels().view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(1, 1), (1, 7), (3, 21), (64, 64), (1024, 1024),
                                       (4096, 4096), (11008, 4096), (1, 1_000_000_000)])
def test_nf4_bytes_match_oracle(L, rows, cols):
    c, q, s = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    tot = L.qlora_nf4_bytes(rows, cols, ctypes.byref(c), ctypes.byref(q), ctypes.byref(s))
    assert (c.value, q.value, s.value) == onf4.storage_bytes(rows * cols)
    assert tot == c.value + q.value + s.value


def test_bits_per_value_closed_form(L):
    n = 4096 * 4096
    tot = L.qlora_nf4_bytes(4096, 4096, None, None, None)
    assert tot == 8_388_608 + 262_144 + 4_096
    assert 8.0 * tot / n == 4.126953125


def test_argument_errors_before_any_launch(L):
    null = _abi.NF4Struct(0, 0, 0, 4, 4)
    assert L.qlora_nf4_quantize(None, 4, 4, ctypes.byref(null), None) == 1
    assert L.qlora_nf4_dequant(ctypes.byref(null), ctypes.c_void_p(16), None) == 1
    bad = _abi.NF4Struct(16, 18, 32, 128, 128)            # q8 pointer misaligned
    assert L.qlora_nf4_dequant(ctypes.byref(bad), ctypes.c_void_p(64), None) == 2
    ok = _abi.NF4Struct(16, 32, 48, 128, 128)
    # r out of range / not a multiple of 8
    for r in (0, 4, 12, 136):
        assert L.qlora_linear_fwd(ctypes.c_void_p(16), 4, ctypes.byref(ok), ctypes.c_void_p(16),
                                  ctypes.c_void_p(16), r, 1.0, ctypes.c_void_p(16), None,
                                  ctypes.c_void_p(16), 1 << 20, None) == 1
    # shapes the fused GEMM does not cover
    odd = _abi.NF4Struct(16, 32, 48, 100, 128)
    assert L.qlora_linear_fwd(ctypes.c_void_p(16), 4, ctypes.byref(odd), ctypes.c_void_p(16),
                              ctypes.c_void_p(16), 8, 1.0, ctypes.c_void_p(16), None,
                              ctypes.c_void_p(16), 1 << 20, None) == 3
    # misaligned activation pointer
    assert L.qlora_linear_fwd(ctypes.c_void_p(18), 4, ctypes.byref(ok), ctypes.c_void_p(16),
                              ctypes.c_void_p(16), 8, 1.0, ctypes.c_void_p(16), None,
                              ctypes.c_void_p(16), 1 << 20, None) == 2
    assert L.qlora_linear_bwd(None, ctypes.c_void_p(16), None, 4, ctypes.byref(ok),
                              ctypes.c_void_p(16), ctypes.c_void_p(16), 8, 1.0, None,
                              ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
                              1 << 20, None) == 1
    assert L.qlora_selftest_wait_timeout(0, None) == 1
    flags = ctypes.c_uint32()
    assert L.qlora_get_device_status(None, None) == 1


def test_wait_limit_setter_roundtrip(L):
    old = L.qlora_set_wait_limit_us(123)
    assert L.qlora_set_wait_limit_us(old) == 123


def test_gemm_pairing_setter_roundtrip(L):
    """The launch-shape switch is process-wide host state: each call returns the
    previous setting, as 0 or 1."""
    prev = L.qlora_set_gemm_pairing(0)
    assert prev in (0, 1)
    assert L.qlora_set_gemm_pairing(7) == 0
    assert L.qlora_set_gemm_pairing(prev) == 1


def test_gemm_units_without_device(L):
    """Without a B200 the unit query reports no device and leaves its outputs alone."""
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    a, b = ctypes.c_int(-1), ctypes.c_int(-1)
    assert L.qlora_gemm_units(ctypes.byref(a), ctypes.byref(b)) != 0
    assert (a.value, b.value) == (-1, -1)


def test_plain_c_consumer(L, tmp_path):
    """tests/csrc/abi_consumer.c: a C11 program built with gcc against the header
    alone (-Wall -Wextra -pedantic -Werror) and linked to the shared library runs
    the host-side checks; its exit status is its number of failed checks."""
    import os
    import subprocess
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    pkg = os.path.dirname(build.LIB_PATH)
    exe = str(tmp_path / "abi_consumer")
    cc = subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(root, "include"), os.path.join(here, "csrc", "abi_consumer.c"),
                         "-L", pkg, "-lqlora_nf4", f"-Wl,-rpath,{pkg}", "-lm", "-o", exe],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert "all checks passed" in run.stdout


def _c_kind(decl: str) -> str:
    d = " ".join(decl.split())
    if "*" in d or "[" in d or d.startswith("qlora_stream_t"):
        return "ptr"
    for prefix, kind in (("int64_t", "i64"), ("uint32_t", "u32"), ("size_t", "sz"), ("float", "f32"),
                         ("qlora_status", "int"), ("int", "int")):
        if d == prefix or d.startswith(prefix + " "):
            return kind
    raise AssertionError(f"unknown C type in {decl!r}")


def _py_kind(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or isinstance(t, type(ctypes.POINTER(ctypes.c_int))):
        return "ptr"
    for ct, kind in ((ctypes.c_int64, "i64"), (ctypes.c_uint32, "u32"), (ctypes.c_size_t, "sz"),
                     (ctypes.c_float, "f32"), (ctypes.c_int, "int")):
        if t is ct:
            return kind
    raise AssertionError(f"unknown ctypes type {t!r}")


def test_binding_signatures_match_the_header():
    """Every prototype in include/qlora_nf4.h has the same return type and the same
    parameter count and kinds (pointer, int64, int, uint32, size_t, float) as its
    ctypes declaration, so the binding cannot drift from the C ABI."""
    import re
    text = re.sub(r"/\*.*?\*/", "", open(_abi.HEADER).read(), flags=re.S)
    protos = re.findall(r"([A-Za-z_][\w \t\*]*?)\b(qlora_\w+)\s*\(([^)]*)\)\s*;", text)
    assert len(protos) == len(_abi.SIGNATURES)
    for ret, name, params in protos:
        res, args = _abi.SIGNATURES[name]
        ret = " ".join(ret.split())
        want_ret = "void" if ret == "void" else _c_kind(ret)
        assert _py_kind(res) == want_ret, (name, ret, res)
        plist = [] if params.strip() in ("", "void") else params.split(",")
        assert [_c_kind(p) for p in plist] == [_py_kind(a) for a in args], name
