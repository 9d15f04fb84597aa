"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/kq.h, and rejects bad arguments with the
documented status before touching the device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mxfp4_activations_b200 import build, _lib

    build.build()
    return _lib.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "kq.h")).read()
    return sorted(set(re.findall(r"^KQ_API\s+[\w\s\*]+?\b(kq_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("kq_expand_blocks", "kq_quantize", "kq_dequantize", "kq_ref_smooth_quantize",
                     "kq_ref_fwht_quantize", "kq_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from mxfp4_activations_b200 import _lib

    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in _lib.EXPORTED


def test_status_strings_and_version(lib):
    assert lib.kq_abi_version() == 204
    for code in range(8):
        s = lib.kq_status_string(code).decode()
        assert s.startswith("KQ_")
    assert lib.kq_status_string(99).decode() == "unknown kq_status"


P = ctypes.c_void_p


def q(lib, x=16 * 1024, M=4, d=64, ldx=64, mats=16 * 2048, dtype=0, fac=16 * 4096, qq=16 * 8192,
      sc=16 * 9000, var=2, layout=0):
    return lib.kq_quantize(P(x) if x else None, M, d, ldx, P(mats) if mats else None, dtype,
                           P(fac) if fac else None, P(qq) if qq else None, P(sc) if sc else None, var, layout, None)


def test_quantize_argument_errors_return_before_launch(lib):
    assert q(lib, d=33, ldx=40) == 2          # d % 32
    assert q(lib, d=64, ldx=32) == 2          # ldx < d
    assert q(lib, M=-1) == 1                  # negative size
    assert q(lib, x=0) == 1                   # null x
    assert q(lib, x=16 * 1024 + 2) == 3       # x not 16-byte aligned
    assert q(lib, ldx=68) == 3                # row stride not a multiple of 8 elements
    assert q(lib, qq=0) == 1                  # null codes
    assert q(lib, qq=16 * 8192 + 4) == 3      # codes not 16-byte aligned
    assert q(lib, mats=0) == 1
    assert q(lib, var=9) == 1                 # bad variant enum
    assert q(lib, layout=2) == 1              # bad scale layout enum
    qn = lambda **kw: lib.kq_quantize_n(P(16 * 1024), kw.get("M", 4), kw.get("d", 128), kw.get("ldx", 128),
                                        kw.get("log2n", 6), P(16 * 2048), kw.get("dtype", 0),
                                        P(16 * 4096) if kw.get("fac", 1) else None, P(16 * 8192), P(16 * 9000),
                                        kw.get("var", 2), 0, None)
    assert qn(log2n=8) == 1                   # transform blocks of 16 to 128 elements
    assert qn(log2n=3) == 1
    assert qn(log2n=7, d=96, ldx=96) == 2     # 128-element blocks need d % 128 == 0
    assert qn(d=96, ldx=96) == 2              # 64-element blocks need d % 64 == 0
    assert qn(var=1) == 5                     # no tensor-core variant for 64-element blocks
    assert qn(dtype=1) == 5                   # nor bf16 matrices
    assert qn(fac=0) == 1                     # the butterfly needs the factored form
    assert q(lib, dtype=7) == 1               # bad dtype enum
    assert q(lib, fac=0) == 1                 # butterfly needs the factored form
    assert q(lib, dtype=1) == 5               # bf16 matrices need the tensor-core variant
    assert q(lib, M=0) == 0                   # empty input: no-op
    assert q(lib, x=0, M=0) == 1              # null x is still an argument error


def test_other_entry_points_argument_errors(lib):
    assert lib.kq_expand_blocks(None, 4, 0, 0, P(64), None) == 1
    assert lib.kq_expand_blocks(P(64), -1, 0, 0, P(64), None) == 1
    assert lib.kq_expand_blocks(P(64), 4, 0, 5, P(64), None) == 1
    assert lib.kq_expand_blocks(P(64), 4, 3, 0, P(64), None) == 1     # mode: 0 K, 1 K^-1, 2 K^-T
    assert lib.kq_expand_blocks_n(P(64), 4, 8, 0, 0, P(64), None) == 1  # at most 2^7-element blocks
    assert lib.kq_expand_blocks_n(P(64), 4, 0, 0, 0, P(64), None) == 1
    assert lib.kq_expand_blocks_n(P(64), 0, 6, 0, 0, P(64), None) == 0
    assert lib.kq_expand_factored_n(P(64), 4, 8, P(64), None) == 1     # butterfly form for 16 to 128
    assert lib.kq_expand_factored_n(P(64), 3, 4, P(64), None) == 2     # 16-element blocks come in pairs
    assert lib.kq_expand_factored_n(P(64), 4, 6, P(72), None) == 3
    assert lib.kq_expand_blocks(P(64), 4, -1, 0, P(64), None) == 1
    assert lib.kq_expand_blocks(P(64), 0, 0, 0, P(64), None) == 0
    assert lib.kq_expand_factored(P(64), 4, P(68), None) == 3
    assert lib.kq_dequantize(P(16), P(16), 4, 48, None, 0, P(16), 0, None) == 2
    assert lib.kq_dequantize(P(16), P(16), 0, 64, None, 0, P(16), 0, None) == 0
    assert lib.kq_dequantize(P(18), P(16), 4, 64, None, 0, P(16), 0, None) == 3
    assert lib.kq_ref_smooth_quantize(P(16), 4, 64, 64, None, P(16), P(16), None) == 1
    assert lib.kq_ref_smooth_quantize(P(16), 4, 64, 64, P(20), P(16), P(16), None) == 3
    assert lib.kq_ref_fwht_quantize(P(16), 4, 40, 40, P(16), P(16), None) == 2
    assert lib.kq_e2m1_pack(P(16), 7, P(16), None) == 2
    assert lib.kq_e2m1_pack(P(16), 0, P(16), None) == 0
    assert lib.kq_e2m1_pack(P(20), 8, P(16), None) == 3
    # kq_gemm_mxf4(a_q, a_scales, M, b_q, b_scales, N, K, c, ldc, c_dtype, stream)
    g = lib.kq_gemm_mxf4
    assert g(P(16), P(16), 4, P(16), P(16), 4, 48, P(16), 4, 0, None) == 2    # K not a multiple of 32
    assert g(P(16), P(16), 4, P(16), P(16), 4, 64, P(16), 3, 0, None) == 2    # ldc < N
    assert g(P(16), P(16), 4, P(16), P(16), 4, 0, P(16), 4, 0, None) == 2     # K = 0 with work to do
    assert g(P(16), P(16), 0, P(16), P(16), 4, 64, P(16), 4, 0, None) == 0    # M = 0: no-op
    assert g(P(16), P(16), 4, P(16), P(16), -1, 64, P(16), 4, 0, None) == 1
    assert g(P(16), P(16), 4, P(16), P(16), 4, 64, P(16), 4, 2, None) == 1    # bad output dtype
    assert g(None, P(16), 4, P(16), P(16), 4, 64, P(16), 4, 0, None) == 1
    assert g(P(16), P(16), 4, P(24), P(16), 4, 64, P(16), 4, 0, None) == 3    # codes 16-byte aligned
    assert g(P(16), P(16), 4, P(16), P(16), 4, 64, P(18), 4, 0, None) == 3    # fp32 C 4-byte aligned


def test_binding_fails_loudly_without_library(tmp_path):
    from mxfp4_activations_b200 import _lib

    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib._lib_backup = _lib._lib
        try:
            _lib._lib = None
            _lib.load(str(tmp_path / "missing.so"))
        finally:
            _lib._lib = _lib._lib_backup
