"""ctypes wrapper of the C oracle (kq_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` use this module.  The product package
never imports it.  It holds no arithmetic of its own: every function marshals
numpy arrays into the C oracle and back.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkq_oracle.so")

F32 = 0
BF16 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "kq_oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB_PATH))
    return _lib


def compile_copy(src_text: str, out_path: str) -> str:
    """Compile another text of kq_oracle.c, with the flags of ``build``, into
    out_path (the tests plant mistakes in copies of the source)."""
    c_path = os.path.splitext(out_path)[0] + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-I", _HERE,
                           "-o", out_path, c_path, "-lm"])
    return out_path


@contextlib.contextmanager
def using_library(path: str):
    """Route every call of this module through the oracle build at path."""
    global _lib
    saved = lib()
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _configure(L):
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.kqo_factor.argtypes = [ctypes.c_float] * 3 + [P]
    L.kqo_factor_inverse.argtypes = [ctypes.c_float] * 3 + [P]
    L.kqo_kron.argtypes = [P, I, P, I, P]
    L.kqo_expand_f64.argtypes = [P, I64, I, P]
    L.kqo_expand.argtypes = [P, I64, I, I, P]
    L.kqo_expand_n_f64.argtypes = [P, I64, I, I, P]
    L.kqo_expand_n.argtypes = [P, I64, I, I, I, P]
    L.kqo_transform_n.argtypes = [P, I64, I64, I64, P, I, I, P]
    L.kqo_quantize_n.argtypes = [P, I64, I64, I64, P, I, I, P, P]
    L.kqo_bf16_from_f64.argtypes = [ctypes.c_double]
    L.kqo_bf16_from_f64.restype = ctypes.c_uint16
    L.kqo_hadamard.argtypes = [I, P]
    L.kqo_e8m0.argtypes = [ctypes.c_float]
    L.kqo_e8m0.restype = I
    L.kqo_e8m0_many.argtypes = [P, I64, P]
    L.kqo_e8m0_many.restype = None
    L.kqo_e2m1.argtypes = [ctypes.c_float]
    L.kqo_e2m1.restype = I
    L.kqo_e2m1_value.argtypes = [I]
    L.kqo_e2m1_value.restype = ctypes.c_double
    L.kqo_e2m1_pack.argtypes = [P, I64, P]
    L.kqo_transform.argtypes = [P, I64, I64, I64, P, I, P]
    L.kqo_mx_quantize.argtypes = [P, I64, I64, P, P]
    L.kqo_quantize.argtypes = [P, I64, I64, I64, P, I, P, P]
    L.kqo_smooth_quantize.argtypes = [P, I64, I64, I64, P, P, P]
    L.kqo_fwht_quantize.argtypes = [P, I64, I64, I64, P, P]
    L.kqo_dequantize.argtypes = [P, P, I64, I64, P, I, P]
    L.kqo_mx_gemm.argtypes = [P, P, I64, P, P, I64, I64, P]
    L.kqo_adaln.argtypes = [P, I64, I64, I64, P, P, I64, ctypes.c_float, P, P]
    L.kqo_adaln_quantize.argtypes = [P, I64, I64, I64, P, P, I64, ctypes.c_float, P, I, P, P, P]
    for name in ("kqo_factor", "kqo_factor_inverse", "kqo_kron", "kqo_expand_f64", "kqo_expand",
                 "kqo_hadamard", "kqo_e2m1_pack", "kqo_transform", "kqo_mx_quantize", "kqo_quantize",
                 "kqo_smooth_quantize", "kqo_fwht_quantize", "kqo_dequantize", "kqo_mx_gemm", "kqo_adaln", "kqo_adaln_quantize"):
        getattr(L, name).restype = None
    return L


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    assert x.dtype == np.uint16, "activations are passed as bf16 bit patterns (uint16)"
    return np.ascontiguousarray(x)


def factor(l: float, u: float, v: float, inverse: bool = False) -> np.ndarray:
    F = np.zeros(4, np.float64)
    (lib().kqo_factor_inverse if inverse else lib().kqo_factor)(l, u, v, _p(F))
    return F.reshape(2, 2)


def kron(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    A = np.ascontiguousarray(A, np.float64)
    B = np.ascontiguousarray(B, np.float64)
    out = np.zeros((A.shape[0] * B.shape[0],) * 2, np.float64)
    lib().kqo_kron(_p(A), A.shape[0], _p(B), B.shape[0], _p(out))
    return out


def expand_f64(params: np.ndarray, inverse: bool = False) -> np.ndarray:
    params = np.ascontiguousarray(params, np.float32).reshape(-1, 5, 3)
    nb = params.shape[0]
    K = np.zeros((nb, 32, 32), np.float64)
    lib().kqo_expand_f64(_p(params), nb, int(inverse), _p(K))
    return K


def expand(params: np.ndarray, dtype: int = F32, inverse: bool = False) -> np.ndarray:
    """fp32 matrices (dtype F32) or bf16 bit patterns as uint16 (dtype BF16)."""
    params = np.ascontiguousarray(params, np.float32).reshape(-1, 5, 3)
    nb = params.shape[0]
    out = np.zeros((nb, 32, 32), np.float32 if dtype == F32 else np.uint16)
    lib().kqo_expand(_p(params), nb, int(inverse), dtype, _p(out))
    return out


def bf16_from_f64(a: float) -> int:
    return int(lib().kqo_bf16_from_f64(float(a)))


def hadamard(n: int) -> np.ndarray:
    H = np.zeros((1 << n, 1 << n), np.float64)
    lib().kqo_hadamard(n, _p(H))
    return H


def e8m0(amax: float) -> int:
    return int(lib().kqo_e8m0(float(amax)))


def e8m0_many(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, np.float32).reshape(-1)
    out = np.zeros(a.size, np.uint8)
    lib().kqo_e8m0_many(_p(a), a.size, _p(out))
    return out


def e2m1(v: float) -> int:
    return int(lib().kqo_e2m1(float(v)))


def e2m1_value(code: int) -> float:
    return float(lib().kqo_e2m1_value(int(code)))


def e2m1_pack(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).reshape(-1)
    out = np.zeros(v.size // 2, np.uint8)
    lib().kqo_e2m1_pack(_p(v), v.size, _p(out))
    return out


def _mats_dtype(mats: np.ndarray) -> int:
    if mats.dtype == np.float32:
        return F32
    if mats.dtype == np.uint16:
        return BF16
    raise TypeError("mats must be float32 or bf16 bits (uint16)")


def transform(x: np.ndarray, mats: np.ndarray, d: int | None = None) -> np.ndarray:
    x = _bf16_bits(x)
    M, ldx = x.shape
    d = ldx if d is None else d
    mats = np.ascontiguousarray(mats)
    y = np.zeros((M, d), np.float32)
    lib().kqo_transform(_p(x), M, d, ldx, _p(mats), _mats_dtype(mats), _p(y))
    return y


def mx_quantize(y: np.ndarray):
    y = np.ascontiguousarray(y, np.float32)
    M, d = y.shape
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    lib().kqo_mx_quantize(_p(y), M, d, _p(q), _p(s))
    return q, s


def quantize(x: np.ndarray, mats: np.ndarray, d: int | None = None):
    x = _bf16_bits(x)
    M, ldx = x.shape
    d = ldx if d is None else d
    mats = np.ascontiguousarray(mats)
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    lib().kqo_quantize(_p(x), M, d, ldx, _p(mats), _mats_dtype(mats), _p(q), _p(s))
    return q, s


def smooth_quantize(x: np.ndarray, inv_s: np.ndarray, d: int | None = None):
    x = _bf16_bits(x)
    M, ldx = x.shape
    d = ldx if d is None else d
    inv_s = np.ascontiguousarray(inv_s, np.float32)
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    lib().kqo_smooth_quantize(_p(x), M, d, ldx, _p(inv_s), _p(q), _p(s))
    return q, s


def fwht_quantize(x: np.ndarray, d: int | None = None):
    x = _bf16_bits(x)
    M, ldx = x.shape
    d = ldx if d is None else d
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    lib().kqo_fwht_quantize(_p(x), M, d, ldx, _p(q), _p(s))
    return q, s


def dequantize(q: np.ndarray, scales: np.ndarray, inv_mats: np.ndarray | None = None) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    M, d = q.shape[0], q.shape[1] * 2
    out = np.zeros((M, d), np.float64)
    if inv_mats is None:
        lib().kqo_dequantize(_p(q), _p(scales), M, d, None, F32, _p(out))
    else:
        inv_mats = np.ascontiguousarray(inv_mats)
        lib().kqo_dequantize(_p(q), _p(scales), M, d, _p(inv_mats), _mats_dtype(inv_mats), _p(out))
    return out


# ---- transform blocks of n = 2^log2n elements (MXFP4 still per 32) -------------------

def expand_n_f64(params: np.ndarray, inverse: bool = False) -> np.ndarray:
    """params [nt][log2n][3] -> K [nt][n][n] in fp64."""
    params = np.ascontiguousarray(params, np.float32)
    nt, log2n = params.shape[0], params.shape[1]
    n = 1 << log2n
    out = np.zeros((nt, n, n), np.float64)
    lib().kqo_expand_n_f64(_p(params), nt, log2n, int(bool(inverse)), _p(out))
    return out


def expand_n(params: np.ndarray, dtype: int = F32, inverse: bool = False) -> np.ndarray:
    params = np.ascontiguousarray(params, np.float32)
    nt, log2n = params.shape[0], params.shape[1]
    n = 1 << log2n
    out = np.zeros((nt, n, n), np.float32 if dtype == F32 else np.uint16)
    lib().kqo_expand_n(_p(params), nt, log2n, int(bool(inverse)), dtype, _p(out))
    return out


def transform_n(x: np.ndarray, mats: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.uint16)
    mats = np.ascontiguousarray(mats)
    M, d = x.shape
    n = mats.shape[-1]
    y = np.zeros((M, d), np.float32)
    lib().kqo_transform_n(_p(x), M, d, d, _p(mats), _mats_dtype(mats), n, _p(y))
    return y


def quantize_n(x: np.ndarray, mats: np.ndarray):
    x = np.ascontiguousarray(x, np.uint16)
    mats = np.ascontiguousarray(mats)
    M, d = x.shape
    n = mats.shape[-1]
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    lib().kqo_quantize_n(_p(x), M, d, d, _p(mats), _mats_dtype(mats), n, _p(q), _p(s))
    return q, s


# ---- the consumer: W4A4 product ------------------------------------------------------

def mx_gemm(a_q: np.ndarray, a_scales: np.ndarray, b_q: np.ndarray, b_scales: np.ndarray) -> np.ndarray:
    """c [M, N] fp64 = sum_k A(m, k) B(n, k) over MXFP4 operands with row-major scales."""
    a_q, b_q = np.ascontiguousarray(a_q, np.uint8), np.ascontiguousarray(b_q, np.uint8)
    a_scales, b_scales = np.ascontiguousarray(a_scales, np.uint8), np.ascontiguousarray(b_scales, np.uint8)
    M, N, K = a_q.shape[0], b_q.shape[0], a_q.shape[1] * 2
    assert b_q.shape[1] * 2 == K and a_scales.shape == (M, K // 32) and b_scales.shape == (N, K // 32)
    c = np.zeros((M, N), np.float64)
    lib().kqo_mx_gemm(_p(a_q), _p(a_scales), M, _p(b_q), _p(b_scales), N, K, _p(c))
    return c


# ---- the producer: AdaLN normalisation in front of the quantizer -------------------

def adaln(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, rows_per_group: int, eps: float):
    """(h bf16 bits [M, d], stats fp32 [M, 2] = (mu, rstd)) of bf16 rows x [M, d] with
    bf16 modulation vectors shift, scale [G, d]."""
    x = _bf16_bits(x)
    M, d = x.shape
    shift, scale = _bf16_bits(shift), _bf16_bits(scale)
    assert shift.shape[1] == d and scale.shape == shift.shape and shift.shape[0] * rows_per_group >= M
    h = np.zeros((M, d), np.uint16)
    stats = np.zeros((M, 2), np.float32)
    lib().kqo_adaln(_p(x), M, d, d, _p(shift), _p(scale), rows_per_group, float(eps), _p(h), _p(stats))
    return h, stats


def adaln_quantize(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, rows_per_group: int, eps: float,
                   mats: np.ndarray):
    """(q, scales, stats): adaln, then quantize with the block matrices."""
    x = _bf16_bits(x)
    M, d = x.shape
    shift, scale = _bf16_bits(shift), _bf16_bits(scale)
    mats = np.ascontiguousarray(mats)
    q = np.zeros((M, d // 2), np.uint8)
    s = np.zeros((M, d // 32), np.uint8)
    stats = np.zeros((M, 2), np.float32)
    lib().kqo_adaln_quantize(_p(x), M, d, d, _p(shift), _p(scale), rows_per_group, float(eps), _p(mats),
                             _mats_dtype(mats), _p(q), _p(s), _p(stats))
    return q, s, stats
