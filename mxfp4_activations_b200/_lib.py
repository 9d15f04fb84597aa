"""ctypes binding of libkq.so (include/kq.h).

Argument marshalling only: every function checks tensor dtypes, devices and
shapes, passes raw device pointers and the current CUDA stream to the C ABI
and raises on a non-zero status.  There is no fallback: if libkq.so is missing
or a call fails, an exception says so.  PyTorch provides device memory and
streams; all arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkq.so")

KQ_F32, KQ_BF16 = 0, 1
VARIANTS = {"auto": 0, "mma": 1, "butterfly": 2}
SCALE_LAYOUTS = {"row": 0, "mma": 1}  # row-major [M][d/32] / 128x4 tiles of block-scaled GEMMs


def scale_bytes(M: int, d: int, layout: str = "row") -> int:
    """Size of the scales buffer kq_quantize writes in the given layout."""
    if layout == "row":
        return M * (d // 32)
    return ((M + 127) // 128) * 128 * ((d + 127) // 128) * 4
STATUS = {
    0: "KQ_OK", 1: "KQ_ERR_INVALID_ARG", 2: "KQ_ERR_SHAPE", 3: "KQ_ERR_ALIGN", 4: "KQ_ERR_SINGULAR",
    5: "KQ_ERR_UNSUPPORTED", 6: "KQ_ERR_CUDA", 7: "KQ_ERR_DEVICE_TIMEOUT",
}
EXPORTED = (
    "kq_expand_blocks", "kq_expand_factored", "kq_quantize", "kq_dequantize", "kq_ref_smooth_quantize",
    "kq_expand_blocks_n", "kq_expand_factored_n", "kq_quantize_n",
    "kq_ref_fwht_quantize", "kq_e2m1_pack", "kq_get_device_error", "kq_status_string", "kq_abi_version",
    "kq_last_error", "kq_select_variant", "kq_gemm_mxf4", "kq_select_gemm_kernel", "kq_adaln_quantize",
)


class KQError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed: {message}")
        self.status = status
        self.status_name = STATUS.get(status, str(status))


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libkq.so (built by mxfp4_activations_b200.build); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libkq.so not found at {path}: build it with `python -m mxfp4_activations_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(path)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "kq_expand_blocks": [P, I64, I, I, P, P],
        "kq_expand_factored": [P, I64, P, P],
        "kq_quantize": [P, I64, I64, I64, P, I, P, P, P, I, I, P],
        "kq_expand_blocks_n": [P, I64, I, I, I, P, P],
        "kq_expand_factored_n": [P, I64, I, P, P],
        "kq_quantize_n": [P, I64, I64, I64, I, P, I, P, P, P, I, I, P],
        "kq_dequantize": [P, P, I64, I64, P, I, P, I, P],
        "kq_ref_smooth_quantize": [P, I64, I64, I64, P, P, P, P],
        "kq_ref_fwht_quantize": [P, I64, I64, I64, P, P, P],
        "kq_e2m1_pack": [P, I64, P, P],
        "kq_get_device_error": [I],
        "kq_status_string": [I],
        "kq_abi_version": [],
        "kq_last_error": [],
        "kq_select_variant": [I64, I64, I, I, I, P],
        "kq_gemm_mxf4": [P, P, I64, P, P, I64, I64, P, I64, I, P],
        "kq_select_gemm_kernel": [I64, I64, I64, P],
        "kq_adaln_quantize": [P, I64, I64, I64, P, P, I64, ctypes.c_float, P, P, P, P, I, P, P],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = I
    L.kq_status_string.restype = ctypes.c_char_p
    L.kq_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(fn: str, status: int):
    if status != 0:
        msg = load().kq_status_string(status).decode()
        if status == 6:
            msg += f" ({load().kq_last_error().decode()})"
        raise KQError(fn, status, msg)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


_BF16_LIKE = (torch.bfloat16, torch.int16, torch.uint16)
_MAT_DTYPES = (torch.float32,) + _BF16_LIKE


def _cuda(t, name: str, device: torch.device | None = None, dtypes=None, contiguous: bool = False,
          min_numel: int | None = None) -> torch.Tensor:
    """Checks that t is a CUDA tensor (on `device`, when given) of one of `dtypes`,
    contiguous when required and holding at least `min_numel` elements, so that no
    host pointer, foreign-device pointer or short buffer reaches a kernel."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the input on {device}")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {[str(d) for d in dtypes]}, not {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {min_numel} are needed")
    return t


def _mat_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KQ_F32
    if t.dtype in _BF16_LIKE:
        return KQ_BF16
    raise TypeError("matrices must be float32 or bfloat16")


def _rows(x, name: str = "x"):
    """(M, d, ldx) of a 2-D bf16 CUDA activation whose rows may be strided."""
    _cuda(x, name, dtypes=_BF16_LIKE)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit column stride")
    return x.shape[0], x.shape[1], x.stride(0)


def _mats(mats, d: int, device: torch.device, name: str = "mats") -> int:
    """Block size n of a contiguous [d/n, n, n] matrix tensor on `device`."""
    _cuda(mats, name, device, _MAT_DTYPES, contiguous=True)
    if mats.dim() != 3 or mats.shape[1] != mats.shape[2]:
        raise ValueError(f"{name} must be [d/n, n, n]")
    n = mats.shape[-1]
    if n not in (16, 32, 64, 128):
        raise ValueError("transform blocks of 16, 32, 64 or 128 elements")
    if mats.shape[0] * n != d:
        raise ValueError(f"{name} holds {mats.shape[0]} blocks of {n}, the input has d = {d}")
    return n


# ---------------------------------------------------------------- set-up

def _params_shape(params: torch.Tensor, log2n: int | None):
    """(transform blocks nt, log2n) of a params tensor [nt, log2n, 3] (a flat
    tensor is read as 5 factors per block)."""
    if log2n is None:
        log2n = params.shape[-2] if params.dim() >= 2 else 5
    per = 3 * log2n
    if params.dtype != torch.float32 or params.numel() % per != 0:
        raise ValueError(f"params must be float32 [nt, {log2n}, 3]")
    return params.numel() // per, log2n


def kq_expand_blocks(params: torch.Tensor, inverse: bool = False, dtype: torch.dtype = torch.float32,
                     out: torch.Tensor | None = None, transpose: bool = False,
                     log2n: int | None = None) -> torch.Tensor:
    """K, K^-1 (inverse=True) or the weight-side K^-T (inverse=True, transpose=True)
    per transform block of n = 2^log2n elements ([nt, n, n]; log2n from params [nt, log2n, 3])."""
    _cuda(params, "params", dtypes=(torch.float32,))
    params = params.contiguous()
    nt, log2n = _params_shape(params, log2n)
    n = 1 << log2n
    if out is None:
        out = torch.empty((nt, n, n), dtype=dtype, device=params.device)
    _cuda(out, "out", params.device, _MAT_DTYPES, contiguous=True, min_numel=nt * n * n)
    if transpose and not inverse:
        raise ValueError("transpose is provided for the inverse (the weight-side transform) only")
    mode = 2 if transpose else int(bool(inverse))
    with torch.cuda.device(params.device):
        _check("kq_expand_blocks_n", load().kq_expand_blocks_n(_ptr(params), nt, log2n, mode, _mat_dtype(out),
                                                                 _ptr(out), _stream(params.device)))
    return out


def factored_floats(log2n: int) -> int:
    """Floats per butterfly record of one 32-element block column."""
    return 64 if log2n == 4 else 48


def kq_expand_factored(params: torch.Tensor, out: torch.Tensor | None = None,
                       log2n: int | None = None) -> torch.Tensor:
    """The butterfly form, one record per 32-element block column ([48] floats;
    [64] for 16-element transform blocks, two per column)."""
    _cuda(params, "params", dtypes=(torch.float32,))
    params = params.contiguous()
    nt, log2n = _params_shape(params, log2n)
    if log2n < 4 or log2n > 7:
        raise ValueError("the butterfly form covers transform blocks of 16 to 128 elements")
    nb32 = nt << (log2n - 5) if log2n >= 5 else nt // 2
    rec = factored_floats(log2n)
    if out is None:
        out = torch.empty((nb32, rec), dtype=torch.float32, device=params.device)
    _cuda(out, "out", params.device, (torch.float32,), contiguous=True, min_numel=nb32 * rec)
    with torch.cuda.device(params.device):
        _check("kq_expand_factored_n", load().kq_expand_factored_n(_ptr(params), nt, log2n, _ptr(out),
                                                                     _stream(params.device)))
    return out


# ---------------------------------------------------------------- hot path

def _outputs(x: torch.Tensor, M: int, d: int, q, scales, layout: str = "row"):
    if layout not in SCALE_LAYOUTS:
        raise ValueError(f"scale_layout must be one of {list(SCALE_LAYOUTS)}")
    if q is None:
        q = torch.empty((M, d // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        if layout == "row":
            scales = torch.empty((M, d // 32), dtype=torch.uint8, device=x.device)
        else:  # padding bytes are not written: start from zeros
            scales = torch.zeros(scale_bytes(M, d, layout), dtype=torch.uint8, device=x.device)
    _cuda(q, "q", x.device, (torch.uint8,), contiguous=True, min_numel=M * (d // 2))
    _cuda(scales, "scales", x.device, (torch.uint8,), contiguous=True, min_numel=scale_bytes(M, d, layout))
    return q, scales


def kq_quantize(x: torch.Tensor, mats: torch.Tensor, factored: torch.Tensor | None = None, variant: str = "auto",
                q: torch.Tensor | None = None, scales: torch.Tensor | None = None, scale_layout: str = "row"):
    """MXFP4 of x K per transform block -> (codes uint8 [M, d/2], E8M0 scales: uint8
    [M, d/32] for scale_layout="row", or the flat 128x4-tiled buffer for "mma").
    The transform block size comes from mats ([d/n, n, n], n = 32 or 64)."""
    M, d, ldx = _rows(x)
    n = _mats(mats, d, x.device)
    if factored is not None:
        _cuda(factored, "factored", x.device, (torch.float32,), contiguous=True,
              min_numel=(d // 32) * factored_floats(n.bit_length() - 1))
    if variant not in VARIANTS:
        raise ValueError(f"variant must be one of {list(VARIANTS)}")
    q, scales = _outputs(x, M, d, q, scales, scale_layout)
    with torch.cuda.device(x.device):
        _check("kq_quantize_n", load().kq_quantize_n(_ptr(x), M, d, ldx, n.bit_length() - 1, _ptr(mats),
                                                     _mat_dtype(mats), _ptr(factored), _ptr(q), _ptr(scales),
                                                     VARIANTS[variant], SCALE_LAYOUTS[scale_layout],
                                                     _stream(x.device)))
    return q, scales


def kq_adaln_quantize(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor, rows_per_group: int,
                      mats: torch.Tensor, factored: torch.Tensor, eps: float = 1e-6, q: torch.Tensor | None = None,
                      scales: torch.Tensor | None = None, scale_layout: str = "row", stats: torch.Tensor | None = None):
    """The quantizer fused with the AdaLN-modulated LayerNorm in front of it:
    h = bf16(LN(x) (1 + scale[g]) + shift[g]) with g = row // rows_per_group, then MXFP4
    of h K per 32-element block (butterfly variant) -> (codes, scales, stats), stats the
    fp32 (mean, 1/sqrt(var + eps)) of each row when a [M, 2] float32 tensor is given."""
    M, d, ldx = _rows(x)
    G = -(-M // max(1, int(rows_per_group)))
    for name, t in (("shift", shift), ("scale", scale)):
        _cuda(t, name, x.device, _BF16_LIKE, contiguous=True)
        if t.dim() != 2 or t.shape[1] != d or t.shape[0] < G:
            raise ValueError(f"{name} must be [ceil(M / rows_per_group), d] = [{G}, {d}]")
    n = _mats(mats, d, x.device)
    if n != 32 or mats.dtype != torch.float32:
        raise ValueError("the fused AdaLN quantizer takes fp32 matrices of 32-element blocks")
    _cuda(factored, "factored", x.device, (torch.float32,), contiguous=True, min_numel=(d // 32) * factored_floats(5))
    q, scales = _outputs(x, M, d, q, scales, scale_layout)
    if stats is not None:
        _cuda(stats, "stats", x.device, (torch.float32,), contiguous=True, min_numel=2 * M)
    with torch.cuda.device(x.device):
        _check("kq_adaln_quantize", load().kq_adaln_quantize(_ptr(x), M, d, ldx, _ptr(shift), _ptr(scale),
                                                             int(rows_per_group), float(eps), _ptr(mats),
                                                             _ptr(factored), _ptr(q), _ptr(scales),
                                                             SCALE_LAYOUTS[scale_layout], _ptr(stats),
                                                             _stream(x.device)))
    return q, scales, stats


def kq_dequantize(q: torch.Tensor, scales: torch.Tensor, inv_mats: torch.Tensor | None = None,
                  out_dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None) -> torch.Tensor:
    """E2M1 value x 2^(scale - 127) per element, then (with inv_mats [d/32, 32, 32])
    the inverse block transform.  Takes row-major scales [M, d/32] only."""
    _cuda(q, "q", dtypes=(torch.uint8,), contiguous=True)
    if q.dim() != 2:
        raise ValueError("q must be [M, d/2]")
    M, d = q.shape[0], q.shape[1] * 2
    _cuda(scales, "scales", q.device, (torch.uint8,), contiguous=True)
    if scales.dim() != 2 or tuple(scales.shape) != (M, d // 32):
        raise ValueError(f"scales must be row-major [M, d/32] = [{M}, {d // 32}] (the 128x4-tiled layout is "
                         "for block-scaled GEMMs and is not read here)")
    if inv_mats is not None:
        n = _mats(inv_mats, d, q.device, "inv_mats")
        if n != 32:
            raise ValueError("kq_dequantize undoes transforms of 32-element blocks only")
    if out is None:
        out = torch.empty((M, d), dtype=out_dtype, device=q.device)
    _cuda(out, "out", q.device, (torch.float32,) + _BF16_LIKE, contiguous=True, min_numel=M * d)
    mdt = _mat_dtype(inv_mats) if inv_mats is not None else KQ_F32
    with torch.cuda.device(q.device):
        _check("kq_dequantize", load().kq_dequantize(_ptr(q), _ptr(scales), M, d, _ptr(inv_mats), mdt, _ptr(out),
                                                     _mat_dtype(out), _stream(q.device)))
    return out


def kq_gemm_mxf4(a_q: torch.Tensor, a_scales: torch.Tensor, b_q: torch.Tensor, b_scales: torch.Tensor,
                 out_dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] = A . B^T on the tensor cores from two MXFP4 operands as kq_quantize
    writes them with scale_layout="mma": codes [M, K/2] and [N, K/2], tiled scales."""
    _cuda(a_q, "a_q", dtypes=(torch.uint8,), contiguous=True)
    _cuda(b_q, "b_q", a_q.device, (torch.uint8,), contiguous=True)
    if a_q.dim() != 2 or b_q.dim() != 2 or a_q.shape[1] != b_q.shape[1]:
        raise ValueError("a_q and b_q must be [M, K/2] and [N, K/2] with the same K")
    M, N, K = a_q.shape[0], b_q.shape[0], a_q.shape[1] * 2
    _cuda(a_scales, "a_scales", a_q.device, (torch.uint8,), contiguous=True, min_numel=scale_bytes(M, K, "mma"))
    _cuda(b_scales, "b_scales", a_q.device, (torch.uint8,), contiguous=True, min_numel=scale_bytes(N, K, "mma"))
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a_q.device)
    _cuda(out, "out", a_q.device, (torch.float32,) + _BF16_LIKE, contiguous=True, min_numel=M * N)
    with torch.cuda.device(a_q.device):
        _check("kq_gemm_mxf4", load().kq_gemm_mxf4(_ptr(a_q), _ptr(a_scales), M, _ptr(b_q), _ptr(b_scales), N, K,
                                                   _ptr(out), N, _mat_dtype(out), _stream(a_q.device)))
    return out


def kq_gemm_kernel(M: int, N: int, K: int) -> str:
    """"2sm" or "1sm": the kernel kq_gemm_mxf4 runs for this shape on the current device."""
    v = ctypes.c_int(0)
    _check("kq_select_gemm_kernel", load().kq_select_gemm_kernel(M, N, K, ctypes.byref(v)))
    return "2sm" if v.value else "1sm"


def kq_ref_smooth_quantize(x: torch.Tensor, inv_s: torch.Tensor, q=None, scales=None):
    M, d, ldx = _rows(x)
    _cuda(inv_s, "inv_s", x.device, (torch.float32,), contiguous=True, min_numel=d)
    q, scales = _outputs(x, M, d, q, scales)
    with torch.cuda.device(x.device):
        _check("kq_ref_smooth_quantize", load().kq_ref_smooth_quantize(_ptr(x), M, d, ldx, _ptr(inv_s), _ptr(q),
                                                                       _ptr(scales), _stream(x.device)))
    return q, scales


def kq_ref_fwht_quantize(x: torch.Tensor, q=None, scales=None):
    M, d, ldx = _rows(x)
    q, scales = _outputs(x, M, d, q, scales)
    with torch.cuda.device(x.device):
        _check("kq_ref_fwht_quantize", load().kq_ref_fwht_quantize(_ptr(x), M, d, ldx, _ptr(q), _ptr(scales),
                                                                   _stream(x.device)))
    return q, scales


def kq_e2m1_pack(v: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    _cuda(v, "v", dtypes=(torch.float32,))
    v = v.contiguous()
    if out is None:
        out = torch.empty(v.numel() // 2, dtype=torch.uint8, device=v.device)
    _cuda(out, "out", v.device, (torch.uint8,), contiguous=True, min_numel=v.numel() // 2)
    with torch.cuda.device(v.device):
        _check("kq_e2m1_pack", load().kq_e2m1_pack(_ptr(v), v.numel(), _ptr(out), _stream(v.device)))
    return out


def kq_select_variant(M: int, d: int, mat_dtype=None, has_factored: bool = True, log2n: int = 5) -> str:
    """The variant ("mma" or "butterfly") that variant="auto" runs for these sizes."""
    mdt = KQ_BF16 if mat_dtype in _BF16_LIKE else KQ_F32
    out = ctypes.c_int(-1)
    _check("kq_select_variant", load().kq_select_variant(M, d, log2n, mdt, int(bool(has_factored)),
                                                         ctypes.byref(out)))
    return {v: k for k, v in VARIANTS.items()}[out.value]


def kq_get_device_error(clear: bool = True) -> int:
    """Synchronises the current device; returns the kq_status of recorded device flags."""
    return int(load().kq_get_device_error(int(bool(clear))))


def kq_status_string(status: int) -> str:
    return load().kq_status_string(int(status)).decode()


def kq_abi_version() -> int:
    return int(load().kq_abi_version())
