"""W4A4 MXFP4 GEMM (kq_gemm_mxf4, tcgen05.mma kind::mxf4) against the oracle.

The oracle's product (oracle.mx_gemm, or the oracle's dequantized operands
multiplied in fp64 for the large sampled cases) is exact up to fp64 rounding.
The kernel adds each 64-element step's sum (two 32-element blocks, each an exact
sum of exact products) to an fp32 accumulator, so its error is bounded by
(K/32 + 1) * 2^-23 * sum_k |A(m,k) B(n,k)|, plus half an output ulp for bf16.
"""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from mxfp4_activations_b200 import inputs  # noqa: E402

from .parity import guarded, guards_intact, tiled_scales, untiled_scales  # noqa: E402

pytestmark = [
    pytest.mark.gpu,
    pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device"),
]


@pytest.fixture(scope="module")
def kq():
    from mxfp4_activations_b200 import build

    build.build()
    import mxfp4_activations_b200 as m

    m.load()
    assert m.kq_get_device_error(clear=True) == 0
    return m


def dev_u8(a: np.ndarray) -> "torch.Tensor":
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).cuda()


def host(t: "torch.Tensor") -> np.ndarray:
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return (t.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    return t.cpu().numpy()


def magnitudes(q: np.ndarray) -> np.ndarray:
    return np.asarray(q, np.uint8) & np.uint8(0x77)  # sign bits of both nibbles cleared


def bound(K: int, mag: np.ndarray, ref: np.ndarray, bf16: bool) -> np.ndarray:
    tol = (K / 32 + 1) * 2.0**-23 * mag
    if bf16:
        tol = tol + 2.0**-8 * np.abs(ref)
    return tol


def run_gemm(kq, aq, sa, bq, sb, out_dtype=torch.float32, pad=0xFF):
    """Device GEMM on operands given with row-major scales: the scales are tiled for
    the kernel with `pad` in the padding bytes (0xFF: NaN if ever read), and C sits
    inside canary bytes."""
    M, N = aq.shape[0], bq.shape[0]
    esz = 4 if out_dtype == torch.float32 else 2
    cv, cbuf = guarded(torch, M * N * esz)
    c = cv.view(out_dtype).view(M, N) if M * N else torch.empty((M, N), dtype=out_dtype, device="cuda")
    out = kq.kq_gemm_mxf4(dev_u8(aq), dev_u8(tiled_scales(sa, pad)), dev_u8(bq), dev_u8(tiled_scales(sb, pad)),
                          out=c)
    torch.cuda.synchronize()
    assert guards_intact(torch, cbuf), "the GEMM wrote outside C"
    assert kq.kq_get_device_error(clear=True) == 0
    return host(out).astype(np.float64)


SMALL = [(1, 1, 32), (1, 8, 64), (127, 129, 96), (130, 260, 160), (256, 128, 128), (300, 384, 1152),
         (129, 257, 4096), (64, 640, 224)]


@pytest.mark.parametrize("M,N,K", SMALL)
def test_gemm_random_operands_every_entry(kq, orc, M, N, K):
    assert kq.kq_gemm_kernel(M, N, K) == "1sm"
    """Every entry, shapes spanning several 128 x 128 tiles, ragged M and N, K ending
    inside a 128-element stage (tiled-scale padding filled with 0xFF), K longer than
    the stage ring."""
    aq, sa = inputs.mx_operand(M, K, seed=[M, N, K, 1])
    bq, sb = inputs.mx_operand(N, K, seed=[M, N, K, 2])
    c = run_gemm(kq, aq, sa, bq, sb)
    ref = orc.mx_gemm(aq, sa, bq, sb)
    mag = orc.mx_gemm(magnitudes(aq), sa, magnitudes(bq), sb)
    err = np.abs(c - ref)
    assert np.all(err <= bound(K, mag, ref, False)), (err.max(), np.unravel_index(err.argmax(), err.shape))


@pytest.mark.parametrize("M,N,K", [(130, 260, 160), (256, 384, 3072)])
def test_gemm_bf16_output(kq, orc, M, N, K):
    aq, sa = inputs.mx_operand(M, K, seed=[M, N, K, 3])
    bq, sb = inputs.mx_operand(N, K, seed=[M, N, K, 4])
    c = run_gemm(kq, aq, sa, bq, sb, out_dtype=torch.bfloat16)
    ref = orc.mx_gemm(aq, sa, bq, sb)
    mag = orc.mx_gemm(magnitudes(aq), sa, magnitudes(bq), sb)
    assert np.all(np.abs(c - ref) <= bound(K, mag, ref, True))


def test_gemm_wide_scale_range(kq, orc):
    """Scale bytes across a wide range (products from 2^-60 to 2^+60): fp32 normal
    results, each block weighted by its own power of two."""
    M, N, K = 192, 136, 512
    aq, sa = inputs.mx_operand(M, K, seed=5, scale_range=(97, 157))
    bq, sb = inputs.mx_operand(N, K, seed=6, scale_range=(97, 157))
    c = run_gemm(kq, aq, sa, bq, sb)
    ref = orc.mx_gemm(aq, sa, bq, sb)
    mag = orc.mx_gemm(magnitudes(aq), sa, magnitudes(bq), sb)
    assert np.all(np.abs(c - ref) <= bound(K, mag, ref, False))


def sample_rows(M: int) -> np.ndarray:
    rng = np.random.default_rng(M)
    fixed = [0, 1, 127, 128, 129, M // 2, M - 129, M - 128, M - 2, M - 1]
    return np.unique(np.concatenate([fixed, rng.choice(M, 14, replace=False)]))


def check_sampled(orc, c, aq, sa, bq, sb, bf16: bool):
    K = aq.shape[1] * 2
    rows = sample_rows(aq.shape[0])
    a_hat = orc.dequantize(aq[rows], sa[rows])
    b_hat = orc.dequantize(bq, sb)
    ref = a_hat @ b_hat.T
    mag = np.abs(a_hat) @ np.abs(b_hat).T
    err = np.abs(c[rows] - ref)
    assert np.all(err <= bound(K, mag, ref, bf16)), err.max()
    assert np.isfinite(c).all()


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("name", sorted(inputs.GEMM_SHAPES))
def test_gemm_flux_layer_shapes_sampled_rows(kq, orc, name, out):
    """The FLUX-shaped products at full size, in the launch configuration the bench
    times (the two-SM kernel); the oracle checks 24 sampled rows (tile edges
    included) against every column, from its dequantized operands multiplied in
    fp64."""
    M, N, K = inputs.GEMM_SHAPES[name]
    aq, sa = inputs.mx_operand(M, K, seed=[M, N, K, 7])
    bq, sb = inputs.mx_operand(N, K, seed=[M, N, K, 8])
    c = run_gemm(kq, aq, sa, bq, sb, out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    check_sampled(orc, c, aq, sa, bq, sb, out == "bf16")


# two-SM kernel (K % 128 == 0 and at least one 256 x 256 tile per SM pair): ragged M
# and N (a pair whose second CTA lies wholly past M), several tiles per cluster, and
# K % 256 == 128 (stages of 128 K-elements instead of 256)
PAIR = [(3900, 2000, 1024), (2304, 4352, 512), (4608, 9216, 3072), (2304, 4352, 640)]


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("M,N,K", PAIR)
def test_gemm_pair_kernel_ragged_and_persistent(kq, orc, M, N, K, out):
    assert kq.kq_gemm_kernel(M, N, K) == "2sm"
    aq, sa = inputs.mx_operand(M, K, seed=[M, N, K, 9])
    bq, sb = inputs.mx_operand(N, K, seed=[M, N, K, 10])
    c = run_gemm(kq, aq, sa, bq, sb, out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    check_sampled(orc, c, aq, sa, bq, sb, out == "bf16")
    cols = np.random.default_rng(M).choice(N, 16, replace=False)
    ref = orc.mx_gemm(aq, sa, bq[cols], sb[cols])  # every row against 16 columns
    mag = orc.mx_gemm(magnitudes(aq), sa, magnitudes(bq[cols]), sb[cols])
    assert np.all(np.abs(c[:, cols] - ref) <= bound(K, mag, ref, out == "bf16"))


def test_gemm_end_to_end_with_the_quantizer(kq, orc):
    """The consumer as a user runs it: FLUX-shaped activations (4608 x 3072) quantized
    with K_b and 3072 weight rows quantized with K_b^-T, both with tiled scales, then
    the product, all queued on one stream without a synchronisation.  Against the
    oracle's own quantization of the same inputs (codes compared first), dequantized
    and multiplied in fp64 on sampled rows; and close to x w^T, the transform
    cancelling."""
    from mxfp4_activations_b200 import BlockTransform

    x, params = inputs.config_case("flux", 3072)
    M, K = x.shape
    N = 3072
    rng = np.random.default_rng(91)
    w = inputs.f32_to_bf16_bits((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    bt = BlockTransform(torch.from_numpy(params).cuda())
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    wd = torch.from_numpy(w.view(np.int16)).cuda().view(torch.bfloat16)
    qa, sa = bt.quantize(xd, scale_layout="mma")
    qb, sb = bt.quantize_weights(wd, scale_layout="mma")
    c = kq.kq_gemm_mxf4(qa, sa, qb, sb)
    c = host(c).astype(np.float64)
    assert kq.kq_get_device_error(clear=True) == 0

    rows = sample_rows(M)
    ka = orc.expand(params, dtype=orc.F32)
    kbt = np.ascontiguousarray(np.swapaxes(orc.expand(params, dtype=orc.F32, inverse=True), 1, 2))
    qar, sar = orc.quantize(np.ascontiguousarray(x[rows]), ka)
    qbr, sbr = orc.quantize(w, kbt)
    assert np.array_equal(host(qa)[rows], qar) and np.array_equal(host(qb), qbr)
    assert np.array_equal(untiled_scales(host(sa), M, K // 32)[rows], sar)
    assert np.array_equal(untiled_scales(host(sb), N, K // 32), sbr)
    a_hat = orc.dequantize(qar, sar)
    b_hat = orc.dequantize(qbr, sbr)
    ref = a_hat @ b_hat.T
    mag = np.abs(a_hat) @ np.abs(b_hat).T
    assert np.all(np.abs(c[rows] - ref) <= bound(K, mag, ref, False))
    xw = inputs.bf16_bits_to_f32(x[rows]).astype(np.float64) @ inputs.bf16_bits_to_f32(w).astype(np.float64).T
    rel = np.linalg.norm(ref - xw) / np.linalg.norm(xw)
    assert rel < 0.25, rel


def test_gemm_nan_scale_reaches_its_row_and_column(kq, orc):
    """Scale byte 0xFF (a block that held a non-finite input) makes every product
    that reads it NaN, as in the oracle."""
    M, N, K = 160, 140, 256
    aq, sa = inputs.mx_operand(M, K, seed=11)
    bq, sb = inputs.mx_operand(N, K, seed=12)
    sa[3, 1] = 0xFF
    sb[133, 6] = 0xFF
    c = run_gemm(kq, aq, sa, bq, sb)
    ref = orc.mx_gemm(aq, sa, bq, sb)
    assert np.array_equal(np.isnan(c), np.isnan(ref))
    assert np.isnan(c[3]).all() and np.isnan(c[:, 133]).all()


def test_gemm_zero_operands_and_padding_never_read(kq, orc):
    """All-zero codes give exact zeros whatever the scales; padding bytes of the tiled
    scales (0xFF here) never reach a result."""
    M, N, K = 70, 90, 96
    aq = np.zeros((M, K // 2), np.uint8)
    bq, sb = inputs.mx_operand(N, K, seed=13)
    sa = np.full((M, K // 32), 200, np.uint8)
    c = run_gemm(kq, aq, sa, bq, sb)
    assert np.array_equal(c, np.zeros((M, N)))


def test_gemm_argument_errors(kq):
    a = torch.zeros((128, 16), dtype=torch.uint8, device="cuda")
    s = torch.zeros(kq.scale_bytes(128, 32, "mma"), dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        kq.kq_gemm_mxf4(a, s, torch.zeros((8, 32), dtype=torch.uint8, device="cuda"), s)  # K differs
    with pytest.raises(ValueError):
        kq.kq_gemm_mxf4(a, s[:100], a, s)  # short scale buffer
    with pytest.raises(ValueError):
        kq.kq_gemm_mxf4(a.cpu(), s, a, s)  # host codes
    empty = torch.zeros((0, 16), dtype=torch.uint8, device="cuda")
    assert kq.kq_gemm_mxf4(empty, s, a, s).shape == (0, 128)
    odd = torch.zeros((128, 8), dtype=torch.uint8, device="cuda")  # K = 16: not a multiple of 32
    with pytest.raises(kq.KQError):
        kq.kq_gemm_mxf4(odd, s, odd, s)
    assert kq.kq_get_device_error(clear=True) == 0


def test_gemm_matches_cublas_block_scaled_fp4(kq, orc):
    """Cross-check only: cuBLAS's block-scaled FP4 GEMM (through torch) on the same
    operands lands within both results' fp32 bounds of the exact product."""
    F = pytest.importorskip("torch.nn.functional")
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("this torch has no block-scaled FP4 matmul")
    M, N, K = 256, 384, 1024
    aq, sa = inputs.mx_operand(M, K, seed=21)
    bq, sb = inputs.mx_operand(N, K, seed=22)
    ours = run_gemm(kq, aq, sa, bq, sb, out_dtype=torch.bfloat16, pad=0)
    try:
        y = F.scaled_mm(dev_u8(aq).view(torch.float4_e2m1fn_x2), dev_u8(bq).view(torch.float4_e2m1fn_x2).t(),
                        dev_u8(tiled_scales(sa)).view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        dev_u8(tiled_scales(sb)).view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError, TypeError, ValueError) as e:
        pytest.skip(f"block-scaled FP4 matmul unavailable here: {str(e).splitlines()[0][:120]}")
    theirs = host(y).astype(np.float64)
    ref = orc.mx_gemm(aq, sa, bq, sb)
    mag = orc.mx_gemm(magnitudes(aq), sa, magnitudes(bq), sb)
    tol = bound(K, mag, ref, True)
    assert np.all(np.abs(ours - ref) <= tol)
    assert np.all(np.abs(theirs - ours) <= 2 * tol)
