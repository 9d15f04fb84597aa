"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Integer outputs (codes, scales, expanded bf16/fp32 matrix
bits) are compared exactly; the tolerance of the quantizer's stated criterion is
checked by tests/parity.py and, because the kernels certify every scale and
code, the tests also require exact equality."""
from __future__ import annotations

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from mxfp4_activations_b200 import inputs  # noqa: E402

from .parity import compare, guarded, guards_intact, oracle_rows, tiled_scales, unpack  # noqa: E402

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


def dev_bf16(x_bits: np.ndarray) -> "torch.Tensor":
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_f32(a: np.ndarray) -> "torch.Tensor":
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host(t: "torch.Tensor") -> np.ndarray:
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


# (variant, matrix dtype): the butterfly serves fp32 matrices; the tensor-core
# variant serves fp32 (three exact bf16 parts) and bf16 matrices.
VARIANTS = [("butterfly", "f32"), ("mma", "f32"), ("mma", "bf16")]


def guarded_outputs(M: int, d: int, layout: str = "row"):
    """q [M, d/2] and scales inside canary bytes (see tests/parity.py), plus the
    backing buffers to check afterwards."""
    from mxfp4_activations_b200 import scale_bytes

    qv, qbuf = guarded(torch, M * (d // 2))
    sv, sbuf = guarded(torch, scale_bytes(M, d, layout))
    if layout == "mma":
        sv.zero_()  # padding bytes of the tiled layout are not written
    return qv.view(M, d // 2), (sv.view(M, d // 32) if layout == "row" else sv), (qbuf, sbuf)


def assert_guards(bufs):
    for b in bufs:
        assert guards_intact(torch, b), "a kernel wrote outside its output buffer"


def gpu_quantize(kq, x_bits, params, x_dev=None, variant="butterfly", mdt="f32"):
    p = dev_f32(params)
    mats = kq.kq_expand_blocks(p, dtype=torch.float32 if mdt == "f32" else torch.bfloat16)
    fac = kq.kq_expand_factored(p) if variant == "butterfly" else None
    x = dev_bf16(x_bits) if x_dev is None else x_dev
    M, d = x.shape
    q, s, bufs = guarded_outputs(M, d)
    kq.kq_quantize(x, mats, fac, variant=variant, q=q, scales=s)
    torch.cuda.synchronize()
    assert_guards(bufs)
    return host(q), host(s)


def oracle_mats(orc, params, mdt):
    return orc.expand(params, dtype=orc.F32 if mdt == "f32" else orc.BF16)


def check(q, s, qr, sr, yr=None, exact=True):
    rep = compare(q, s, qr, sr, yr)
    assert rep["ok"], rep
    if exact:
        assert rep["scale_mismatch"] == 0 and rep["code_mismatch"] == 0, rep
    return rep


# ---------------------------------------------------------------- set-up kernels

def special_params():
    p = inputs.lu_params(40, seed=77, noise=0.5)
    p[0] = inputs.identity_params(1)[0]
    p[1] = inputs.hadamard_params(1)[0]
    p[2, :, 0] = -0.0          # signed-zero l
    p[3, :, 2] = -0.0          # signed-zero v
    p[4, :, 1] = 1e-3          # large 1/u
    p[5, :, 1] = 3e3
    p[6, 2] = (-1.0, 1.0, 1.0)  # d = l v + 1/u = 0: butterfly ratio undefined
    return p


@pytest.mark.parametrize("mode", ["K", "K^-1", "K^-T"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_expand_bit_exact(kq, orc, mode, dtype):
    params = special_params()
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    inverse, transpose = mode != "K", mode == "K^-T"
    got = host(kq.kq_expand_blocks(dev_f32(params), inverse=inverse, dtype=tdt, transpose=transpose))
    want = orc.expand(params, dtype=orc.F32 if dtype == "f32" else orc.BF16, inverse=inverse)
    if transpose:
        want = np.ascontiguousarray(np.swapaxes(want, 1, 2))
    if dtype == "f32":
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        assert np.array_equal(got, want)


def test_expand_factored_reproduces_matrix(kq, orc):
    params = special_params()
    fac = host(kq.kq_expand_factored(dev_f32(params))).astype(np.float64)
    K = orc.expand_f64(params)
    for b in range(params.shape[0]):
        lam, bet, D, kmax, flag = fac[b, :5], fac[b, 5:10], fac[b, 10:42], fac[b, 42], fac[b, 43]
        assert kmax >= np.abs(K[b]).max()
        if flag:
            continue
        Mk = np.ones((1, 1))
        for k in range(5):
            Mk = np.kron(Mk, np.array([[1.0, bet[k]], [lam[k], 1.0]]))
        Kf = Mk * D[None, :]
        assert np.all(np.abs(Kf - K[b]) <= 1e-6 * np.abs(K[b]) + 1e-30)
    assert fac[6, 43] == 1.0  # d = 0 factor is routed to the exact path


def test_singular_factor_sets_device_flag(kq):
    p = inputs.lu_params(2, seed=1)
    p[1, 3, 1] = 0.0
    kq.kq_expand_blocks(dev_f32(p))
    assert kq.kq_get_device_error(clear=True) == 4
    assert kq.kq_get_device_error(clear=True) == 0


# ---------------------------------------------------------------- element step

def test_e2m1_pack_core_binades_exhaustive(kq, orc):
    lo = int(np.float32(0.125).view(np.uint32))
    hi = int(np.float32(8.0).view(np.uint32))
    pos = np.arange(lo, hi, dtype=np.uint32)
    for bits in (pos, pos | np.uint32(0x80000000)):
        v = bits.view(np.float32)
        got = host(kq.kq_e2m1_pack(dev_f32(v)))
        want = orc.e2m1_pack(v)
        assert np.array_equal(got, want)


def test_e2m1_pack_random_and_specials(kq, orc):
    rng = np.random.default_rng(5)
    v = rng.integers(0, 2**32, 1 << 22, dtype=np.uint64).astype(np.uint32).view(np.float32)
    v = v[~np.isnan(v)]
    v = np.concatenate([v, np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 6.0, 7.0, 5.0, 0.25, 0.75],
                                    np.float32)])
    v = v[: (v.size // 2) * 2].astype(np.float32)
    for n in (v.size, 2, 6, 10, 18):  # also tails shorter than 8 values
        got = host(kq.kq_e2m1_pack(dev_f32(v[:n])))
        assert np.array_equal(got, orc.e2m1_pack(v[:n]))


# ---------------------------------------------------------------- quantizer vs oracle

@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_cfg0_full(kq, orc, variant, mdt):
    x, params = inputs.config_case("cfg0", 1152)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    K = oracle_mats(orc, params, mdt)
    qr, sr = orc.quantize(x, K)
    check(q, s, qr, sr, orc.transform(x, K))


@pytest.mark.parametrize("variant,mdt", VARIANTS)
@pytest.mark.parametrize("M,d", [(1, 32), (3, 96), (65, 1152), (7, 5600), (130, 2240), (33, 12288), (257, 3072),
                                 (300, 4608)])
def test_quantize_ragged_shapes(kq, orc, M, d, variant, mdt):
    x = inputs.activations(M, d, "t3", seed=[M, d], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    params = inputs.lu_params(d // 32, seed=[M, d, 9])
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    K = oracle_mats(orc, params, mdt)
    qr, sr = orc.quantize(x, K)
    check(q, s, qr, sr, orc.transform(x, K))


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_strided_rows(kq, orc, variant, mdt):
    M, d, ldx = 50, 2240, 2240 + 136
    full = inputs.activations(M, ldx, "normal", seed=3, outlier_frac=0.01, outlier_scale=(50.0, 50.0))
    params = inputs.lu_params(d // 32, seed=4)
    xd = dev_bf16(full)[:, :d]
    assert xd.stride(0) == ldx
    q, s = gpu_quantize(kq, None, params, x_dev=xd, variant=variant, mdt=mdt)
    qr, sr = orc.quantize(np.ascontiguousarray(full[:, :d]), oracle_mats(orc, params, mdt))
    check(q, s, qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_degenerate_blocks(kq, orc, variant, mdt):
    rng = np.random.default_rng(8)
    M, d = 24, 256
    a = rng.standard_normal((M, d)).astype(np.float32)
    a[0] = 0.0                                   # all-zero row
    a[1, 32:64] = 0.0                            # one all-zero block
    a[2, 64:96] = -0.0                           # negative zeros
    a[3, 5] = np.inf                             # non-finite inputs
    a[4, 40] = np.nan
    a[5, 100] = -np.inf
    a[6] *= 1e37                                 # near fp32 overflow after the transform
    a[7] *= 1e-39                                # bf16 subnormals
    a[8, 0:32] = 0.0
    a[8, 3] = 1e-40                              # a single tiny value in a zero block
    a[9, 0:32] = 3.0                             # constant block (exact cancellations)
    a[10] = 3.4e38                               # overflow of the fp32 transform
    x = inputs.f32_to_bf16_bits(a)
    params = inputs.lu_params(d // 32, seed=9)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    K = oracle_mats(orc, params, mdt)
    qr, sr = orc.quantize(x, K)
    check(q, s, qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
@pytest.mark.parametrize("M,d", [(1, 32), (130, 96), (257, 1152), (64, 12288)])
def test_quantize_tiled_scale_layout(kq, orc, M, d, variant, mdt):
    x = inputs.activations(M, d, "t3", seed=[M, d, 5], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    params = inputs.lu_params(d // 32, seed=[M, d, 6])
    p = dev_f32(params)
    mats = kq.kq_expand_blocks(p, dtype=torch.float32 if mdt == "f32" else torch.bfloat16)
    fac = kq.kq_expand_factored(p) if variant == "butterfly" else None
    qd, sd = kq.kq_quantize(dev_bf16(x), mats, fac, variant=variant, scale_layout="mma")
    assert sd.numel() == kq.scale_bytes(M, d, "mma")
    qr, sr = orc.quantize(x, oracle_mats(orc, params, mdt))
    assert np.array_equal(host(qd), qr)
    assert np.array_equal(host(sd), tiled_scales(sr))  # padding stays zero


def test_w4a4_gemm_through_block_scaled_mma(kq, orc):
    """End to end: activations quantized with K_b, weights with K_b^-T, both with
    scales in the tiled layout, multiplied by cuBLAS's block-scaled FP4 GEMM
    (through torch) -- the consumer the layout is for.  The product equals the
    oracle's dequantized operands multiplied in fp64 up to fp32 accumulation and
    the bf16 output rounding, and approximates x w^T (the transform cancels)."""
    F = pytest.importorskip("torch.nn.functional")
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("this torch has no block-scaled FP4 matmul")
    M, N, d = 256, 128, 512
    x = inputs.activations(M, d, "t3", seed=51, outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    rng = np.random.default_rng(52)
    w = inputs.f32_to_bf16_bits((rng.standard_normal((N, d)) * 0.05).astype(np.float32))
    params = inputs.lu_params(d // 32, seed=53)
    bt = kq.BlockTransform(dev_f32(params))
    qa, sa = bt.quantize(dev_bf16(x), scale_layout="mma")
    qb, sb = bt.quantize_weights(dev_bf16(w), scale_layout="mma")
    try:
        y = F.scaled_mm(qa.view(torch.float4_e2m1fn_x2), qb.view(torch.float4_e2m1fn_x2).t(),
                        sa.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        sb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)
    except (RuntimeError, NotImplementedError, TypeError, ValueError) as e:
        pytest.skip(f"block-scaled FP4 matmul unavailable here: {str(e).splitlines()[0][:120]}")
    y = y.float().cpu().numpy().astype(np.float64)
    ka = orc.expand(params, dtype=orc.F32)
    kbt = np.ascontiguousarray(np.swapaxes(orc.expand(params, dtype=orc.F32, inverse=True), 1, 2))
    qar, sar = orc.quantize(x, ka)
    qbr, sbr = orc.quantize(w, kbt)
    a_hat = orc.dequantize(qar, sar).astype(np.float64)
    b_hat = orc.dequantize(qbr, sbr).astype(np.float64)
    yref = a_hat @ b_hat.T
    mag = np.abs(a_hat) @ np.abs(b_hat).T
    assert np.all(np.abs(y - yref) <= 2.0**-8 * np.abs(yref) + 2.0**-16 * mag), np.abs(y - yref).max()
    xw = inputs.bf16_bits_to_f32(x).astype(np.float64) @ inputs.bf16_bits_to_f32(w).astype(np.float64).T
    rel = np.linalg.norm(yref - xw) / np.linalg.norm(xw)
    assert rel < 0.25, rel  # FP4 noise only: a wrong transform pair would not cancel


@pytest.mark.parametrize("mdt", ["f32", "bf16"])
def test_weight_side_quantize(kq, orc, mdt):
    """Weight rows quantized with the weight-side transform K_b^-T through the
    public BlockTransform API, against the oracle on the same matrices."""
    rng = np.random.default_rng(41)
    n_out, d = 96, 320
    w = inputs.f32_to_bf16_bits((rng.standard_normal((n_out, d)) * 0.02).astype(np.float32))
    params = inputs.lu_params(d // 32, seed=42)
    bt = kq.BlockTransform(dev_f32(params))
    qd, sd = bt.quantize_weights(dev_bf16(w), mat_dtype=torch.float32 if mdt == "f32" else torch.bfloat16)
    kit = np.ascontiguousarray(np.swapaxes(orc.expand(params, dtype=orc.F32 if mdt == "f32" else orc.BF16,
                                                      inverse=True), 1, 2))
    qr, sr = orc.quantize(w, kit)
    check(host(qd), host(sd), qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_singular_and_exact_only_columns(kq, orc, variant, mdt):
    """A factor with u = 0 puts inf and NaN into K, so even an all-zero block has
    y = 0 * inf = NaN by definition (scale byte 0xFF); a factor with d = 0 keeps K
    finite but has no butterfly form.  Both columns go through the exact path."""
    rng = np.random.default_rng(31)
    M, d = 40, 192
    a = rng.standard_normal((M, d)).astype(np.float32)
    a[0] = 0.0                    # an all-zero row crosses every column
    a[1, 32:64] = 0.0             # zero block in the singular column
    a[2, 64:96] = -0.0            # negative zeros in the d = 0 column
    a[3, 0:32] = 0.0              # zero block in an ordinary column
    x = inputs.f32_to_bf16_bits(a)
    params = inputs.lu_params(d // 32, seed=32)
    params[1, 2, 1] = 0.0         # u = 0: singular factor in block column 1
    params[2, 1] = (-1.0, 1.0, 1.0)  # d = l v + 1/u = 0 in block column 2
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    assert kq.kq_get_device_error(clear=True) == 4  # the set-up kernels flag the singular factor
    K = oracle_mats(orc, params, mdt)
    qr, sr = orc.quantize(x, K)
    check(q, s, qr, sr)
    assert np.all(s[:, 1] == 0xFF) and np.all(qr[:, 16:32] == 0)  # every block of the singular column is NaN


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_identity_all_bf16_patterns(kq, orc, variant, mdt):
    """K = I: every bf16 bit pattern (NaN/Inf included) goes through the scale and
    element steps as its own value; 2048 blocks of 32 consecutive patterns, plus a
    shuffled copy so that each block mixes magnitudes."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rng = np.random.default_rng(10)
    x = np.concatenate([pats, rng.permutation(pats)]).reshape(-1, 1024)
    params = inputs.identity_params(1024 // 32)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    qr, sr = orc.quantize(x, oracle_mats(orc, params, mdt))
    check(q, s, qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_exact_ties_identity(kq, orc, variant, mdt):
    """Blocks whose elements sit exactly on E2M1 midpoints (and one bf16 step
    away) under K = I, so the certified path must resolve every one of them."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    rows = []
    for e in (-3, 0, 5):
        blk = np.zeros(32, np.float32)
        blk[0] = 4.0 * 2.0 ** e  # fixes the scale to 2^e
        vals = np.concatenate([mids, -mids, mids * (1 + 2 ** -7), mids * (1 - 2 ** -8)])
        blk[1:1 + len(vals[:31])] = vals[:31] * 2.0 ** e
        rows.append(blk)
    x = inputs.f32_to_bf16_bits(np.stack(rows).reshape(1, -1))
    params = inputs.identity_params(x.shape[1] // 32)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    qr, sr = orc.quantize(x, oracle_mats(orc, params, mdt))
    check(q, s, qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
def test_quantize_hadamard_init_onehot(kq, orc, variant, mdt):
    x = np.zeros((32, 32), np.float32)
    for c in range(32):
        x[c, c] = 32.0
    xb = inputs.f32_to_bf16_bits(x)
    params = inputs.hadamard_params(1)
    q, s = gpu_quantize(kq, xb, params, variant=variant, mdt=mdt)
    qr, sr = orc.quantize(xb, oracle_mats(orc, params, mdt))
    check(q, s, qr, sr)
    assert np.all(s == 127) and np.all((unpack(q) & 7) == 7)


_CASE_CACHE = {}


def case_full(orc, key, make, mdt):
    """(x, params, oracle codes, oracle scales) of one input, every row; the oracle
    runs over the host cores.  Cached per input and matrix precision, so the
    variants that share a matrix share one oracle run (the variants are the
    fastest-varying parameter of the tests below)."""
    if key not in _CASE_CACHE:
        _CASE_CACHE.clear()
        _CASE_CACHE[key] = {"input": make()}
    entry = _CASE_CACHE[key]
    x, params = entry["input"]
    if mdt not in entry:
        entry[mdt] = oracle_rows("quantize", x, oracle_mats(orc, params, mdt))
    return (x, params) + entry[mdt]


@pytest.mark.parametrize("variant,mdt", VARIANTS)
@pytest.mark.parametrize("name,d", [("pixart", 1152), ("pixart", 4608), ("sana", 2240), ("sana", 5600),
                                    ("flux", 3072), ("flux", 12288)])
def test_quantize_full_config_every_row(kq, orc, name, d, variant, mdt):
    x, params, qr, sr = case_full(orc, (name, d), lambda: inputs.config_case(name, d), mdt)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    check(q, s, qr, sr)


@pytest.mark.parametrize("variant,mdt", VARIANTS)
@pytest.mark.parametrize("d", inputs.SWEEP_D)
@pytest.mark.parametrize("M", inputs.SWEEP_M)
def test_quantize_sweep_shapes_every_row(kq, orc, M, d, variant, mdt):
    x, params, qr, sr = case_full(orc, ("sweep", M, d), lambda: inputs.sweep_case(M, d), mdt)
    q, s = gpu_quantize(kq, x, params, variant=variant, mdt=mdt)
    check(q, s, qr, sr)


# ---------------------------------------------------------------- comparison kernels

@pytest.mark.parametrize("M,d", [(64, 1152), (7, 5600), (1, 32), (300, 3072)])
def test_smooth_parity(kq, orc, M, d):
    x = inputs.activations(M, d, "t4", seed=[M, d, 2], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    inv_s = inputs.smooth_inv_scale(x)
    qd, sd, bufs = guarded_outputs(M, d)
    kq.kq_ref_smooth_quantize(dev_bf16(x), dev_f32(inv_s), q=qd, scales=sd)
    qr, sr = orc.smooth_quantize(x, inv_s)
    check(host(qd), host(sd), qr, sr)
    assert_guards(bufs)


@pytest.mark.parametrize("M,d", [(64, 1152), (7, 5600), (1, 32), (300, 3072)])
def test_fwht_parity(kq, orc, M, d):
    x = inputs.activations(M, d, "t3", seed=[M, d, 3], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    qd, sd, bufs = guarded_outputs(M, d)
    kq.kq_ref_fwht_quantize(dev_bf16(x), q=qd, scales=sd)
    qr, sr = orc.fwht_quantize(x)
    check(host(qd), host(sd), qr, sr)
    assert_guards(bufs)


def test_fwht_degenerate_blocks(kq, orc):
    a = np.random.default_rng(12).standard_normal((6, 96)).astype(np.float32)
    a[0] = 0.0
    a[1, :32] = 1.0    # exact cancellations: every output but one is zero
    a[2, 3] = np.nan
    a[3] *= 3e37
    x = inputs.f32_to_bf16_bits(a)
    qd, sd = kq.kq_ref_fwht_quantize(dev_bf16(x))
    qr, sr = orc.fwht_quantize(x)
    check(host(qd), host(sd), qr, sr)


# ---------------------------------------------------------------- dequantize

def test_dequantize_exact_without_transform(kq, orc):
    x, params = inputs.config_case("cfg0", 1152)
    p = dev_f32(params)
    qd, sd = kq.kq_quantize(dev_bf16(x), kq.kq_expand_blocks(p), kq.kq_expand_factored(p))
    got = host(kq.kq_dequantize(qd, sd))
    want = orc.dequantize(host(qd), host(sd)).astype(np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    gotb = host(kq.kq_dequantize(qd, sd, out_dtype=torch.bfloat16))
    assert np.array_equal(gotb, inputs.f32_to_bf16_bits(want))


def test_dequantize_inverse_within_fp32_bound(kq, orc):
    x, params = inputs.config_case("cfg0", 1152)
    p = dev_f32(params)
    qd, sd = kq.kq_quantize(dev_bf16(x), kq.kq_expand_blocks(p), kq.kq_expand_factored(p))
    inv = kq.kq_expand_blocks(p, inverse=True)
    got = host(kq.kq_dequantize(qd, sd, inv)).astype(np.float64)
    Ki = orc.expand(params, inverse=True)
    want = orc.dequantize(host(qd), host(sd), Ki)
    yh = orc.dequantize(host(qd), host(sd))
    M, d = want.shape
    bound = np.einsum("rbj,bji->rbi", np.abs(yh).reshape(M, d // 32, 32),
                      np.abs(Ki.astype(np.float64))).reshape(M, d) * 33 * 2.0 ** -24
    assert np.all(np.abs(got - want) <= bound + 1e-30)
    # and the round trip reconstructs x to MXFP4 accuracy (sanity, not parity)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64)
    rel = np.linalg.norm(got - xf) / np.linalg.norm(xf)
    assert rel < 0.2


def test_no_device_error_after_suite(kq):
    assert kq.kq_get_device_error(clear=True) == 0


# ---------------------------------------------------------------- 64-element transform blocks

@pytest.mark.parametrize("log2n", [4, 6, 7])
@pytest.mark.parametrize("mode", ["K", "K^-1", "K^-T"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_expand_n_bit_exact(kq, orc, log2n, mode, dtype):
    params = inputs.lu_params(5, seed=80 + log2n, noise=0.3, factors=log2n)
    params[1] = inputs.hadamard_params(1, factors=log2n)[0]
    inverse, transpose = mode != "K", mode == "K^-T"
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    got = host(kq.kq_expand_blocks(dev_f32(params), inverse=inverse, dtype=tdt, transpose=transpose))
    want = orc.expand_n(params, dtype=orc.F32 if dtype == "f32" else orc.BF16, inverse=inverse)
    if transpose:
        want = np.ascontiguousarray(np.swapaxes(want, 1, 2))
    if dtype == "f32":
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        assert np.array_equal(got, want)


def test_expand_factored_n64_reproduces_matrix(kq, orc):
    params = inputs.lu_params(6, seed=90, noise=0.3, factors=6)
    params[5, 3] = (-1.0, 1.0, 1.0)  # d = 0 in one factor: no butterfly form
    fac = host(kq.kq_expand_factored(dev_f32(params))).astype(np.float64)
    assert fac.shape == (12, 48)
    K = orc.expand_n_f64(params)
    for c in range(6):
        lo, hi = fac[2 * c], fac[2 * c + 1]
        assert lo[43] == hi[43] and lo[42] == hi[42] and lo[42] >= np.abs(K[c]).max()
        if lo[43]:
            continue
        assert np.array_equal(lo[:10], hi[:10]) and np.array_equal(lo[45:47], hi[45:47])
        Mk = np.array([[1.0, lo[46]], [lo[45], 1.0]])
        for k in range(5):
            Mk = np.kron(Mk, np.array([[1.0, lo[5 + k]], [lo[k], 1.0]]))
        Kf = Mk * np.concatenate([lo[10:42], hi[10:42]])[None, :]
        assert np.all(np.abs(Kf - K[c]) <= 1e-6 * np.abs(K[c]) + 1e-30)
    assert fac[10, 43] == 1.0 and fac[11, 43] == 1.0


def test_expand_factored_n16_reproduces_matrices(kq, orc):
    """16-element transform blocks: one [64] record per 32-element column holds the
    butterfly of both of its 16-element blocks."""
    params = inputs.lu_params(12, seed=91, noise=0.3, factors=4)
    params[9, 1] = (-1.0, 1.0, 1.0)  # d = 0 in one factor: no butterfly form for column 4
    fac = host(kq.kq_expand_factored(dev_f32(params))).astype(np.float64)
    assert fac.shape == (6, 64) and np.all(fac[:, 51:] == 0.0)
    K = orc.expand_n_f64(params)
    for c in range(6):
        r = fac[c]
        assert r[48] >= max(np.abs(K[2 * c]).max(), np.abs(K[2 * c + 1]).max())
        if r[49]:
            continue
        for h in range(2):
            Mk = np.ones((1, 1))
            for k in range(4):
                Mk = np.kron(Mk, np.array([[1.0, r[8 * h + 4 + k]], [r[8 * h + k], 1.0]]))
            Kf = Mk * r[16 + 16 * h:32 + 16 * h][None, :]
            assert np.all(np.abs(Kf - K[2 * c + h]) <= 1e-6 * np.abs(K[2 * c + h]) + 1e-30)
    assert fac[4, 49] == 1.0


def test_expand_factored_n128_reproduces_matrix(kq, orc):
    """128-element transform blocks: each of the four columns of a block carries the
    five inner factors, its 32 entries of D, and the coefficients of the two
    cross-column factors that its position uses."""
    params = inputs.lu_params(3, seed=92, noise=0.3, factors=7)
    fac = host(kq.kq_expand_factored(dev_f32(params))).astype(np.float64)
    assert fac.shape == (12, 48)
    K = orc.expand_n_f64(params)
    for t in range(3):
        rec = fac[4 * t:4 * t + 4]
        assert np.all(rec[:, 43] == 0.0) and np.all(rec[:, 42] >= np.abs(K[t]).max())
        assert all(np.array_equal(rec[0, :10], rec[q, :10]) for q in range(4))
        lam1, bet1 = rec[0, 45], rec[1, 45]   # factor 1 (index bit 5): lower / upper column
        lam0, bet0 = rec[0, 46], rec[2, 46]   # factor 0 (index bit 6): lower / upper 64-element half
        assert rec[2, 45] == lam1 and rec[3, 45] == bet1 and rec[1, 46] == lam0 and rec[3, 46] == bet0
        Mk = np.kron(np.array([[1.0, bet0], [lam0, 1.0]]), np.array([[1.0, bet1], [lam1, 1.0]]))
        for k in range(5):
            Mk = np.kron(Mk, np.array([[1.0, rec[0, 5 + k]], [rec[0, k], 1.0]]))
        Kf = Mk * np.concatenate([rec[q, 10:42] for q in range(4)])[None, :]
        assert np.all(np.abs(Kf - K[t]) <= 1e-6 * np.abs(K[t]) + 1e-30)


def gpu_quantize_n(kq, x_bits, params, x_dev=None, scale_layout="row"):
    p = dev_f32(params)
    mats = kq.kq_expand_blocks(p)
    fac = kq.kq_expand_factored(p)
    x = dev_bf16(x_bits) if x_dev is None else x_dev
    M, d = x.shape
    q, s, bufs = guarded_outputs(M, d, scale_layout)
    kq.kq_quantize(x, mats, fac, variant="butterfly", q=q, scales=s, scale_layout=scale_layout)
    torch.cuda.synchronize()
    assert_guards(bufs)
    return host(q), host(s)


# (log2 n, shapes): d a multiple of max(32, n)
N_SHAPES = {
    4: [(1, 32), (3, 96), (65, 1152), (130, 2240), (33, 12288), (257, 3072)],
    6: [(1, 64), (3, 128), (65, 1152), (130, 2240), (33, 12288), (257, 3072), (300, 4608)],
    7: [(1, 128), (3, 256), (65, 1152), (33, 12288), (257, 3072), (300, 4608)],
}


@pytest.mark.parametrize("log2n,M,d", [(k, M, d) for k, v in N_SHAPES.items() for M, d in v])
def test_quantize_n_ragged_shapes(kq, orc, log2n, M, d):
    x = inputs.activations(M, d, "t3", seed=[M, d, 64 + log2n], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    params = inputs.lu_params(d >> log2n, seed=[M, d, 65 + log2n], factors=log2n)
    q, s = gpu_quantize_n(kq, x, params)
    K = orc.expand_n(params)
    qr, sr = orc.quantize_n(x, K)
    check(q, s, qr, sr, orc.transform_n(x, K))


@pytest.mark.parametrize("log2n", [4, 6, 7])
def test_quantize_n_flux_shape(kq, orc, log2n):
    x, _ = inputs.config_case("flux", 3072)
    params = inputs.lu_params(3072 >> log2n, seed=66 + log2n, factors=log2n)
    q, s = gpu_quantize_n(kq, x, params)
    qr, sr = oracle_rows("quantize_n", x, orc.expand_n(params))
    check(q, s, qr, sr)


@pytest.mark.parametrize("log2n", [4, 6, 7])
def test_quantize_n_degenerate_and_singular(kq, orc, log2n):
    n = 1 << log2n
    rng = np.random.default_rng(67 + log2n)
    M, d = 24, 384
    a = rng.standard_normal((M, d)).astype(np.float32)
    a[0] = 0.0                       # all-zero row
    a[1, 128:256] = 0.0              # all-zero transform blocks
    a[2, 0:16] = 0.0                 # a zero part: its outputs still see the rest of the block
    a[3, 5] = np.inf
    a[4, 100] = np.nan
    a[6] *= 1e37
    a[7] *= 1e-39
    a[8, 33] = 3.4e38
    a[9, 128:256] = 3.0              # constant blocks (exact cancellations)
    x = inputs.f32_to_bf16_bits(a)
    params = inputs.lu_params(d // n, seed=68 + log2n, factors=log2n)
    params[1, log2n - 2, 1] = 0.0    # u = 0: singular factor in transform block 1
    params[2, 0] = (-1.0, 1.0, 1.0)  # d = 0 in the outermost factor of block 2
    q, s = gpu_quantize_n(kq, x, params)
    assert kq.kq_get_device_error(clear=True) == 4
    qr, sr = orc.quantize_n(x, orc.expand_n(params))
    check(q, s, qr, sr)


@pytest.mark.parametrize("log2n", [4, 6, 7])
def test_quantize_n_strided_rows_and_tiled_scales(kq, orc, log2n):
    M, d, ldx = 70, 1280, 1280 + 72
    full = inputs.activations(M, ldx, "normal", seed=69 + log2n, outlier_frac=0.01, outlier_scale=(50.0, 50.0))
    params = inputs.lu_params(d >> log2n, seed=70 + log2n, factors=log2n)
    xd = dev_bf16(full)[:, :d]
    qr, sr = orc.quantize_n(np.ascontiguousarray(full[:, :d]), orc.expand_n(params))
    q, s = gpu_quantize_n(kq, None, params, x_dev=xd)
    check(q, s, qr, sr)
    q, s = gpu_quantize_n(kq, None, params, x_dev=xd, scale_layout="mma")
    assert np.array_equal(q, qr) and np.array_equal(s, tiled_scales(sr))


def test_no_device_error_after_n_blocks(kq):
    assert kq.kq_get_device_error(clear=True) == 0


# ---------------------------------------------------------------- back-to-back launches

@pytest.mark.parametrize("kind", ["butterfly", "butterfly64", "mma_f32", "mma_bf16", "butterfly_tiled", "smooth",
                                  "fwht"])
def test_back_to_back_launches_every_output_exact(kq, orc, kind):
    """Launches queued back to back on one stream at the FLUX.1-schnell shape
    4608 x 12288 (each may start while the previous one drains): every launch's
    output must equal the oracle's, not only the last one.  Each launch of a round
    writes its own buffer; the buffers are compared on the device between rounds,
    and every other round starts after an L2-sized write."""
    d = 12288
    x, params = inputs.config_case("flux", d)
    xd = dev_bf16(x)
    layout = "mma" if kind == "butterfly_tiled" else "row"
    if kind == "smooth":
        inv_s = inputs.smooth_inv_scale(x)
        inv_s_d = dev_f32(inv_s)
        qr, sr = orc.smooth_quantize(x, inv_s)
        launch = lambda q, s: kq.kq_ref_smooth_quantize(xd, inv_s_d, q=q, scales=s)
    elif kind == "fwht":
        qr, sr = orc.fwht_quantize(x)
        launch = lambda q, s: kq.kq_ref_fwht_quantize(xd, q=q, scales=s)
    else:
        if kind == "butterfly64":
            params = inputs.lu_params(d // 64, seed=71, factors=6)
            qr, sr = orc.quantize_n(x, orc.expand_n(params))
        else:
            mdt = "bf16" if kind == "mma_bf16" else "f32"
            qr, sr = orc.quantize(x, oracle_mats(orc, params, mdt))
        p = dev_f32(params)
        mats = kq.kq_expand_blocks(p, dtype=torch.bfloat16 if kind == "mma_bf16" else torch.float32)
        variant = "mma" if kind.startswith("mma") else "butterfly"
        fac = kq.kq_expand_factored(p) if variant == "butterfly" else None
        launch = lambda q, s: kq.kq_quantize(xd, mats, fac, variant=variant, q=q, scales=s, scale_layout=layout)
    if layout == "mma":
        sr = tiled_scales(sr)
    qr_d, sr_d = torch.from_numpy(qr).cuda(), torch.from_numpy(sr).cuda()
    nbuf = 8
    qs = [torch.zeros_like(qr_d) for _ in range(nbuf)]
    ss = [torch.zeros_like(sr_d) for _ in range(nbuf)]
    flush = torch.empty(192 * 2**20, dtype=torch.uint8, device="cuda")
    bad = []
    for rnd in range(10):
        if rnd % 2:
            flush.fill_(rnd)
        for i in range(nbuf):
            launch(qs[i], ss[i])
        for i in range(nbuf):
            nq, ns = int((qs[i] != qr_d).sum()), int((ss[i] != sr_d).sum())
            if nq or ns:
                bad.append((rnd * nbuf + i, nq, ns))
    assert not bad, f"(launch, wrong code bytes, wrong scales): {bad}"
    assert kq.kq_get_device_error(clear=True) == 0
