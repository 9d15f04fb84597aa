"""The certified fast path's error bound, checked on the CPU.

The quantizer kernels take a scale or a code from their fp32 butterfly result
y_f only when the whole interval y_f +- E maps to it, with

    E = C * ||x||_1 * max|K|        (C = 14u (1 + 2^-16) for 32-element blocks, 32u for 64,
                                     8u for the FWHT comparison kernel)

("KroQuant: Kronecker-Structured Block Transforms ...", Approach: K is the
Kronecker product of 2x2 unit-determinant LU factors).  Exactness of the device
output rests on |y_f - y32| <= E, y32 being the definition's value.  These tests
run the butterfly's arithmetic in numpy (each factor F = M diag(a, d) with
M = [[1, b/d], [c/a, 1]], one fp32 fused multiply-add per element and stage,
then one fp32 multiply by D) and check the bound against the oracle's y32 on
outlier-heavy inputs, in the stage order the kernels use: for 32-element blocks
the factor on index bit 0 first and F0 last; for 64-element blocks the
half-mixing factor F0 first, then the in-half factors from bit 0 up.
"""
from __future__ import annotations

import numpy as np
import pytest

from mxfp4_activations_b200 import inputs

U = 2.0 ** -24


def fma32(a, b, c):
    """fp32 a*b + c with one rounding (the product is exact in fp64; the fp64 sum
    may add a rounding of 2^-53 relative, far below what is checked here)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def butterfly_coefficients(orc, params):
    """Per transform block: fp32 ratios (c/a, b/d) of every factor and the fp32
    diagonal D_j = prod_k (a_k or d_k, by bit k of j from the top)."""
    nt, nf = params.shape[0], params.shape[1]
    n = 1 << nf
    lam = np.zeros((nt, nf), np.float32)
    bet = np.zeros((nt, nf), np.float32)
    D = np.ones((nt, n), np.float64)
    j = np.arange(n)
    for t in range(nt):
        for k in range(nf):
            F = orc.factor(*params[t, k])
            lam[t, k] = np.float32(F[1, 0] / F[0, 0])
            bet[t, k] = np.float32(F[0, 1] / F[1, 1])
            bit = (j >> (nf - 1 - k)) & 1
            D[t] *= np.where(bit == 1, F[1, 1], F[0, 0])
    return lam, bet, D.astype(np.float32)


def stage(y, k, nf, lam, bet):
    """Factor k acts on index bit nf-1-k: out_lo = lo + lam hi, out_hi = hi + bet lo."""
    n = 1 << nf
    s = 1 << (nf - 1 - k)
    R, nt = y.shape[0], y.shape[1]
    v = y.reshape(R, nt, n // (2 * s), 2, s)
    lo, hi = v[:, :, :, 0, :], v[:, :, :, 1, :]
    L = lam[None, :, k, None, None]
    B = bet[None, :, k, None, None]
    out = np.empty_like(v)
    out[:, :, :, 0, :] = fma32(L, hi, lo)
    out[:, :, :, 1, :] = fma32(B, lo, hi)
    return out.reshape(R, nt, n)


def butterfly(x32, lam, bet, D, order):
    R, nt, n = x32.shape
    nf = n.bit_length() - 1
    y = x32.copy()
    for k in order:
        y = stage(y, k, nf, lam, bet)
    return (y.astype(np.float64) * D[None].astype(np.float64)).astype(np.float32)


def worst_error_in_u(orc, x_bits, params, order, y32):
    nt, nf = params.shape[0], params.shape[1]
    n = 1 << nf
    R = x_bits.shape[0]
    x32 = inputs.bf16_bits_to_f32(x_bits).reshape(R, nt, n)
    lam, bet, D = butterfly_coefficients(orc, params)
    yf = butterfly(x32, lam, bet, D, order).astype(np.float64)
    kmax = np.array([np.prod([np.abs(orc.factor(*params[t, k])).max() for k in range(nf)]) for t in range(nt)])
    l1 = np.abs(x32.astype(np.float64)).sum(-1)
    scale = (l1 * kmax[None, :])[..., None] * U
    err = np.abs(yf - y32.reshape(R, nt, n).astype(np.float64))
    ok = scale > 0
    return float((err[np.broadcast_to(ok, err.shape)] / np.broadcast_to(scale, err.shape)[np.broadcast_to(ok, err.shape)]).max())


def cases(n):
    out = []
    for name, d in (("flux", 3072), ("pixart", 1152)):
        x, _ = inputs.config_case(name, d, M=256)
        out.append(x)
    a = np.random.default_rng(5).standard_normal((128, 1152)).astype(np.float32)
    a *= np.float32(2.0) ** np.random.default_rng(6).integers(-20, 20, size=(128, 1152)).astype(np.float32)
    out.append(inputs.f32_to_bf16_bits(a))  # magnitudes spanning 2^40 inside a block
    return out


def test_bound_32_element_blocks(orc):
    for x in cases(32):
        d = x.shape[1]
        params = inputs.lu_params(d // 32, seed=[d, 7])
        y32 = orc.transform(x, orc.expand(params))
        w = worst_error_in_u(orc, x, params, order=[4, 3, 2, 1, 0], y32=y32)
        assert w <= 14.0, w   # the proven first-order need; the kernels allow 14u (1 + 2^-16)


def test_bound_64_element_blocks_half_mixing_first(orc):
    for x in cases(64):
        d = x.shape[1] - x.shape[1] % 64
        x = np.ascontiguousarray(x[:, :d])
        params = inputs.lu_params(d // 64, seed=[d, 8], factors=6)
        y32 = orc.transform_n(x, orc.expand_n(params))
        for order in ([0, 5, 4, 3, 2, 1], [5, 4, 3, 2, 1, 0]):
            w = worst_error_in_u(orc, x, params, order=order, y32=y32)
            assert w <= 16.0, (order, w)   # the proven need; the kernel allows 32u


def test_bound_fwht_comparison_kernel(orc):
    """The FWHT comparison kernel runs the same butterfly with every ratio +-1
    (exact add and subtract) and D_j = +-fp32(2^-2.5); its allowance is 8u
    against a proven need of 7u."""
    for x in cases(32):
        d = x.shape[1]
        R, nt = x.shape[0], d // 32
        x32 = inputs.bf16_bits_to_f32(x).reshape(R, nt, 32)
        lam = np.ones((nt, 5), np.float32)
        bet = -np.ones((nt, 5), np.float32)
        H = orc.hadamard(5)
        c = np.float32(2.0 ** -2.5)
        # the Sylvester H32 equals (M (x) ... (x) M) D with M = [[1, -1], [1, 1]] and D_j = c (-1)^popcount(j)
        D = np.array([c if bin(j).count("1") % 2 == 0 else -c for j in range(32)], np.float32)
        yf = butterfly(x32, lam, bet, np.tile(D, (nt, 1)), order=[4, 3, 2, 1, 0]).astype(np.float64)
        H32 = H.astype(np.float32)
        y32 = orc.transform(x, np.ascontiguousarray(np.tile(H32, (nt, 1, 1)))).reshape(R, nt, 32)
        l1 = np.abs(x32.astype(np.float64)).sum(-1, keepdims=True)
        kmax = float(np.abs(H32).max())
        ok = l1 > 0
        err = np.abs(yf - y32) / np.where(ok, l1 * kmax * U, 1.0)
        assert err[np.broadcast_to(ok, err.shape)].max() <= 7.0


@pytest.mark.parametrize("bad_constant", [0.25])
def test_bound_check_detects_a_wrong_bound(orc, bad_constant):
    """The check is not vacuous: the observed worst error exceeds a quarter of a
    unit roundoff times ||x||_1 max|K| on these inputs."""
    x = cases(32)[0]
    d = x.shape[1]
    params = inputs.lu_params(d // 32, seed=[d, 7])
    y32 = orc.transform(x, orc.expand(params))
    assert worst_error_in_u(orc, x, params, order=[4, 3, 2, 1, 0], y32=y32) > bad_constant


def test_exact_path_rate_estimate_orders_the_allowances(orc):
    """The host estimate of the exact-path share (tests/exact_path_rate.py) on 256 rows
    of the FLUX d=3072 input: wider allowances send more blocks to the exact path, the
    derived tensor-core allowances stay below a few per cent, and the butterfly's
    stays near the 0.15 % measured on the device."""
    from . import exact_path_rate as epr

    x, params = inputs.config_case("flux", 3072)
    x = x[:256]
    k32 = orc.expand(params, dtype=orc.F32)
    k16 = orc.expand(params, dtype=orc.BF16)
    r = {name: epr.rate(orc, x, k16 if dt == "bf16" else k32, c, e1, ek, e0)
         for name, (dt, c, e1, ek, e0) in epr.ALLOWANCES.items()}
    assert r["tensor_core_bf16_K_calibrated_16u"] <= r["tensor_core_bf16_K"] < 0.02
    assert r["tensor_core_fp32_K_calibrated_32u"] <= r["tensor_core_fp32_K"] < 0.05
    assert 0.0005 < r["butterfly"] < 0.005
