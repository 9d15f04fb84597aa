"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against a closed form, a textbook
identity, a library routine used as a step, a brute force on small inputs, or a
value printed on the pages (tests/golden/).  A dropped term, a wrong sign, a
transposed operand or a swapped factor order in the oracle fails at least one.
"""
from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from mxfp4_activations_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---------------------------------------------------------------- helpers (independent formulations)

def brute_e2m1(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 magnitude by exhaustive distance search; on equal distance the
    code with mantissa bit 0 (even code) wins; magnitudes above the largest grid
    value saturate to it; sign bit from the sign of v."""
    v = np.asarray(v, np.float32)
    a = np.minimum(np.abs(v.astype(np.float64)), E2M1_MAGS[-1])
    best = np.full(a.shape, np.inf)
    code = np.zeros(a.shape, np.int64)
    for c, g in enumerate(E2M1_MAGS):
        dist = np.abs(a - g)
        take = (dist < best) | ((dist == best) & (c % 2 == 0))
        best = np.where(take, dist, best)
        code = np.where(take, c, code)
    return code | (np.signbit(v).astype(np.int64) << 3)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, np.uint8).reshape(-1)
    out = np.empty(packed.size * 2, np.int64)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out


def f32_exponent_field(a: np.ndarray) -> np.ndarray:
    return ((np.asarray(a, np.float32).view(np.uint32) >> 23) & 0xFF).astype(np.int64)


def e8m0_from_bits(amax: np.ndarray) -> np.ndarray:
    """floor(log2 amax) from the fp32 bit fields: normal -> field - 127,
    subnormal -> index of the top set mantissa bit - 149; then e = that - 2,
    clamped to [-127, 127], byte = e + 127; amax = 0 -> 0."""
    a = np.asarray(amax, np.float32)
    bits = a.view(np.uint32).astype(np.int64)
    field = (bits >> 23) & 0xFF
    mant = bits & 0x7FFFFF
    top = np.zeros_like(mant)
    for k in range(23):
        top = np.where((mant >> k) & 1 == 1, k, top)
    flog = np.where(field > 0, field - 127, top - 149)
    e = np.clip(flog - 2, -127, 127)
    byte = e + 127
    return np.where(a == 0, 0, byte)


def lu_numpy(l, u, v):
    L = np.array([[1.0, 0.0], [float(l), 1.0]])
    U = np.array([[float(u), float(v)], [0.0, 1.0 / float(u)]])
    return L @ U


def f32_round_fraction(q: Fraction) -> np.float32:
    """Correct rounding of an exact rational to fp32 (nearest, ties to even),
    by bracketing between adjacent fp32 values."""
    if q == 0:
        return np.float32(0.0)
    f = np.float32(float(q))  # within one ulp
    lo = f if Fraction(float(f)) <= q else np.nextafter(f, np.float32(-np.inf))
    hi = np.nextafter(lo, np.float32(np.inf))
    dlo, dhi = q - Fraction(float(lo)), Fraction(float(hi)) - q
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if (lo.view(np.uint32) & 1) == 0 else hi


def bf16_bits_to_frac(h: int) -> Fraction:
    return Fraction(float(np.array([h << 16], np.uint32).view(np.float32)[0]))


# ---------------------------------------------------------------- E2M1 element rounding (C5)

def test_e2m1_golden_grid(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_grid.txt")) if l.strip() and not l.startswith("#")]
    for r in rows:
        if r[0] == "tie":
            v, code = float(r[1]), int(r[2])
            assert orc.e2m1(v) == code, r
            assert orc.e2m1(-v) == code | 8, r
        else:
            code, val = int(r[0]), float(r[1])
            assert orc.e2m1_value(code) == val and math.copysign(1, orc.e2m1_value(code)) == math.copysign(1, val)
            assert orc.e2m1(val) == code  # every representable value maps to itself (incl. -0 -> 8)


def test_e2m1_exhaustive_core_binades(orc):
    """Every fp32 pattern with |v| in [2^-3, 2^3) (all midpoints, neighbours of
    midpoints and saturation region), both signs, against the brute force."""
    lo = np.float32(0.125).view(np.uint32)
    hi = np.float32(8.0).view(np.uint32)
    step = 1 << 23
    for start in range(int(lo), int(hi), step):
        pos = np.arange(start, min(start + step, int(hi)), dtype=np.uint32)
        for bits in (pos, pos | np.uint32(0x80000000)):
            v = bits.view(np.float32)
            got = unpack_nibbles(orc.e2m1_pack(v))
            want = brute_e2m1(v)
            bad = np.nonzero(got != want)[0]
            assert bad.size == 0, (v[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_e2m1_random_patterns_and_specials(orc):
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 2**32, size=1 << 21, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1.17549435e-38, 0.2499999, 0.2500001, 5.9999995, 6.0,
                         6.0000005, 7.0, 1e30, -1e30, 3.4028235e38, -3.4028235e38], np.float32)
    v = np.concatenate([v, specials]).astype(np.float32)
    if v.size % 2:
        v = v[:-1]
    got = unpack_nibbles(orc.e2m1_pack(v))
    assert np.array_equal(got, brute_e2m1(v))


def test_e2m1_pack_nibble_order(orc):
    # byte k = code(v[2k]) | code(v[2k+1]) << 4
    p = orc.e2m1_pack(np.array([0.5, 6.0, -1.0, 0.0], np.float32))
    assert list(p) == [0x71, 0x0A]


# ---------------------------------------------------------------- E8M0 shared scale (C4)

def test_e8m0_every_exponent_field(orc):
    rng = np.random.default_rng(7)
    mants = np.concatenate([[0, 1, 2, (1 << 22), (1 << 23) - 2, (1 << 23) - 1],
                            rng.integers(0, 1 << 23, size=250)]).astype(np.uint32)
    fields = np.arange(0, 255, dtype=np.uint32)
    bits = (fields[:, None] << 23) | mants[None, :]
    a = bits.reshape(-1).view(np.float32)
    assert np.array_equal(orc.e8m0_many(a).astype(np.int64), e8m0_from_bits(a))


def test_e8m0_closed_forms(orc):
    # powers of two map exactly: amax = 2^k -> e = k - 2
    for k in range(-124, 128):
        assert orc.e8m0(math.ldexp(1.0, k)) == max(k - 2, -127) + 127
    assert orc.e8m0(0.0) == 0
    assert orc.e8m0(float("inf")) == 0xFF and orc.e8m0(float("nan")) == 0xFF
    assert orc.e8m0(4.0) == 127 and orc.e8m0(np.nextafter(np.float32(4.0), np.float32(0))) == 126
    assert orc.e8m0(7.999999) == 127 and orc.e8m0(8.0) == 128


# ---------------------------------------------------------------- bf16 rounding of the expanded matrix

def test_bf16_from_f64_against_bracketing(orc):
    rng = np.random.default_rng(11)
    vals = list(rng.normal(0, 1, 3000) * np.exp2(rng.integers(-140, 120, 3000)))
    # exact bf16 midpoints (ties) and their neighbours
    for h in rng.integers(1, 0x7F7F, 500):
        a = float(bf16_bits_to_frac(int(h)))
        b = float(bf16_bits_to_frac(int(h) + 1))
        m = 0.5 * (a + b)
        vals += [m, np.nextafter(m, 0), np.nextafter(m, np.inf), -m]
    vals += [0.0, -0.0, 1e-45, 3.0e38, 3.4e38, 3.3961e38, 1e-40, -1e-41]
    for a in vals:
        got = orc.bf16_from_f64(a)
        q = Fraction(abs(a))
        # bracket |a| between adjacent bf16 patterns (patterns are monotone in value)
        f = np.array([abs(a)], np.float32)  # nearest fp32, then truncate to bf16
        h = int(f.view(np.uint32)[0] >> 16)
        cands = [c for c in (h - 1, h, h + 1, h + 2) if 0 <= c <= 0x7F80]
        best = None
        for c in cands:
            cv = bf16_bits_to_frac(c) if c < 0x7F80 else Fraction(2) ** 128
            dist = abs(cv - q)
            if best is None or dist < best[0] or (dist == best[0] and c % 2 == 0):
                best = (dist, c)
        want = best[1] | (0x8000 if math.copysign(1, a) < 0 else 0)
        assert got == want, (a, hex(got), hex(want))


# ---------------------------------------------------------------- factors and Kronecker expansion (C1, C2)

def test_factor_is_lu_product_with_unit_det(orc):
    rng = np.random.default_rng(3)
    for l, u, v in rng.normal(0, 1, (200, 3)).astype(np.float32):
        if abs(u) < 1e-3:
            continue
        F = orc.factor(l, u, v)
        assert np.array_equal(F, lu_numpy(l, u, v))
        assert abs(np.linalg.det(F) - 1.0) < 1e-12 * max(1.0, np.abs(F).max() ** 2)
        Fi = orc.factor(l, u, v, inverse=True)
        assert np.allclose(Fi, np.linalg.inv(F), rtol=1e-12, atol=1e-12 * np.abs(F).max() ** 2)


def test_expand_matches_numpy_kron_and_bit_convention(orc):
    params = inputs.lu_params(6, seed=5)
    K = orc.expand_f64(params)
    for b in range(6):
        Fs = [lu_numpy(*params[b, k]) for k in range(5)]
        ref = Fs[0]
        for F in Fs[1:]:
            ref = np.kron(ref, F)
        assert np.allclose(K[b], ref, rtol=1e-14, atol=0)
        # entry-wise: K[i][j] = prod_k F_k[bit(4-k) of i][bit(4-k) of j]  (F0 on the top bit)
        for i, j in itertools.product(range(32), range(32)):
            prod = 1.0
            for k in range(5):
                prod *= Fs[k][(i >> (4 - k)) & 1, (j >> (4 - k)) & 1]
            assert abs(K[b, i, j] - prod) <= 1e-14 * abs(prod)


def test_oracle_kron_against_numpy(orc):
    rng = np.random.default_rng(9)
    A = rng.normal(size=(2, 2))
    B = rng.normal(size=(4, 4))
    assert np.array_equal(orc.kron(A, B), np.kron(A, B))


def test_param_count_is_3log2n_and_under_half_of_per_channel():
    # "five 2x2 unit-determinant LU factors (15 parameters per block)" and
    # 3 log2(n) per block; "less than half the parameters of per-channel scaling"
    p = inputs.lu_params(36, seed=0)
    assert p.shape == (36, 5, 3) and p[0].size == 15 == 3 * int(math.log2(32))
    d = 1152
    assert (d // 32) * 15 < d / 2


def test_det_is_one(orc):
    params = inputs.lu_params(64, seed=21)
    K = orc.expand_f64(params)
    dets = np.linalg.det(K)
    assert np.all(np.abs(dets - 1.0) < 1e-9)
    K32 = orc.expand(params).astype(np.float64)
    assert np.all(np.abs(np.linalg.det(K32) - 1.0) < 1e-5)


def test_inverse_is_kron_of_factor_inverses(orc):
    params = inputs.lu_params(32, seed=22)
    K = orc.expand_f64(params)
    Ki = orc.expand_f64(params, inverse=True)
    assert np.allclose(Ki, np.linalg.inv(K), rtol=0, atol=1e-12)
    eye = np.broadcast_to(np.eye(32), K.shape)
    assert np.abs(K @ Ki - eye).max() < 1e-12


def test_weight_side_transform_keeps_products(orc):
    """[LRQ] eq. 2: Y = X W^T = (X H)(W H)^T for orthogonal H; with an invertible
    block transform the weight side takes K^-T instead: (x K)(w K^-T)^T = x w^T,
    block by block, in exact arithmetic (checked in fp64 against numpy)."""
    params = inputs.lu_params(8, seed=25)
    K = orc.expand_f64(params)
    KiT = np.swapaxes(orc.expand_f64(params, inverse=True), 1, 2)
    rng = np.random.default_rng(26)
    x = rng.standard_normal((16, 8, 32))
    w = rng.standard_normal((12, 8, 32))
    lhs = np.einsum("rbj,nbj->rn", np.einsum("rbi,bij->rbj", x, K), np.einsum("nbi,bij->nbj", w, KiT))
    rhs = np.einsum("rbi,nbi->rn", x, w)
    assert np.abs(lhs - rhs).max() < 1e-9 * np.abs(x).sum(axis=(1, 2)).max() * np.abs(w).max()


def test_round_trip_fp32_below_1e_5(orc):
    params = inputs.lu_params(36, seed=23)
    K32 = orc.expand(params).astype(np.float32)
    Ki32 = orc.expand(params, inverse=True).astype(np.float32)
    x = np.random.default_rng(24).standard_normal((64, 36, 32)).astype(np.float32)
    y = np.einsum("rbi,bij->rbj", x, K32).astype(np.float32)
    xr = np.einsum("rbj,bji->rbi", y, Ki32).astype(np.float32)
    err = np.abs(xr - x).max(axis=-1) / np.abs(x).max(axis=-1)
    assert err.max() < 1e-5


def test_bf16_expand_is_rounding_of_fp64(orc):
    params = inputs.lu_params(8, seed=25)
    K = orc.expand_f64(params)
    Kb = orc.expand(params, dtype=orc.BF16)
    # every bf16 entry is the nearest bf16 of the fp64 entry (checked with the
    # independent bracketing of test_bf16_from_f64_against_bracketing on a sample)
    vals = inputs.bf16_bits_to_f32(Kb).astype(np.float64)
    spacing = np.exp2(np.floor(np.log2(np.abs(K))) - 7)
    assert np.all(np.abs(vals - K) <= 0.5 * spacing)


# ---------------------------------------------------------------- Hadamard initialisation and Lemma 1

def sylvester_closed_form(n: int) -> np.ndarray:
    N = 1 << n
    i = np.arange(N)
    pc = np.vectorize(lambda t: bin(t).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0) * 2.0 ** (-n / 2)


def test_hadamard_matches_golden_h2_and_closed_form(orc):
    lines = [l.split() for l in open(os.path.join(GOLDEN, "hadamard_h2.txt")) if l.strip() and not l.startswith("#")]
    norm = float(lines[0][1])
    H2 = norm * np.array([[float(t) for t in r] for r in lines[1:]])
    assert np.allclose(orc.hadamard(1), H2, rtol=0, atol=4e-16)
    for n in (2, 3, 5):
        H = orc.hadamard(n)
        assert np.allclose(H, sylvester_closed_form(n), rtol=0, atol=1e-15)
        assert np.allclose(H @ H.T, np.eye(1 << n), atol=1e-14)  # eq. 2: H H^T = I


def test_hadamard_init_reproduces_h32_up_to_signs(orc):
    K = orc.expand_f64(inputs.hadamard_params(1))[0]
    D = np.diag([(-1.0) ** bin(i).count("1") for i in range(32)])
    H32 = sylvester_closed_form(5)
    assert np.abs(K - D @ H32).max() < 1e-6  # only fp32 rounding of 1/sqrt2 in the params
    assert np.allclose(np.abs(K), 2.0 ** -2.5, rtol=5e-7, atol=0)  # fp32 params: 1/u - u != u exactly
    assert np.abs(K @ K.T - np.eye(32)).max() < 1e-6
    # the FWHT comparison path uses fp32(H_32): entries are +-fp32(2^-2.5)
    assert np.all(np.abs(orc.hadamard(5).astype(np.float32)) == np.float32(2.0 ** -2.5))


def test_lemma1_norm_and_spread(orc):
    params = inputs.hadamard_params(1)
    K32 = orc.expand(params)
    rng = np.random.default_rng(31)
    for c in range(32):
        alpha = float(rng.choice([1.0, 3.5, -20.0, 96.0]))
        x = np.zeros((1, 32), np.float32)
        x[0, c] = alpha
        y = orc.transform(inputs.f32_to_bf16_bits(x), K32)[0].astype(np.float64)
        assert abs(np.linalg.norm(y) - abs(alpha)) < 1e-6 * abs(alpha)
        assert np.allclose(np.abs(y), abs(alpha) / math.sqrt(32), rtol=1e-6)


def test_lemma1_golden_quantized_onehot(orc):
    K32 = orc.expand(inputs.hadamard_params(1))
    rows = [l.split() for l in open(os.path.join(GOLDEN, "lemma1_onehot.txt")) if l.strip() and not l.startswith("#")]
    for c, byte, hexcodes in rows:
        x = np.zeros((1, 32), np.float32)
        x[0, int(c)] = 32.0
        q, s = orc.quantize(inputs.f32_to_bf16_bits(x), K32)
        assert s[0, 0] == int(byte)
        assert q[0].tobytes().hex() == hexcodes


# ---------------------------------------------------------------- transform and end-to-end quantize, brute force (C3..C6)

@pytest.mark.parametrize("dtype", [0, 1])
def test_transform_exact_rational_brute_force(orc, dtype):
    rng = np.random.default_rng(41 + dtype)
    M, d = 3, 64
    x = inputs.f32_to_bf16_bits((rng.standard_t(3, (M, d)) * rng.choice([1, 100], (M, d))).astype(np.float32))
    params = inputs.lu_params(d // 32, seed=42)
    mats = orc.expand(params, dtype=dtype)
    y = orc.transform(x, mats)
    matf = mats if dtype == 0 else inputs.bf16_bits_to_f32(mats)
    for r in range(M):
        for b in range(d // 32):
            xs = [bf16_bits_to_frac(int(h)) for h in x[r, 32 * b:32 * b + 32]]
            for j in range(32):
                exact = sum(xs[i] * Fraction(float(matf[b, i, j])) for i in range(32))
                assert y[r, 32 * b + j] == f32_round_fraction(exact), (r, b, j)


def test_quantize_end_to_end_brute_force(orc):
    rng = np.random.default_rng(51)
    M, d = 4, 96
    x = inputs.f32_to_bf16_bits((rng.standard_normal((M, d)) * 3).astype(np.float32))
    x[1, 32:64] = 0  # an all-zero block
    x[2, 5] = inputs.f32_to_bf16_bits(np.array([200.0], np.float32))[0]
    params = inputs.lu_params(d // 32, seed=52)
    K32 = orc.expand(params)
    q, s = orc.quantize(x, K32)
    for r in range(M):
        for b in range(d // 32):
            xs = [bf16_bits_to_frac(int(h)) for h in x[r, 32 * b:32 * b + 32]]
            y = np.array([f32_round_fraction(sum(xs[i] * Fraction(float(K32[b, i, j])) for i in range(32)))
                          for j in range(32)], np.float32)
            byte = int(e8m0_from_bits(np.array([np.abs(y).max()], np.float32))[0])
            assert s[r, b] == byte
            v = (y.astype(np.float64) * 2.0 ** (127 - byte)).astype(np.float32)
            assert np.array_equal(unpack_nibbles(q[r, 16 * b:16 * b + 16]), brute_e2m1(v))


def test_nonfinite_block_rule(orc):
    y = np.zeros((1, 64), np.float32)
    y[0, 3] = np.inf
    y[0, 40] = 1.0
    q, s = orc.mx_quantize(y)
    assert s[0, 0] == 0xFF and not q[0, :16].any()
    assert s[0, 1] == orc.e8m0(1.0)


def test_scale_and_nonfinite_rule_see_every_position(orc):
    """Under K = I, a block whose largest magnitude sits at position j, for every
    j: amax = 24 gives e = floor(log2 24) - 2 = 2 (byte 129); 24 / 4 = 6 is code 7
    at j, and 0.5 / 4 = 0.125 (below the 0.25 midpoint) is code 0 elsewhere.  A
    NaN at position j alone gives byte 0xFF and 32 zero codes."""
    K = orc.expand(inputs.identity_params(1))
    for j in range(32):
        a = np.full((1, 32), 0.5, np.float32)
        a[0, j] = 24.0
        q, s = orc.quantize(inputs.f32_to_bf16_bits(a), K)
        codes = np.stack([q[0] & 0xF, q[0] >> 4], axis=-1).reshape(-1)
        expected = np.zeros(32, np.uint8)
        expected[j] = 7
        assert s[0, 0] == 129 and np.array_equal(codes, expected), j
        a[0, j] = np.nan
        q, s = orc.quantize(inputs.f32_to_bf16_bits(a), K)
        assert s[0, 0] == 0xFF and not q.any(), j


def test_dequantize_is_grid_value_times_scale(orc):
    rng = np.random.default_rng(61)
    y = (rng.standard_normal((8, 64)) * np.exp2(rng.integers(-10, 10, (8, 1)))).astype(np.float32)
    q, s = orc.mx_quantize(y)
    yh = orc.dequantize(q, s)
    codes = unpack_nibbles(q.reshape(-1)).reshape(8, 64)
    scale = np.exp2(np.repeat(s.astype(np.int64) - 127, 32, axis=1).astype(np.float64))
    sign = np.where(codes >= 8, -1.0, 1.0)
    assert np.array_equal(yh, sign * E2M1_MAGS[codes & 7] * scale)
    # the error of each element is at most half a grid step (or the saturation gap)
    assert np.all(np.abs(yh - y) <= np.maximum(1.0 * scale, np.abs(y) - 6 * scale + 1e-30))


def test_dequantize_with_inverse_undoes_transform(orc):
    params = inputs.lu_params(4, seed=62)
    K32, Ki32 = orc.expand(params), orc.expand(params, inverse=True)
    y = np.random.default_rng(63).standard_normal((5, 128)).astype(np.float32)
    q, s = orc.mx_quantize(y)
    yh = orc.dequantize(q, s)
    xh = orc.dequantize(q, s, inv_mats=Ki32)
    ref = np.einsum("rbj,bji->rbi", yh.reshape(5, 4, 32), Ki32.astype(np.float64)).reshape(5, 128)
    assert np.allclose(xh, ref, rtol=1e-12, atol=1e-12)


def test_smooth_is_single_rounding_of_product(orc):
    rng = np.random.default_rng(71)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((6, 64)).astype(np.float32) * 7)
    inv_s = rng.uniform(0.01, 3.0, 64).astype(np.float32)
    q, s = orc.smooth_quantize(x, inv_s)
    y = inputs.bf16_bits_to_f32(x) * inv_s[None, :]  # fp32 multiply: one IEEE rounding
    q2, s2 = orc.mx_quantize(y.astype(np.float32))
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


def test_fwht_equals_kroquant_with_sylvester_matrix(orc):
    rng = np.random.default_rng(81)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((7, 96)).astype(np.float32))
    q, s = orc.fwht_quantize(x)
    H = np.broadcast_to(sylvester_closed_form(5).astype(np.float32), (3, 32, 32)).copy()
    q2, s2 = orc.quantize(x, H)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


# ---------------------------------------------------------------- transform blocks of n = 2^k elements

@pytest.mark.parametrize("log2n", [4, 6, 7])
def test_expand_n_matches_numpy_kron(orc, log2n):
    """[KQ-sum, Limitations]: 3 log2(n) parameters per n-element block; K is the
    Kronecker product of the log2(n) LU factors, F_0 on the top index bit."""
    params = inputs.lu_params(3, seed=60 + log2n, factors=log2n)
    K = orc.expand_n_f64(params)
    n = 1 << log2n
    assert K.shape == (3, n, n) and params[0].size == 3 * log2n
    for c in range(3):
        ref = lu_numpy(*params[c, 0])
        for k in range(1, log2n):
            ref = np.kron(ref, lu_numpy(*params[c, k]))
        assert np.allclose(K[c], ref, rtol=1e-13, atol=0)
    sign, logdet = np.linalg.slogdet(K)
    assert np.all(sign > 0) and np.abs(logdet).max() < 1e-9       # det = 1
    Ki = orc.expand_n_f64(params, inverse=True)
    assert np.allclose(Ki, np.linalg.inv(K), rtol=0, atol=1e-10)


def test_expand_n_at_32_is_the_block_expansion(orc):
    params = inputs.lu_params(4, seed=66)
    assert np.array_equal(orc.expand_n(params).view(np.uint32), orc.expand(params).view(np.uint32))
    assert np.array_equal(orc.expand_n(params, dtype=orc.BF16), orc.expand(params, dtype=orc.BF16))


def test_hadamard_init_n64_reproduces_h64_up_to_signs(orc):
    K = orc.expand_n_f64(inputs.hadamard_params(1, factors=6))[0]
    D = np.diag([(-1.0) ** bin(i).count("1") for i in range(64)])
    assert np.abs(K - D @ sylvester_closed_form(6)).max() < 1e-6
    assert np.abs(K @ K.T - np.eye(64)).max() < 1e-6


@pytest.mark.parametrize("log2n", [4, 6, 7])
@pytest.mark.parametrize("dtype", [0, 1])
def test_transform_n_exact_rational_brute_force(orc, dtype, log2n):
    n = 1 << log2n
    rng = np.random.default_rng(67 + dtype + 10 * log2n)
    M, d = 2, 2 * n if n >= 32 else 64
    x = inputs.f32_to_bf16_bits((rng.standard_t(3, (M, d)) * rng.choice([1, 100], (M, d))).astype(np.float32))
    params = inputs.lu_params(d // n, seed=68 + log2n, factors=log2n)
    mats = orc.expand_n(params, dtype=dtype)
    y = orc.transform_n(x, mats)
    matf = mats if dtype == 0 else inputs.bf16_bits_to_f32(mats)
    for r in range(M):
        for c in range(d // n):
            xs = [bf16_bits_to_frac(int(h)) for h in x[r, n * c:n * c + n]]
            for j in range(0, n, 5 if n <= 64 else 11):
                exact = sum(xs[i] * Fraction(float(matf[c, i, j])) for i in range(n))
                assert y[r, n * c + j] == f32_round_fraction(exact), (r, c, j)


@pytest.mark.parametrize("log2n", [4, 6, 7])
def test_quantize_n_is_mx_of_the_transform(orc, log2n):
    """MXFP4 per 32 elements of the n-element block transform: scales by the
    bit-field rule from each 32-block's amax, codes by the brute-force nearest
    value."""
    n = 1 << log2n
    rng = np.random.default_rng(69 + log2n)
    d = max(128, 2 * n)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((3, d)).astype(np.float32))
    mats = orc.expand_n(inputs.lu_params(d // n, seed=70 + log2n, factors=log2n))
    y = orc.transform_n(x, mats)
    q, s = orc.quantize_n(x, mats)
    nb = d // 32
    amax = np.abs(y.reshape(3, nb, 32)).max(axis=2)
    assert np.array_equal(s, e8m0_from_bits(amax.astype(np.float32)).astype(np.uint8))
    scale = np.exp2(s.astype(np.float64) - 127.0)
    v = (y.reshape(3, nb, 32) / scale[:, :, None]).astype(np.float32).reshape(3, d)
    assert np.array_equal(unpack_nibbles(q).reshape(3, d), brute_e2m1(v))


# ---------------------------------------------------------------- the W4A4 product (consumer of the codes)

def _golden_e2m1_values() -> dict:
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_grid.txt")) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 2 and parts[0].isdigit():
                vals[int(parts[0])] = Fraction(parts[1])
    assert len(vals) == 16
    return vals


def test_mx_gemm_exact_rational_brute_force(orc):
    """Every entry of the oracle's W4A4 product against an exact rational sum written
    from the E2M1 table of the OCP definition (tests/golden/e2m1_grid.txt) and the
    header's nibble order, with ragged K (three 32-blocks) and scales of both signs
    of exponent.  A swapped nibble, a scale read from the wrong block or row, or a
    transposed operand changes some entry."""
    vals = _golden_e2m1_values()
    rng = np.random.default_rng(71)
    M, N, K = 3, 4, 96
    aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(100, 150, (M, K // 32), dtype=np.uint8)
    sb = rng.integers(100, 150, (N, K // 32), dtype=np.uint8)
    c = orc.mx_gemm(aq, sa, bq, sb)

    def elem(q, s, r, k):
        byte = int(q[r, k // 2])
        code = byte >> 4 if k % 2 else byte & 0xF
        return vals[code] * Fraction(2) ** (int(s[r, k // 32]) - 127)

    for m in range(M):
        for n in range(N):
            exact = sum(elem(aq, sa, m, k) * elem(bq, sb, n, k) for k in range(K))
            assert c[m, n] == float(exact), (m, n)  # fp64 holds every partial sum exactly here


def test_mx_gemm_one_hot_closed_form(orc):
    """A single nonzero element on each side: c = value_a value_b 2^(sa + sb - 254)
    at exactly one (m, n), zero elsewhere."""
    M, N, K = 2, 3, 64
    aq = np.zeros((M, K // 2), np.uint8)
    bq = np.zeros((N, K // 2), np.uint8)
    aq[1, 37 // 2] = 0x7 << 4          # element 37 (odd: high nibble) = +6
    bq[2, 37 // 2] = 0xB << 4          # element 37 of weight row 2 = -1.5
    sa = np.full((M, K // 32), 127, np.uint8)
    sb = np.full((N, K // 32), 127, np.uint8)
    sa[1, 1], sb[2, 1] = 130, 120     # block 1 holds element 37
    c = orc.mx_gemm(aq, sa, bq, sb)
    want = np.zeros((M, N))
    want[1, 2] = 6.0 * -1.5 * 2.0 ** (3 - 7)
    assert np.array_equal(c, want)


def test_mx_gemm_nan_scale_poisons_its_row_and_column(orc):
    """Scale byte 0xFF is NaN (OCP MX): every product that reads such a block is NaN."""
    rng = np.random.default_rng(72)
    M, N, K = 3, 3, 64
    aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    bq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = np.full((M, 2), 127, np.uint8)
    sb = np.full((N, 2), 127, np.uint8)
    sa[0, 1] = 0xFF
    sb[2, 0] = 0xFF
    c = orc.mx_gemm(aq, sa, bq, sb)
    assert np.isnan(c[0]).all() and np.isnan(c[:, 2]).all()
    assert np.isfinite(c[1:, :2]).all()


# ---------------------------------------------------------------- AdaLN normalisation (the quantizer's producer)

def _bf16_near(h_bits: np.ndarray, ref: np.ndarray, slack: np.ndarray) -> np.ndarray:
    """True where the bf16 value h lies within half a bf16 place of the reference plus
    `slack` (the fp32 evaluation's distance from the exact value): the nearest bf16 value,
    or a neighbour when the reference is that close to a rounding midpoint."""
    h = inputs.bf16_bits_to_f32(h_bits).astype(np.float64)
    mag = np.maximum(np.abs(ref), 2.0**-126)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    return (np.abs(h - ref) <= 0.5 * ulp + slack) | ~np.isfinite(ref)


def test_adaln_matches_torch_fp64_layer_norm(orc):
    """The oracle's modulated LayerNorm (fp32, fixed pairwise order) against torch's fp64
    layer_norm (a library routine with its own reduction order): the statistics agree
    to fp32 accuracy, and every bf16 output is within half a bf16 place of torch's fp64
    result plus the fp32 evaluation's error bound (so almost always the nearest bf16
    value).  Rows with outliers of 2^12, a large mean, two groups, ragged d."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(81)
    u = 2.0**-24
    for d, rpg in ((96, 3), (1152, 5), (3104, 4)):
        M = 8
        a = rng.standard_normal((M, d)).astype(np.float32)
        a[:, rng.choice(d, 3, replace=False)] *= 4096.0
        a[2] += 1000.0                                  # a large mean
        x = inputs.f32_to_bf16_bits(a)
        G = -(-M // rpg)
        shift = inputs.f32_to_bf16_bits(rng.standard_normal((G, d)).astype(np.float32))
        scale = inputs.f32_to_bf16_bits((0.3 * rng.standard_normal((G, d))).astype(np.float32))
        eps = 1e-6
        h, stats = orc.adaln(x, shift, scale, rpg, eps)
        xt = torch.from_numpy(inputs.bf16_bits_to_f32(x).astype(np.float64))
        ln = torch.nn.functional.layer_norm(xt, (d,), eps=eps)
        g = np.arange(M) // rpg
        sc = inputs.bf16_bits_to_f32(scale).astype(np.float64)[g]
        sh = inputs.bf16_bits_to_f32(shift).astype(np.float64)[g]
        ref = ln.numpy() * (1 + sc) + sh
        xa = np.abs(xt.numpy())
        mu = xt.mean(dim=1).numpy()
        var = xt.var(dim=1, unbiased=False).numpy()
        rstd = 1 / np.sqrt(var + eps)
        # fp32 error of the definition: the mean to within (log2 d + 1) u of sum|x| / d, the
        # normalised value to within a few u of (|x - mu| + mu error) rstd, then two more
        # roundings through the modulation
        lg = np.ceil(np.log2(d)) + 2
        mu_err = lg * u * xa.sum(axis=1) / d
        assert np.all(np.abs(stats[:, 0] - mu) <= mu_err + 1e-30)
        assert np.allclose(stats[:, 1], rstd, rtol=64 * lg * u * (1 + (np.abs(mu) / np.sqrt(var)) ** 2))
        tn = (np.abs(xt.numpy() - mu[:, None]) + mu_err[:, None]) * rstd[:, None]
        slack = 8 * u * (tn * np.abs(1 + sc) + np.abs(sh)) + 4 * lg * u * (1 + (np.abs(mu) / np.sqrt(var)) ** 2)[:, None] * tn * np.abs(1 + sc)
        assert _bf16_near(h, ref, slack).all(), d


def test_adaln_constant_row_is_the_shift(orc):
    """A constant row has mean equal to the constant and variance 0, so its normalised
    values are 0 and the output is the shift vector exactly (any d, any eps > 0)."""
    d = 160
    x = np.full((3, d), 0x4049, np.uint16)               # 3.140625
    x[1] = 0xC2C8                                          # -100
    rng = np.random.default_rng(82)
    shift = inputs.f32_to_bf16_bits(rng.standard_normal((1, d)).astype(np.float32))
    scale = inputs.f32_to_bf16_bits(rng.standard_normal((1, d)).astype(np.float32))
    h, stats = orc.adaln(x, shift, scale, 3, 1e-5)
    assert np.array_equal(inputs.bf16_bits_to_f32(h), np.repeat(inputs.bf16_bits_to_f32(shift), 3, axis=0))
    assert stats[0, 0] == np.float32(3.140625) and stats[1, 0] == np.float32(-100.0)
    assert stats[0, 1] == np.float32(1) / np.sqrt(np.float32(1e-5))


def test_adaln_group_of_each_row(orc):
    """Rows take the modulation vectors of group row // rows_per_group: constant rows
    with group g's shift equal to g give h = g."""
    d, M, rpg = 64, 11, 4
    x = np.full((M, d), 0x3F80, np.uint16)                # 1.0
    shift = inputs.f32_to_bf16_bits(np.repeat(np.arange(3, dtype=np.float32)[:, None] + 10, d, axis=1))
    scale = np.zeros((3, d), np.uint16)
    h, _ = orc.adaln(x, shift, scale, rpg, 1e-6)
    assert np.array_equal(inputs.bf16_bits_to_f32(h)[:, 0], 10.0 + np.arange(M) // rpg)


def test_adaln_symmetric_row_closed_form(orc):
    """x = (+a, -a, +a, ...): mean 0 and variance a^2 exactly in fp32 (every partial sum
    is exact), so h_i = +-a (1 + s_i) / sqrt(a^2 + eps) + b_i up to the fp32 roundings
    of rstd and the modulation, against exact arithmetic in fp64."""
    d, a = 256, 3.5
    x = np.where(np.arange(d) % 2 == 0, 0x4060, 0xC060).astype(np.uint16)[None, :]  # +-3.5
    rng = np.random.default_rng(83)
    shift = inputs.f32_to_bf16_bits(rng.standard_normal((1, d)).astype(np.float32))
    scale = inputs.f32_to_bf16_bits((0.5 * rng.standard_normal((1, d))).astype(np.float32))
    eps = 2.0**-20
    h, stats = orc.adaln(x, shift, scale, 1, eps)
    assert stats[0, 0] == 0.0
    rstd = 1.0 / math.sqrt(a * a + eps)
    assert abs(stats[0, 1] - rstd) <= 2 * 2.0**-24 * rstd
    sgn = np.where(np.arange(d) % 2 == 0, 1.0, -1.0)
    s1 = 1 + inputs.bf16_bits_to_f32(scale)[0].astype(np.float64)
    b = inputs.bf16_bits_to_f32(shift)[0].astype(np.float64)
    ref = sgn * a * rstd * s1 + b
    slack = 6 * 2.0**-24 * (a * rstd * np.abs(s1) + np.abs(b))
    assert _bf16_near(h[0], ref, slack).all()


# ---------------------------------------------------------------- exhaustive sweeps of the element rules

E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def e2m1_by_midpoints(v: np.ndarray) -> np.ndarray:
    """E2M1 code from the position of |v| among the midpoints of the grid: the number of
    midpoints strictly below |v|, plus one at an exact midpoint whose lower code is odd
    (ties to the even code); everything above 5 saturates to 7; sign bit from v."""
    m = np.abs(v.astype(np.float64))
    k = np.searchsorted(E2M1_MIDPOINTS, m, side="left")
    tie = (k < 7) & (m == E2M1_MIDPOINTS[np.minimum(k, 6)])
    code = k + (tie & (k % 2 == 1))
    return code | (np.signbit(v).astype(np.int64) << 3)


def test_e2m1_every_fp32_pattern(orc):
    """All 2^32 fp32 bit patterns but NaN: inside [2^-3, 2^3) against the midpoint rule
    (an independent formulation of nearest-even on the grid), outside it the two constant
    answers (0 below 2^-3, 7 from 2^3 up, infinities included) with the sign bit."""
    step = 1 << 24
    lo = int(np.float32(0.125).view(np.uint32))
    hi = int(np.float32(8.0).view(np.uint32))
    inf = int(np.float32(np.inf).view(np.uint32))
    for start in range(0, 1 << 31, step):
        pos = np.arange(start, start + step, dtype=np.uint32)
        keep = pos <= inf                                    # NaN patterns dropped
        pos = pos[keep]
        for sign in (0, 0x80000000):
            bits = pos | np.uint32(sign)
            v = bits.view(np.float32)
            if v.size % 2:
                v = np.append(v, v[-1])
            packed = orc.e2m1_pack(v)
            s = 8 if sign else 0
            if start + step <= lo:                           # two equal nibbles per byte
                assert np.all(packed == s * 17), start
            elif start >= hi:
                assert np.all(packed == (7 | s) * 17), start
            else:
                assert np.array_equal(unpack_nibbles(packed), e2m1_by_midpoints(v)), start


def test_e8m0_every_positive_finite_value(orc):
    """Every positive finite fp32 value (and +0): the byte is floor(log2 amax) - 2 + 127,
    clamped, from the exponent field for normal values; subnormals (field 0) and zero
    against the bit-field reference."""
    step = 1 << 23                                           # one exponent field per chunk
    for field in range(0, 255):
        bits = (np.uint32(field) << np.uint32(23)) | np.arange(step, dtype=np.uint32)
        a = bits.view(np.float32)
        got = orc.e8m0_many(a).astype(np.int64)
        if field == 0:
            assert np.array_equal(got, e8m0_from_bits(a))
        else:
            assert np.all(got == min(max(field - 127 - 2, -127), 127) + 127), field
