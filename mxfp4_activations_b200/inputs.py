"""Seeded synthetic inputs for the quantizer (shared by tests and bench).

This module holds no arithmetic of the method: it only draws activations and
per-block LU parameters with numpy's PCG64 and rounds the activations to bf16
bit patterns.  The workloads stand in for the DiT activations named on the
KroQuant pages (PixArt-Sigma, SANA, FLUX.1-schnell); no real activations or
weights are used.
"""
from __future__ import annotations

import math

import numpy as np

# (l, u, v) of the 2x2 LU factor L(l) U(u, v) that equals (1/sqrt2)[[1,1],[-1,1]],
# the unit-determinant stand-in for the Hadamard H_2 used as initialisation.
HADAMARD_INIT = (-1.0, 1.0 / math.sqrt(2.0), 1.0 / math.sqrt(2.0))

CONFIGS = {
    # name: M, list of d, activation law, outlier recipe, seed
    "cfg0": dict(M=64, ds=(1152,), law="normal", outlier_count=12, outlier_scale=(50.0, 50.0), token_lognormal=None, seed=0),
    "pixart": dict(M=8192, ds=(1152, 4608), law="t4", outlier_frac=0.01, outlier_scale=(20.0, 100.0), token_lognormal=None, seed=1),
    "sana": dict(M=2048, ds=(2240, 5600), law="normal", outlier_frac=0.005, outlier_scale=(100.0, 100.0), token_lognormal=0.5, seed=2),
    "flux": dict(M=4608, ds=(3072, 12288), law="t3", outlier_frac=0.005, outlier_scale=(100.0, 100.0), token_lognormal=None, seed=3),
}
SWEEP_M = (1, 16, 256, 4096, 16384, 65536)
# W4A4 products of the FLUX.1-schnell-shaped workload (4608 tokens of width 3072):
# name: (M tokens, N outputs, K inputs) of the linear layer the quantized rows feed.
GEMM_SHAPES = {
    "flux_proj": (4608, 3072, 3072),
    "flux_fc1": (4608, 12288, 3072),
    "flux_fc2": (4608, 3072, 12288),
}
SWEEP_D = (1152, 3072, 12288)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    a = np.ascontiguousarray(a, np.float32)
    w = a.view(np.uint32)
    # only NaN patterns can wrap around in 32 bits; they are replaced below
    rounded = ((w + np.uint32(0x7FFF) + ((w >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        rounded[nan] = 0x7FC0
    return rounded


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def lu_params(nb: int, seed, noise: float = 0.05, factors: int = 5) -> np.ndarray:
    """Per-block params [nb, factors, 3] fp32 (5 factors for 32-element blocks, 6
    for 64): Hadamard initialisation + N(0, noise)."""
    rng = np.random.default_rng(seed)
    base = np.array(HADAMARD_INIT, np.float64)
    p = base[None, None, :] + rng.normal(0.0, noise, size=(nb, factors, 3))
    return p.astype(np.float32)


def hadamard_params(nb: int, factors: int = 5) -> np.ndarray:
    return np.tile(np.array(HADAMARD_INIT, np.float32), (nb, factors, 1))


def identity_params(nb: int) -> np.ndarray:
    """l = 0, u = 1, v = 0 for every factor: K = I."""
    p = np.zeros((nb, 5, 3), np.float32)
    p[:, :, 1] = 1.0
    return p


def activations(M: int, d: int, law: str, seed, outlier_frac: float | None = None,
                outlier_count: int | None = None, outlier_scale=(50.0, 50.0),
                token_lognormal: float | None = None, row_chunk: int = 4096) -> np.ndarray:
    """bf16 bit patterns [M, d].  Outlier channels are drawn without replacement
    and multiplied by a per-channel factor uniform in outlier_scale; with
    token_lognormal every row is multiplied by a lognormal(0, sigma) factor."""
    rng = np.random.default_rng(seed)
    k = outlier_count if outlier_count is not None else max(1, int(round(outlier_frac * d)))
    chans = rng.choice(d, size=k, replace=False)
    lo, hi = outlier_scale
    ch_scale = np.ones(d, np.float32)
    ch_scale[chans] = rng.uniform(lo, hi, size=k) if hi > lo else lo
    out = np.empty((M, d), np.uint16)
    for r0 in range(0, M, row_chunk):
        r1 = min(M, r0 + row_chunk)
        n = (r1 - r0, d)
        if law == "normal":
            a = rng.standard_normal(n, dtype=np.float32)
        elif law.startswith("t"):
            a = rng.standard_t(float(law[1:]), size=n).astype(np.float32)
        else:
            raise ValueError(law)
        a *= ch_scale[None, :]
        if token_lognormal is not None:
            a *= rng.lognormal(0.0, token_lognormal, size=(r1 - r0, 1)).astype(np.float32)
        out[r0:r1] = f32_to_bf16_bits(a)
    return out


def config_case(name: str, d: int, M: int | None = None):
    """(x bf16 bits [M, d], params [d/32, 5, 3]) for one shape of a named config."""
    c = CONFIGS[name]
    M = c["M"] if M is None else M
    x = activations(M, d, c["law"], seed=[c["seed"], d, 0], outlier_frac=c.get("outlier_frac"),
                    outlier_count=c.get("outlier_count"), outlier_scale=c["outlier_scale"],
                    token_lognormal=c["token_lognormal"])
    params = lu_params(d // 32, seed=[c["seed"], d, 1])
    return x, params


def sweep_case(M: int, d: int):
    idx = SWEEP_M.index(M) * len(SWEEP_D) + SWEEP_D.index(d) if (M in SWEEP_M and d in SWEEP_D) else 0
    x = activations(M, d, "normal", seed=[4 + idx, 0], outlier_frac=0.01, outlier_scale=(50.0, 50.0))
    params = lu_params(d // 32, seed=[4 + idx, 1])
    return x, params


def smooth_inv_scale(x_bits: np.ndarray) -> np.ndarray:
    """Per-channel smoothing vector for the comparison kernel: SmoothQuant with
    alpha = 0.5 and unit weight statistics, inv_s_j = 1 / sqrt(max_rows |x_j|)."""
    a = np.abs(bf16_bits_to_f32(x_bits)).max(axis=0).astype(np.float64)
    a = np.maximum(a, 1e-6)
    return (1.0 / np.sqrt(a)).astype(np.float32)


def mx_operand(rows: int, K: int, seed, scale_range=(118, 136)):
    """A random MXFP4 operand: codes [rows, K/2] (uniform bytes: every E2M1 code and
    sign in both nibbles) and row-major E8M0 scale bytes [rows, K/32] drawn uniformly
    from scale_range (inclusive)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    s = rng.integers(scale_range[0], scale_range[1] + 1, (rows, K // 32), dtype=np.uint8)
    return q, s
