"""Host estimate of the share of 32-element blocks that the certified kernels send to
their exact (fp64) path.

A block goes there when its allowance E, the kernel's bound on the error of its fast
result, leaves the block's E8M0 scale or one of its E2M1 codes undecided.  This
estimate centres each interval on the oracle's fp32 result (a kernel centres it on
its own fast result, which lies within E of that) and uses the exact ||x||_1 (the
kernels use an upper bound), so it tracks the rate without reproducing it block for
block.  It uses the oracle and numpy only.

    python tests/exact_path_rate.py          # writes profiles/kq_exact_path_rate.json
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mxfp4_activations_b200 import inputs  # noqa: E402

U = 2.0**-24
# name: (matrix dtype, C (units of u), extra per unit of ||x||_1, per unit of max|K|, absolute)
ALLOWANCES = {
    "tensor_core_bf16_K": ("bf16", 66, 2.0**-124, 2.0**-120, 2.0**-118),
    "tensor_core_fp32_K": ("f32", 198, 2.0**-124, 2.0**-120, 2.0**-118),
    "butterfly": ("f32", 14 * (1 + 2.0**-16), 0.0, 0.0, 0.0),
    # the allowances the tensor-core variant used before its bound was derived
    "tensor_core_bf16_K_calibrated_16u": ("bf16", 16, 0.0, 0.0, 2.0**-110),
    "tensor_core_fp32_K_calibrated_32u": ("f32", 32, 0.0, 0.0, 2.0**-110),
}


def _codes(orc, v: np.ndarray) -> np.ndarray:
    packed = orc.e2m1_pack(v.astype(np.float32))
    out = np.empty(packed.size * 2, np.uint8)
    out[0::2] = packed & 0xF
    out[1::2] = packed >> 4
    return out.reshape(v.shape)


def rate(orc, x: np.ndarray, mats: np.ndarray, c_units: float, l1_extra: float, abs_k: float, abs0: float) -> float:
    """Share of the non-zero blocks of x (bf16 bits [M, d]) whose interval
    y32 -+ E decides neither the scale nor every code."""
    M, d = x.shape
    nb = d // 32
    y = orc.transform(x, mats).astype(np.float64).reshape(M, nb, 32)
    xf = inputs.bf16_bits_to_f32(x).astype(np.float64).reshape(M, nb, 32)
    k = inputs.bf16_bits_to_f32(mats) if mats.dtype == np.uint16 else mats
    kmax = np.abs(k.astype(np.float64)).reshape(nb, -1).max(axis=1)
    l1 = np.abs(xf).sum(axis=2)
    E = (c_units * U * kmax + l1_extra)[None, :] * l1 + abs_k * kmax[None, :] + abs0
    amax = np.abs(y).max(axis=2)
    hi = orc.e8m0_many((amax + E).astype(np.float32)).reshape(M, nb).astype(np.int64)
    lo = orc.e8m0_many(np.maximum(amax - E, 0.0).astype(np.float32)).reshape(M, nb).astype(np.int64)
    s = np.ldexp(1.0, 127 - hi)[..., None]
    cl = _codes(orc, (y - E[..., None]) * s)
    ch = _codes(orc, (y + E[..., None]) * s)
    undecided = (hi != lo) | (cl != ch).any(axis=2)
    nonzero = (xf != 0).any(axis=2)
    return float((undecided & nonzero).sum() / max(1, nonzero.sum()))


def estimate(orc, rows: int | None = None) -> dict:
    out = {}
    for d in inputs.CONFIGS["flux"]["ds"]:
        x, params = inputs.config_case("flux", d)
        if rows is not None:
            x = x[:rows]
        mats = {"f32": orc.expand(params, dtype=orc.F32), "bf16": orc.expand(params, dtype=orc.BF16)}
        out[str(d)] = {name: rate(orc, x, mats[dt], c, e1, ek, e0)
                       for name, (dt, c, e1, ek, e0) in ALLOWANCES.items()}
    return out


def main():
    from oracle import oracle as orc

    orc.build()
    rates = estimate(orc)
    rec = {
        "what": "share of non-zero 32-element blocks sent to the exact path (host estimate, see tests/exact_path_rate.py)",
        "workload": "FLUX.1-schnell-shaped activations, M=4608 x d in {3072, 12288}, the bench's inputs",
        "command": "python tests/exact_path_rate.py",
        "allowances": {k: {"matrices": v[0], "C_u": v[1]} for k, v in ALLOWANCES.items()},
        "rates": rates,
    }
    path = os.path.join(ROOT, "profiles", "kq_exact_path_rate.json")
    with open(path, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec["rates"], indent=1))


if __name__ == "__main__":
    main()
