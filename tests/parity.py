"""Parity accounting between a device result and the oracle, as the quantizer's
tolerance states it: scales bit-exact; codes bit-exact except codes whose fp32
pre-rounding value v* lies within 1e-6 (relative) of an E2M1 rounding boundary,
which may differ by one code, and at most 1e-4 of all codes may do so."""
from __future__ import annotations

import numpy as np

BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
# value order of codes: magnitude index for codes 0..7, sign from bit 3
REL_WINDOW = 1e-6
MAX_EXEMPT_FRACTION = 1e-4


def unpack(q: np.ndarray) -> np.ndarray:
    q = np.asarray(q, np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), np.int64)
    out[..., 0::2] = q & 0xF
    out[..., 1::2] = q >> 4
    return out


def signed_rank(code: np.ndarray) -> np.ndarray:
    """Position on the ordered E2M1 grid (-7..7; +0 and -0 both 0)."""
    mag = code & 7
    return np.where(code & 8, -mag, mag)


def compare(q_dev, s_dev, q_ref, s_ref, y_ref=None) -> dict:
    q_dev, q_ref = np.asarray(q_dev), np.asarray(q_ref)
    s_dev, s_ref = np.asarray(s_dev), np.asarray(s_ref)
    assert q_dev.shape == q_ref.shape and s_dev.shape == s_ref.shape
    scale_mis = int(np.count_nonzero(s_dev != s_ref))
    cd, cr = unpack(q_dev), unpack(q_ref)
    mis = cd != cr
    n_mis = int(np.count_nonzero(mis))
    exempt = 0
    bad = n_mis
    if n_mis and y_ref is not None:
        y = np.asarray(y_ref, np.float32)
        e = np.repeat(s_ref.astype(np.int64) - 127, 32, axis=-1)
        v = np.abs(y.astype(np.float64) * np.exp2(-e.astype(np.float64)))
        near = np.zeros_like(mis)
        for B in BOUNDARIES:
            near |= np.abs(v - B) <= REL_WINDOW * B
        one_code = np.abs(signed_rank(cd) - signed_rank(cr)) == 1
        ok = mis & near & one_code
        exempt = int(np.count_nonzero(ok))
        bad = n_mis - exempt
    n_codes = cd.size
    return dict(
        n_codes=n_codes, n_scales=s_ref.size, scale_mismatch=scale_mis, code_mismatch=n_mis, exempt=exempt,
        bad=bad, ok=(scale_mis == 0 and bad == 0 and exempt <= MAX_EXEMPT_FRACTION * n_codes),
    )
