"""The quantizer fused with the AdaLN-modulated LayerNorm (kq_adaln_quantize) against the
oracle: statistics, codes and scales bit for bit, every row, outputs inside canary
bytes."""
from __future__ import annotations

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from mxfp4_activations_b200 import inputs  # noqa: E402

from .parity import guarded, guards_intact, oracle_rows, tiled_scales  # noqa: E402

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


def dev_bits(a: np.ndarray) -> "torch.Tensor":
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def modulation(G: int, d: int, seed) -> tuple[np.ndarray, np.ndarray]:
    rng = np.random.default_rng(seed)
    shift = inputs.f32_to_bf16_bits((0.5 * rng.standard_normal((G, d))).astype(np.float32))
    scale = inputs.f32_to_bf16_bits((0.3 * rng.standard_normal((G, d))).astype(np.float32))
    return shift, scale


FORMS = ("two_kernel", "fused")


def run(kq, x, shift, scale, rpg, params, eps=1e-6, layout="row", form="two_kernel"):
    """Device codes, scales and statistics, each inside canary bytes.  form: "two_kernel"
    asks for the statistics (the statistics pass, then the butterfly quantizer's AdaLN
    form); "fused" passes none (one fused kernel), and the statistics come back None."""
    M, d = x.shape
    bt = kq.BlockTransform(torch.from_numpy(params).cuda())
    qv, qbuf = guarded(torch, M * (d // 2))
    sv, sbuf = guarded(torch, kq.scale_bytes(M, d, layout))
    if layout == "mma":
        sv.zero_()
    tv, tbuf = guarded(torch, M * 8)
    q = qv.view(M, d // 2)
    s = sv.view(M, d // 32) if layout == "row" else sv
    st = tv.view(torch.float32).view(M, 2) if form == "two_kernel" else None
    bt.adaln_quantize(dev_bits(x), dev_bits(shift), dev_bits(scale), rpg, eps=eps, q=q, scales=s,
                      scale_layout=layout, stats=st)
    torch.cuda.synchronize()
    for b in (qbuf, sbuf, tbuf):
        assert guards_intact(torch, b), "a kernel wrote outside its output buffer"
    assert kq.kq_get_device_error(clear=True) == 0
    return q.cpu().numpy(), s.cpu().numpy(), None if st is None else st.cpu().numpy()


def oracle(orc, x, shift, scale, rpg, params, eps=1e-6):
    h, stats = orc.adaln(x, shift, scale, rpg, eps)
    K = orc.expand(params, dtype=orc.F32)
    q, s = oracle_rows("quantize", h, K)
    return q, s, stats


def same_stats(a: np.ndarray, b: np.ndarray) -> bool:
    """Bit-equal, NaN payloads aside."""
    both_nan = np.isnan(a) & np.isnan(b)
    return bool(np.all(both_nan | (a.view(np.uint32) == b.view(np.uint32))))


@pytest.mark.parametrize("d", [3072, 12288])
def test_adaln_flux_every_row(kq, orc, d):
    """FLUX-shaped rows (4608 tokens in two samples of 2304), every row."""
    x, params = inputs.config_case("flux", d)
    shift, scale = modulation(2, d, seed=[d, 1])
    qr, sr, str_ = oracle(orc, x, shift, scale, 2304, params)
    for form in FORMS:
        q, s, st = run(kq, x, shift, scale, 2304, params, form=form)
        assert st is None or same_stats(st, str_), form
        assert np.array_equal(s, sr) and np.array_equal(q, qr), form


@pytest.mark.parametrize("M,d,rpg", [(1, 32, 1), (7, 96, 3), (130, 1152, 64), (33, 2240, 5), (20, 5600, 7),
                                     (9, 16384, 4), (64, 640, 1000)])
def test_adaln_ragged_shapes(kq, orc, M, d, rpg):
    """Widths from one block to the largest supported (512 blocks), column counts that are
    not powers of two, rows that do not fill the last group or the last CTA step."""
    x = inputs.activations(M, d, "t3", seed=[M, d, 2], outlier_frac=0.01, outlier_scale=(20.0, 100.0))
    params = inputs.lu_params(d // 32, seed=[M, d, 3])
    shift, scale = modulation(-(-M // rpg), d, seed=[M, d, 4])
    qr, sr, str_ = oracle(orc, x, shift, scale, rpg, params)
    for form in FORMS:
        q, s, st = run(kq, x, shift, scale, rpg, params, form=form)
        assert st is None or same_stats(st, str_), form
        assert np.array_equal(s, sr) and np.array_equal(q, qr), form


def test_adaln_tiled_scales(kq, orc):
    M, d, rpg = 300, 1152, 128
    x = inputs.activations(M, d, "normal", seed=5, outlier_frac=0.01)
    params = inputs.lu_params(d // 32, seed=6)
    shift, scale = modulation(3, d, seed=7)
    qr, sr, _ = oracle(orc, x, shift, scale, rpg, params)
    for form in FORMS:
        q, s, _ = run(kq, x, shift, scale, rpg, params, layout="mma", form=form)
        assert np.array_equal(q, qr) and np.array_equal(s, tiled_scales(sr)), form


def test_adaln_degenerate_rows(kq, orc):
    """Constant rows (variance 0), all-zero rows, a huge-magnitude row, rows holding inf
    and NaN, a row of signed zeros, and eps = 0 (a constant row then has rstd = inf)."""
    d = 192
    rng = np.random.default_rng(8)
    a = rng.standard_normal((10, d)).astype(np.float32)
    a[0] = 3.0
    a[1] = 0.0
    a[2] *= 1e30
    a[3, 5] = np.inf
    a[4, 7] = np.nan
    a[5] = -0.0
    a[6, ::2] = 1e-30
    x = inputs.f32_to_bf16_bits(a)
    params = inputs.lu_params(d // 32, seed=9)
    shift, scale = modulation(1, d, seed=10)
    for eps in (1e-6, 0.0):
        qr, sr, str_ = oracle(orc, x, shift, scale, 10, params, eps=eps)
        for form in FORMS:
            q, s, st = run(kq, x, shift, scale, 10, params, eps=eps, form=form)
            assert st is None or same_stats(st, str_), (eps, form)
            assert np.array_equal(s, sr) and np.array_equal(q, qr), (eps, form)


def test_adaln_without_stats_and_binding_checks(kq, orc):
    M, d = 16, 256
    x = inputs.activations(M, d, "normal", seed=11, outlier_frac=0.01)
    params = inputs.lu_params(d // 32, seed=12)
    shift, scale = modulation(2, d, seed=13)
    bt = kq.BlockTransform(torch.from_numpy(params).cuda())
    q, s, st = bt.adaln_quantize(dev_bits(x), dev_bits(shift), dev_bits(scale), 8)
    torch.cuda.synchronize()
    assert st is None
    qr, sr, _ = oracle(orc, x, shift, scale, 8, params)
    assert np.array_equal(q.cpu().numpy(), qr) and np.array_equal(s.cpu().numpy(), sr)
    with pytest.raises(ValueError):
        bt.adaln_quantize(dev_bits(x), dev_bits(shift[:1]), dev_bits(scale[:1]), 8)  # one group short
    big = torch.zeros((2, 16416), dtype=torch.bfloat16, device="cuda")  # 513 blocks
    pb = kq.BlockTransform(torch.from_numpy(inputs.lu_params(513, seed=1)).cuda())
    mod = torch.zeros((1, 16416), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kq.KQError):
        pb.adaln_quantize(big, mod, mod, 2)
    assert kq.kq_get_device_error(clear=True) == 0
