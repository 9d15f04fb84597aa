"""The Python binding checks every tensor before a pointer reaches the C ABI:
CUDA residency, the input's device, dtype, contiguity, shape and size.  Each
case must raise and must not call into the library (a stub library that fails
on any call stands in for it)."""
from __future__ import annotations

import pytest

torch = pytest.importorskip("torch")


class _NoCalls:
    def __getattr__(self, name):
        raise AssertionError(f"the binding called {name} for an argument it should have rejected")


@pytest.fixture
def kq(monkeypatch):
    import mxfp4_activations_b200 as m
    from mxfp4_activations_b200 import _lib

    monkeypatch.setattr(_lib, "_lib", _NoCalls())
    return m


def test_host_tensors_are_rejected(kq):
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    mats = torch.zeros((2, 32, 32))
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_quantize(x, mats)
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_ref_smooth_quantize(x, torch.ones(64))
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_ref_fwht_quantize(x)
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_dequantize(torch.zeros((4, 32), dtype=torch.uint8), torch.zeros((4, 2), dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_expand_blocks(torch.zeros((2, 5, 3)))
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_expand_factored(torch.zeros((2, 5, 3)))
    with pytest.raises(ValueError, match="CUDA"):
        kq.kq_e2m1_pack(torch.zeros(8))
    with pytest.raises((TypeError, ValueError)):
        kq.kq_quantize(x.float(), mats)


@pytest.mark.parametrize("case", ["mats_small", "mats_cpu", "mats_transposed", "mats_dtype", "fac_small",
                                  "fac_cpu", "q_small", "q_noncontig", "q_dtype", "scales_small",
                                  "scales_cpu", "variant", "layout"])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_quantize_rejects_bad_tensors(kq, case):
    M, d = 8, 128
    x = torch.zeros((M, d), dtype=torch.bfloat16, device="cuda")
    mats = torch.zeros((d // 32, 32, 32), device="cuda")
    fac = torch.zeros((d // 32, 48), device="cuda")
    q = torch.empty((M, d // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((M, d // 32), dtype=torch.uint8, device="cuda")
    kw = dict(variant="butterfly", scale_layout="row")
    if case == "mats_small":
        mats = mats[:2]
    elif case == "mats_cpu":
        mats = mats.cpu()
    elif case == "mats_transposed":
        mats = mats.transpose(1, 2)
    elif case == "mats_dtype":
        mats = mats.double()
    elif case == "fac_small":
        fac = fac[:3]
    elif case == "fac_cpu":
        fac = fac.cpu()
    elif case == "q_small":
        q = q[: M - 1]
    elif case == "q_noncontig":
        q = torch.empty((M, d), dtype=torch.uint8, device="cuda")[:, ::2]
    elif case == "q_dtype":
        q = q.view(torch.int8)
    elif case == "scales_small":
        s = s.flatten()[:-1]
    elif case == "scales_cpu":
        s = s.cpu()
    elif case == "variant":
        kw["variant"] = "fast"
    elif case == "layout":
        kw["scale_layout"] = "tiles"
    with pytest.raises((ValueError, TypeError)):
        kq.kq_quantize(x, mats, fac, q=q, scales=s, **kw)


@pytest.mark.parametrize("case", ["inv_s_small", "inv_s_cpu", "inv_s_dtype"])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_smooth_rejects_bad_scaling_vector(kq, case):
    x = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    inv_s = torch.ones(128, device="cuda")
    inv_s = {"inv_s_small": inv_s[:100], "inv_s_cpu": inv_s.cpu(), "inv_s_dtype": inv_s.half()}[case]
    with pytest.raises((ValueError, TypeError)):
        kq.kq_ref_smooth_quantize(x, inv_s)


@pytest.mark.parametrize("case", ["tiled_scales", "scales_short", "q_noncontig", "inv_small", "inv_64",
                                  "out_small", "out_cpu"])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_dequantize_rejects_bad_tensors(kq, case):
    from mxfp4_activations_b200 import scale_bytes

    M, d = 8, 128
    q = torch.zeros((M, d // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((M, d // 32), dtype=torch.uint8, device="cuda")
    inv = None
    out = None
    if case == "tiled_scales":
        s = torch.zeros(scale_bytes(M, d, "mma"), dtype=torch.uint8, device="cuda")
    elif case == "scales_short":
        s = s[: M - 1]
    elif case == "q_noncontig":
        q = torch.zeros((M, d), dtype=torch.uint8, device="cuda")[:, ::2]
    elif case == "inv_small":
        inv = torch.zeros((1, 32, 32), device="cuda")
    elif case == "inv_64":
        inv = torch.zeros((d // 64, 64, 64), device="cuda")
    elif case == "out_small":
        out = torch.empty((M - 1, d), device="cuda")
    elif case == "out_cpu":
        out = torch.empty((M, d))
    with pytest.raises((ValueError, TypeError)):
        kq.kq_dequantize(q, s, inv, out=out)
