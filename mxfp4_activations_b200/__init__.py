"""B200-native (sm_100a) KroQuant online activation quantizer.

Every 32-element block of a bf16 activation row is multiplied by its own
Kronecker-structured 32x32 transform (five 2x2 unit-determinant LU factors,
15 parameters per block) and quantized to MXFP4 (E2M1 codes + one E8M0 scale
per block), as described on the "KroQuant: Kronecker-Structured Block
Transforms for Efficient Post-Training Quantization of Diffusion Transformers"
pages.  The work is done by libkq.so (include/kq.h); this package is its
thin ctypes binding plus seeded input generators (``inputs``).
"""
from ._lib import (  # noqa: F401
    EXPORTED,
    kq_adaln_quantize,
    SCALE_LAYOUTS,
    KQError,
    kq_abi_version,
    kq_dequantize,
    kq_e2m1_pack,
    kq_expand_blocks,
    kq_expand_factored,
    kq_gemm_kernel,
    kq_gemm_mxf4,
    kq_get_device_error,
    kq_quantize,
    kq_ref_fwht_quantize,
    kq_ref_smooth_quantize,
    kq_select_variant,
    kq_status_string,
    load,
    scale_bytes,
)


class BlockTransform:
    """The per-layer set-up of one KroQuant transform: the LU parameters
    [d/n, log2 n, 3] (n = 32: five factors per block; n = 64: six) expanded once into
    the dense block matrices, their inverses and the butterfly (factored) form, then
    reused for every call."""

    def __init__(self, params):
        self.params = params.contiguous()
        self.mats = kq_expand_blocks(self.params)
        self.factored = kq_expand_factored(self.params)
        self._inv = None

    @property
    def inverse_mats(self):
        if self._inv is None:
            self._inv = kq_expand_blocks(self.params, inverse=True)
        return self._inv

    def quantize(self, x, variant: str = "auto", q=None, scales=None, scale_layout: str = "row"):
        return kq_quantize(x, self.mats, self.factored, variant=variant, q=q, scales=scales,
                           scale_layout=scale_layout)

    def quantize_weights(self, w, mat_dtype=None, q=None, scales=None, scale_layout: str = "row"):
        """MXFP4 of the weight rows w [n_out, d] (bf16) times K_b^-T per block, the
        weight side of the transform: dot products with quantize(x) rows then
        approximate x . w.  Runs the tensor-core variant with the dense K^-T."""
        import torch

        if self.mats.shape[-1] != 32:
            raise NotImplementedError("the weight side is provided for 32-element transform blocks")
        key = mat_dtype or torch.float32
        if getattr(self, "_inv_t", None) is None or self._inv_t.dtype != key:
            self._inv_t = kq_expand_blocks(self.params, inverse=True, transpose=True, dtype=key)
        return kq_quantize(w, self._inv_t, None, variant="mma", q=q, scales=scales, scale_layout=scale_layout)

    def adaln_quantize(self, x, shift, scale, rows_per_group: int, eps: float = 1e-6, q=None, scales=None,
                       scale_layout: str = "row", stats=None):
        """The DiT block's modulated LayerNorm fused in front of the quantizer: MXFP4 of
        bf16(LN(x) (1 + scale[g]) + shift[g]) K_b, g = row // rows_per_group."""
        if self.mats.shape[-1] != 32:
            raise NotImplementedError("the fused AdaLN quantizer is provided for 32-element transform blocks")
        return kq_adaln_quantize(x, shift, scale, rows_per_group, self.mats, self.factored, eps=eps, q=q,
                                 scales=scales, scale_layout=scale_layout, stats=stats)

    def dequantize(self, q, scales, undo_transform: bool = True, out_dtype=None):
        import torch

        return kq_dequantize(q, scales, self.inverse_mats if undo_transform else None,
                             out_dtype=out_dtype or torch.float32)
