/*
 * kq_oracle.h -- CPU oracle of the KroQuant online activation quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, scalar restatement of what
 * the method computes, in fp64, written from the method's description.  Only
 * the tests, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
 * arm may load it.  The product library (include/kq.h) never includes, links or
 * calls anything here, and nothing here includes the product's headers.
 *
 * Sources (cited by page title and section):
 *   [KQ-sum]  "KroQuant: Kronecker-Structured Block Transforms for Efficient
 *             Post-Training Quantization of Diffusion Transformers", research-map
 *             summary page: "Approach", "Key results", "Limitations".
 *   [KQ-abs]  the KroQuant abstract (reprinted on two paper-listing pages).
 *   [LRQ]     "LRQ-DiT: Log-Rotation Post-Training Quantization of Diffusion
 *             Transformers", Sec. 3.2 (eq. 2, eq. 3) and Sec. 4.3 (Lemma 1).
 *   The pages name the element format only as "W4A4 MXFP4" / "MXFP4e2"; the
 *   E2M1 value grid and the E8M0 shared-scale rule are taken from the public
 *   OCP Microscaling (MX) v1.0 format definition, the plainest reading.
 *
 * Conventions (readings where the pages are silent):
 *   - params[b][k] = (l, u, v) for factor k = 0..4 of block b;
 *     F_k = L U, L = [[1,0],[l,1]], U = [[u,v],[0,1/u]]  (det F_k = 1).
 *   - K_b = F_0 (x) F_1 (x) F_2 (x) F_3 (x) F_4; F_0 acts on the most
 *     significant bit of the 5-bit index inside the 32-element block.
 *   - Row-vector form y = x K (as in eq. 2, X H).
 *   - Scale: e = floor(log2(amax)) - 2 clamped to [-127, 127], byte e + 127;
 *     amax == 0 gives byte 0; a non-finite y in the block gives byte 0xFF and
 *     all-zero codes.
 *   - Element: round v = y * 2^-e to the E2M1 grid, ties to the even code,
 *     |v| > 6 saturates to 6, sign kept (a negative value that rounds to zero
 *     gives code 0x8).  Byte k of a row holds element 2k in its low nibble.
 */
#ifndef KQ_ORACLE_H
#define KQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { KQO_F32 = 0, KQO_BF16 = 1 };

/* 2x2 factor F = L U from (l, u, v); F row-major [a b; c d]. */
void kqo_factor(float l, float u, float v, double F[4]);
/* Its inverse U^-1 L^-1, formed as a product of the two triangular inverses. */
void kqo_factor_inverse(float l, float u, float v, double Finv[4]);
/* Kronecker product: A is na x na, B is nb x nb, out is (na nb) x (na nb). */
void kqo_kron(const double* A, int na, const double* B, int nbd, double* out);
/* K_b (or K_b^-1) for nb blocks, fp64, [nb][32][32]. */
void kqo_expand_f64(const float* params, int64_t nb, int inverse, double* K);
/* Same, rounded once to fp32 (dtype KQO_F32, float out) or bf16 (uint16 out). */
void kqo_expand(const float* params, int64_t nb, int inverse, int dtype, void* out);
/* Round-to-nearest-even of a double to bf16 bits. */
uint16_t kqo_bf16_from_f64(double a);
/* Normalised Sylvester Hadamard of order 2^n (eq. 3), fp64, row-major. */
void kqo_hadamard(int n, double* H);

/* E8M0 shared-scale byte for a block whose largest magnitude is amax. */
int kqo_e8m0(float amax);
/* kqo_e8m0 over an array. */
void kqo_e8m0_many(const float* amax, int64_t n, uint8_t* out);
/* E2M1 code (0..15) of an already scaled fp32 value v (v must not be NaN). */
int kqo_e2m1(float v);
/* Value of an E2M1 code. */
double kqo_e2m1_value(int code);
/* out[k] = code(v[2k]) | code(v[2k+1]) << 4, n even. */
void kqo_e2m1_pack(const float* v, int64_t n, uint8_t* out);

/* y[r][j] = fp32( sum_i x[r][32b+i] * K_b[i][j] ), fp64 accumulation in
 * index order from +0.  x is bf16 bits [M][ldx]; mats are the block matrices in
 * dtype (float or bf16 bits) [nb][32][32]; y is [M][d]. */
void kqo_transform(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                   const void* mats, int dtype, float* y);
/* MXFP4 of already transformed rows y [M][d]: codes q [M][d/2], scales [M][d/32]. */
void kqo_mx_quantize(const float* y, int64_t M, int64_t d, uint8_t* q, uint8_t* scales);
/* Full quantizer: transform then MXFP4. */
void kqo_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                  const void* mats, int dtype, uint8_t* q, uint8_t* scales);
/* Comparison point 1: per-channel scaling, y_j = fp32(x_j * inv_s_j), then MXFP4. */
void kqo_smooth_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                         const float* inv_s, uint8_t* q, uint8_t* scales);
/* Comparison point 2: fixed 32-point normalised Hadamard (K = fp32(H_32)), then MXFP4. */
void kqo_fwht_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                       uint8_t* q, uint8_t* scales);
/* Dequantize: yhat = value(code) * 2^(byte-127); if inv_mats != NULL also
 * xhat = yhat K^-1 per block (fp64).  out is fp64 [M][d]. */
void kqo_dequantize(const uint8_t* q, const uint8_t* scales, int64_t M, int64_t d,
                    const void* inv_mats, int dtype, double* out);

/* ---- transform blocks of n = 2^log2n elements (log2n in 4..7), MXFP4 still per 32
 *
 * [KQ-sum, Limitations]: the Kronecker parametrization has 3 log2(n) parameters
 * per block of n elements.  K_c = F_0 (x) ... (x) F_{log2n-1} (F_0 on the most
 * significant index bit) acts on elements [c n, c n + n) of a row; params are
 * [nt][log2n][3].  The MX scale blocks stay 32 elements long. */
/* K_c (or K_c^-1) in fp64, [nt][n][n]. */
void kqo_expand_n_f64(const float* params, int64_t nt, int log2n, int inverse, double* K);
/* Same, rounded once to fp32 (float out) or bf16 (uint16 out). */
void kqo_expand_n(const float* params, int64_t nt, int log2n, int inverse, int dtype, void* out);
/* y[r][c n + j] = fp32( sum_i x[r][c n + i] K_c[i][j] ), fp64 accumulation in
 * index order from +0; d % n == 0. */
void kqo_transform_n(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const void* mats, int dtype,
                     int n, float* y);
/* transform_n, then MXFP4 per 32 elements. */
void kqo_quantize_n(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const void* mats, int dtype,
                    int n, uint8_t* q, uint8_t* scales);

/* ---- the producer: AdaLN normalisation fused in front of the quantizer
 *
 * [KQ §Problem] (AdaLN blocks keep the transform from being absorbed offline) and
 * [KQ abstract] (normalisation layers between blocks force the transform to run
 * online).  The pages do not define the normalisation; this is the DiT block's
 * modulated LayerNorm without a learned affine, computed in fp32 as DiT models do,
 * with every step fixed so that it is reproducible bit for bit (every operation one
 * IEEE binary32 operation, rounded to nearest even; sqrt and division correctly
 * rounded):
 *   S1  = pairwise sum of the row's d inputs (pad with +0 to a power of two, then add
 *         neighbours level by level: a'_j = a_2j + a_2j+1)
 *   mu  = S1 / d
 *   t_i = x_i - mu;  S2 = pairwise sum of t_i * t_i;  var = S2 / d
 *   rstd = 1 / sqrt(var + eps)
 *   h_i = bf16( ((t_i * rstd) * (1 + scale[g][i])) + shift[g][i] ),  g = row / rows_per_group
 * shift, scale: bf16 [G][d]; h: bf16 bits [M][d]; stats: fp32 [M][2] (mu, rstd) or NULL. */
void kqo_adaln(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const uint16_t* shift,
               const uint16_t* scale, int64_t rows_per_group, float eps, uint16_t* h, float* stats);
/* kqo_adaln, then kqo_quantize of h with the block matrices. */
void kqo_adaln_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const uint16_t* shift,
                        const uint16_t* scale, int64_t rows_per_group, float eps, const void* mats,
                        int dtype, uint8_t* q, uint8_t* scales, float* stats);

/* ---- the consumer: W4A4 product of two MXFP4 operands
 *
 * [KQ-sum, Approach] and [KQ-abs] ("W4A4 (MXFP4e2)"): activations quantized with
 * K_b, weights with K_b^-T, so the layer's product is taken between the two MXFP4
 * tensors.  c[m][n] = sum_k A(m,k) B(n,k) in fp64 with
 * A(m,k) = value(code of a_q[m], element k) * 2^(a_scales[m][k/32] - 127) and B alike;
 * a scale byte 0xFF makes its values NaN.  Codes [rows][K/2] (element 2j in the low
 * nibble of byte j), scales row-major [rows][K/32], c fp64 [M][N]. */
void kqo_mx_gemm(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                 const uint8_t* b_scales, int64_t N, int64_t K, double* c);

#ifdef __cplusplus
}
#endif
#endif
