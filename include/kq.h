/*
 * kq.h -- C ABI of the B200 (sm_100a) KroQuant online activation quantizer.
 *
 * The method (cited by page title and section):
 *   [KQ-sum] "KroQuant: Kronecker-Structured Block Transforms for Efficient
 *            Post-Training Quantization of Diffusion Transformers", research-map
 *            summary page, sections "Approach", "Key results", "Limitations".
 *   [KQ-abs] the KroQuant abstract (reprinted on two paper-listing pages).
 *   [LRQ]    "LRQ-DiT: Log-Rotation Post-Training Quantization of Diffusion
 *            Transformers", Sec. 3.2 eq. (2)-(3).
 * Every 32-element block of a bf16 activation row is multiplied by its own
 * learned invertible 32x32 matrix K_b = F0 (x) F1 (x) F2 (x) F3 (x) F4, each F_k a
 * 2x2 unit-determinant LU factor (15 parameters per block) [KQ-sum, Approach],
 * and the result is quantized to MXFP4 ("W4A4 (MXFP4e2)" [KQ-abs]): E2M1
 * codes plus one E8M0 scale per 32 elements.
 *
 * Conventions fixed by this library (readings where the pages are silent):
 *   params  fp32 [nb][5][3]: (l, u, v) of factor k; F_k = L U with
 *           L = [[1,0],[l,1]], U = [[u,v],[0,1/u]]; F0 acts on the most
 *           significant bit of the index inside the block.
 *   y = x K (row vector, as X H in [LRQ] eq. 2); y_j is the fp32 rounding of the
 *           exact sum over the block, K being the matrices given to kq_quantize.
 *   scale   e = floor(log2 max|y|) - 2 clamped to [-127,127]; byte e + 127;
 *           a block with max|y| = 0 has byte 0; a block holding a non-finite y
 *           has byte 0xFF and zero codes.
 *   codes   v = y 2^-e rounded to E2M1 (nearest, ties to even code, saturating
 *           at 6, sign kept: a negative v that rounds to 0 gives code 0x8);
 *           byte k of a row holds element 2k in its low nibble.
 *
 * Ownership: the caller owns every buffer (device memory unless stated).  No
 * entry point allocates or frees memory, and none but kq_get_device_error
 * synchronises; all device work is enqueued on the given stream.  Argument errors are returned before anything is launched.
 * A launch failure returns KQ_ERR_CUDA.  Kernels that wait on asynchronous
 * copies bound every wait; a wait that runs out records a flag that
 * kq_get_device_error() reports.
 */
#ifndef KQ_H
#define KQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KQ_API __attribute__((visibility("default")))
#else
#define KQ_API
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* kq_stream_t;

typedef enum {
  KQ_OK = 0,
  KQ_ERR_INVALID_ARG = 1, /* NULL pointer where one is required, bad enum, negative size */
  KQ_ERR_SHAPE = 2,       /* d not a multiple of 32, ldx < d, odd n, size overflow      */
  KQ_ERR_ALIGN = 3,       /* a pointer or a row stride breaks the alignment stated below */
  KQ_ERR_SINGULAR = 4,    /* a factor had u == 0 (reported by kq_get_device_error)      */
  KQ_ERR_UNSUPPORTED = 5, /* variant / dtype combination not provided                   */
  KQ_ERR_CUDA = 6,        /* a CUDA call failed (launch, attribute, tensor map)         */
  KQ_ERR_DEVICE_TIMEOUT = 7 /* a kernel gave up a bounded wait (kq_get_device_error)    */
} kq_status;

typedef enum { KQ_F32 = 0, KQ_BF16 = 1 } kq_dtype;

/* Which kernel computes the block transform inside kq_quantize.
 *   KQ_VAR_BUTTERFLY: 5-stage 2x2 butterfly over registers (needs KQ_F32
 *                     matrices and the factored form from kq_expand_factored).
 *   KQ_VAR_MMA:       tensor-core product with the dense block matrix.
 *   KQ_VAR_AUTO:      the faster provided variant for the shape and dtype: bf16
 *                     matrices, or fp32 without the factored form, take the
 *                     tensor core; fp32 with the factored form takes the winner
 *                     measured at the nearest shape of the library's sweep table
 *                     (log2 M, log2 d), unless the environment variable
 *                     KQ_VARIANT=mma|butterfly (read once per process) names one.
 *                     kq_select_variant reports the choice. */
typedef enum { KQ_VAR_AUTO = 0, KQ_VAR_MMA = 1, KQ_VAR_BUTTERFLY = 2 } kq_variant;

/* Where kq_quantize writes the E8M0 scales.
 *   KQ_SCALES_ROW_MAJOR: [M][d/32], scale of block b of row r at byte r*(d/32) + b.
 *   KQ_SCALES_MMA_TILED: the layout that block-scaled tensor-core GEMMs read their
 *     per-32-element scale factors in (tcgen05.mma kind::mxf4, cuBLASLt VEC32_UE8M0
 *     scales).  The [M][d/32] scale matrix is padded to multiples of 128 rows and
 *     4 columns and cut into 128x4 tiles of 512 bytes, stored tile row by tile row:
 *     tile (R, C) starts at byte (R * ceil(d/128) + C) * 512, and inside it the scale
 *     of row r and column c (r < 128, c < 4) sits at byte 16*(r % 32) + 4*(r / 32) + c.
 *     The buffer holds ceil(M/128)*128 * ceil(d/128)*4 bytes; padding bytes are not
 *     written. */
typedef enum { KQ_SCALES_ROW_MAJOR = 0, KQ_SCALES_MMA_TILED = 1 } kq_scale_layout;

#define KQ_BLOCK 32          /* elements per block / per E8M0 scale                */
#define KQ_NFACTORS 5        /* 2x2 factors per block                              */
#define KQ_PARAMS_PER_BLOCK 15
#define KQ_FACTORED_FLOATS 48 /* floats per block in the factored form            */

/* ---------------------------------------------------------------- set-up (once per layer)
 *
 * kq_expand_blocks -- [KQ-sum, Approach]: K_b = F0 (x) F1 (x) F2 (x) F3 (x) F4
 * from the 15 LU parameters of each block.
 *   inverse 0: K_b.
 *           1: K_b^-1 = F0^-1 (x) ... (x) F4^-1 (det F_k = 1, so F^-1 = [[d,-b],[-c,a]]).
 *           2: (K_b^-1)^T, the weight-side transform: quantizing each weight row w
 *              with it ([KQ-abs] "its inverse to the weights") keeps products
 *              invariant, (x K_b) . (w K_b^-T) = x . w ([LRQ] eq. 2).
 *           any other value: KQ_ERR_INVALID_ARG.
 *   params  device fp32 [nb][5][3], 4-byte aligned.
 *   nb      number of blocks (>= 0; 0 is a no-op).
 *   mats    device [nb][32][32] row-major (row = input index i, column = output
 *           index j, so y_j = sum_i x_i mats[i][j]); fp32 (KQ_F32) or bf16 bits
 *           (KQ_BF16), 4-byte aligned.  Every entry is computed in fp64 and
 *           rounded once (to nearest even) to out_dtype.
 * A factor with u == 0 yields non-finite entries and sets the device flag
 * read by kq_get_device_error() (KQ_ERR_SINGULAR).
 */
KQ_API kq_status kq_expand_blocks(const float* params, int64_t nb, int inverse, kq_dtype out_dtype,
                           void* mats, kq_stream_t stream);

/* kq_expand_blocks_n -- the same for transform blocks of n = 2^log2n elements
 * ([KQ-sum, Limitations]: 3 log2(n) parameters per block; log2n in 1..7):
 * K_c = F0 (x) ... (x) F_{log2n-1}, F0 on the most significant index bit.
 *   params  device fp32 [nt][log2n][3];  mats device [nt][n][n] in out_dtype.
 *   inverse as for kq_expand_blocks (0: K, 1: K^-1, 2: K^-T).
 * kq_expand_blocks(p, nb, ...) is kq_expand_blocks_n(p, nb, 5, ...).
 */
KQ_API kq_status kq_expand_blocks_n(const float* params, int64_t nt, int log2n, int inverse, kq_dtype out_dtype,
                             void* mats, kq_stream_t stream);

/* kq_expand_factored -- the same K_b in the form the butterfly kernel applies:
 * F_k = M_k diag(a_k, d_k) with M_k = [[1, b_k/d_k],[c_k/a_k, 1]], so that
 * K_b = (M_0 (x) ... (x) M_4) D_b with D_b = diag_j prod_k (a_k or d_k).
 *   factored  device fp32 [nb][48], 16-byte aligned:
 *             [0..4]  c_k/a_k   [5..9] b_k/d_k   [10..41] D_b[j]
 *             [42]    max_ij |K_b[i][j]| rounded up   [43] 1.0 when the block
 *             must use the exact fp64 path (some d_k == 0 or a ratio overflows)
 *             [44]    absolute error allowance for fp32-subnormal results
 *             [45..47] zero.  Coefficients are fp64 values rounded once.
 */
KQ_API kq_status kq_expand_factored(const float* params, int64_t nb, float* factored, kq_stream_t stream);

/* kq_expand_factored_n -- the butterfly form for transform blocks of n = 2^log2n
 * elements, log2n 4..7 ([KQ-sum, Limitations]), one record per 32-element block
 * column, factored 16-byte aligned:
 *   log2n 5..7: nt * n / 32 records of [48] floats: the five factors acting inside
 *     the 32-element block in [0..9] as above (factors log2n-5 .. log2n-1), this
 *     block's 32 entries of D in [10..41], max|K| bound, exact-only flag and absolute
 *     allowance in [42..44];
 *     log2n 6: c/a, b/d of F0 (it mixes the two 32-element halves) in [45], [46];
 *     log2n 7: [45] the coefficient of F1 (index bit 5) that this column applies
 *       (c/a if it is the lower column of its pair, else b/d), [46] the same for F0
 *       (index bit 6) and the column's 64-element half.
 *   log2n 4: nt / 2 records of [64] floats (nt even; a 32-element column holds two
 *     16-element blocks h = 0, 1): [8h .. 8h+3] c/a and [8h+4 .. 8h+7] b/d of factors
 *     0..3 of block h, [16..47] D for the 32 outputs, [48] max|K| bound over both
 *     blocks, [49] exact-only flag, [50] absolute allowance, [51..63] zero.
 * log2n outside 4..7: KQ_ERR_INVALID_ARG; odd nt with log2n 4: KQ_ERR_SHAPE.
 * kq_expand_factored(p, nb, ...) is kq_expand_factored_n(p, nb, 5, ...).
 */
KQ_API kq_status kq_expand_factored_n(const float* params, int64_t nt, int log2n, float* factored,
                               kq_stream_t stream);

/* ---------------------------------------------------------------- hot path
 *
 * kq_quantize -- [KQ-abs]: each 32-element block goes through its own
 * transform, then MXFP4 ("W4A4 (MXFP4e2)"): y = x K_b, one E8M0 scale and 32
 * E2M1 codes per block, in one pass over x.
 *   x        device bf16 bits [M][ldx]; 16-byte aligned; ldx % 8 == 0; ldx >= d.
 *   M        rows (tokens) >= 0 (0 is a no-op);  d = channels, d % 32 == 0.
 *   mats     device [d/32][32][32] from kq_expand_blocks in mat_dtype.  The
 *            output is defined by these matrices (see the header comment).
 *   factored device [d/32][48] from kq_expand_factored for the same params, or
 *            NULL; required by KQ_VAR_BUTTERFLY.
 *   q        device [M][d/2] packed E2M1 codes, 16-byte aligned.
 *   scales   device E8M0 bytes in scale_layout (see kq_scale_layout for sizes).
 *   variant  which kernel computes the transform (kq_variant).
 *   scale_layout  KQ_SCALES_ROW_MAJOR or KQ_SCALES_MMA_TILED; anything else is
 *            KQ_ERR_INVALID_ARG.
 * Both variants compute y in fp32, bound its rounding error from the block's L1
 * norm and max|K_b| (the butterfly by a proof, the tensor core by a calibrated
 * allowance), and recompute in fp64 (summing in increasing i) exactly those
 * scales and codes that the bound cannot certify, so the output equals the fp64
 * definition.
 */
KQ_API kq_status kq_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const void* mats,
                      kq_dtype mat_dtype, const float* factored, uint8_t* q, uint8_t* scales,
                      kq_variant variant, kq_scale_layout scale_layout, kq_stream_t stream);

/* kq_quantize_n -- the same with transform blocks of n = 2^log2n elements, log2n 4..7
 * ([KQ-sum, Limitations]: 3 log2(n) parameters per block); the MX scale blocks stay
 * 32 elements long.
 *   log2n 5: exactly kq_quantize.
 *   log2n 4, 6, 7: d % max(32, n) == 0 (else KQ_ERR_SHAPE); mats fp32 [d/n][n][n]
 *            from kq_expand_blocks_n and factored from kq_expand_factored_n with the
 *            same params are both required; only the butterfly serves them
 *            (KQ_VAR_MMA or bf16 matrices: KQ_ERR_UNSUPPORTED).  y_j = fp32(sum over
 *            the n inputs of the block), certified and recomputed exactly like
 *            kq_quantize.
 *   log2n other: KQ_ERR_INVALID_ARG.
 */
KQ_API kq_status kq_quantize_n(const void* x, int64_t M, int64_t d, int64_t ldx, int log2n, const void* mats,
                        kq_dtype mat_dtype, const float* factored, uint8_t* q, uint8_t* scales,
                        kq_variant variant, kq_scale_layout scale_layout, kq_stream_t stream);

/* kq_dequantize -- inverse of the MXFP4 step [KQ-abs]: yhat_j = E2M1(code_j) *
 * 2^(byte-127) (byte 0xFF gives NaN), and, when inv_mats != NULL, the block
 * transform is undone, xhat = yhat K_b^-1 (the activation side of [LRQ] eq. 2).
 *   q, scales  device, as produced by kq_quantize ([M][d/2], [M][d/32]); q 16-byte aligned.
 *   inv_mats   device [d/32][32][32] in mat_dtype (kq_expand_blocks, inverse=1) or NULL.
 *   out        device [M][d] in out_dtype (fp32 or bf16 bits), 16-byte aligned.
 * Without inv_mats the fp32 result is exact; with it, the fp32 sum has the
 * rounding error of 32 fused multiply-adds.
 */
KQ_API kq_status kq_dequantize(const uint8_t* q, const uint8_t* scales, int64_t M, int64_t d,
                        const void* inv_mats, kq_dtype mat_dtype, void* out, kq_dtype out_dtype,
                        kq_stream_t stream);

/* ---------------------------------------------------------------- producer
 *
 * kq_adaln_quantize -- the quantizer fused with the AdaLN normalisation in front of it
 * ([KQ-sum, Problem]: AdaLN blocks keep the transform from being absorbed offline;
 * [KQ-abs]: normalisation layers between blocks force it to run online).  The pages do
 * not define the normalisation; this library takes the DiT block's modulated LayerNorm
 * without a learned affine, in fp32 as DiT models compute it, every step one IEEE binary32
 * operation rounded to nearest even (sqrt and division correctly rounded):
 *   S1 = pairwise sum of the row's d inputs (padded with +0 to a power of two, then
 *        neighbours added level by level), mu = S1 / d,
 *   S2 = pairwise sum of (x_i - mu)^2, var = S2 / d, rstd = 1 / sqrt(var + eps),
 *   h_i = bf16( ((x_i - mu) * rstd) * (1 + scale[g][i]) + shift[g][i] ),  g = row / rows_per_group,
 * then q, scales = kq_quantize of h with the butterfly variant (h never reaches memory).
 *   x             device bf16 [M][ldx], as kq_quantize (16-byte aligned, ldx % 8 == 0).
 *   shift, scale  device bf16 bits [ceil(M / rows_per_group)][d], 16-byte aligned.
 *   rows_per_group  rows that share one pair of modulation vectors (tokens per sample), >= 1.
 *   eps           added to the variance (any float).
 *   mats, factored  fp32 [d/32][32][32] and [d/32][48], as kq_quantize's butterfly variant.
 *   q, scales, scale_layout  as kq_quantize.
 *   stats         device fp32 [M][2]: (mu, rstd) of each row, or NULL; 8-byte aligned.
 * With stats, two kernels run on the stream: a statistics pass writes (mu, rstd) of every
 * row into stats, then the butterfly quantizer forms h from x, stats and the modulation
 * vectors inside its row loop (the faster form).  With stats NULL, one fused kernel
 * computes the statistics and quantizes; no memory beyond the outputs is used either way.
 * d must be a multiple of 32 and at most 16384 (KQ_ERR_UNSUPPORTED above).  Codes, scales
 * and statistics equal the definition bit for bit in both forms. */
KQ_API kq_status kq_adaln_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const void* shift,
                                   const void* scale, int64_t rows_per_group, float eps, const float* mats,
                                   const float* factored, uint8_t* q, uint8_t* scales, kq_scale_layout scale_layout,
                                   float* stats, kq_stream_t stream);

/* ---------------------------------------------------------------- consumer
 *
 * kq_gemm_mxf4 -- the W4A4 product the quantizer feeds [KQ-sum, Approach; KQ-abs,
 * "W4A4 (MXFP4e2)"]: activations quantized with K_b and weights with K_b^-T, so
 *   C[m][n] = sum_k A(m,k) B(n,k),  A(m,k) = E2M1(a_q code) * 2^(a_scale byte - 127),
 *                                   B(n,k) = E2M1(b_q code) * 2^(b_scale byte - 127),
 * computed on the tensor cores (tcgen05.mma kind::mxf4, block scales of 32
 * elements) with fp32 accumulation, then rounded to c_dtype.
 *   a_q       device [M][K/2] codes as written by kq_quantize (x rows), 16-byte aligned.
 *   a_scales  device, KQ_SCALES_MMA_TILED layout for M rows and K/32 blocks, 16-byte
 *             aligned; its padding bytes are never used.
 *   b_q       device [N][K/2] codes of the weight rows (BlockTransform.quantize_weights).
 *   b_scales  device, KQ_SCALES_MMA_TILED layout for N rows, 16-byte aligned.
 *   c         device [M][ldc] fp32 (KQ_F32) or bf16 bits (KQ_BF16), element aligned;
 *             ldc >= N.  Only columns < N are written.
 * K must be a positive multiple of 32 (KQ_ERR_SHAPE otherwise); M or N = 0 is a
 * no-op.  A block whose scale byte is 0xFF (non-finite input) yields NaN in the rows
 * or columns it touches.  The sum of each 64-element step is formed by the tensor
 * core and added to an fp32 accumulator; the result is within the fp32 rounding of
 * K/64 such additions of the exact product.  Bounded waits (kq_get_device_error). */
KQ_API kq_status kq_gemm_mxf4(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                              const uint8_t* b_scales, int64_t N, int64_t K, void* c, int64_t ldc, kq_dtype c_dtype,
                              kq_stream_t stream);

/* kq_select_gemm_kernel -- which kernel kq_gemm_mxf4 runs for M x N x K on the current
 * device, without launching: *two_sm = 1 for the persistent two-SM kernel (tcgen05
 * cta_group::2, 256 x 256 tiles; needs K % 128 == 0 and at least one tile per SM
 * pair), 0 for the one-SM kernel (128 x 128 tiles).  The environment variable
 * KQ_GEMM=1sm|2sm (read once per process) overrides the choice where both apply.
 * KQ_ERR_INVALID_ARG for a NULL two_sm or a negative size, KQ_ERR_SHAPE for
 * K % 32 != 0, KQ_ERR_CUDA without a device. */
KQ_API kq_status kq_select_gemm_kernel(int64_t M, int64_t N, int64_t K, int* two_sm);

/* ---------------------------------------------------------------- comparison points
 *
 * kq_ref_smooth_quantize -- per-channel scaling (SmoothQuant) then MXFP4, the
 * cheaper comparison kernel of [KQ-sum, Key results] and [KQ-abs]:
 * y_j = fp32(x_j * inv_s[j]).  Same layouts and alignment as kq_quantize;
 * inv_s is device fp32 [d], 16-byte aligned.
 */
KQ_API kq_status kq_ref_smooth_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const float* inv_s,
                                 uint8_t* q, uint8_t* scales, kq_stream_t stream);

/* kq_ref_fwht_quantize -- fixed 32-point Hadamard then MXFP4, the FWHT
 * comparison point of [KQ-sum, Key results]: every block is multiplied by the
 * normalised Sylvester matrix H_32 of [LRQ] eq. 3 rounded to fp32, with the same
 * exactness guarantee as the butterfly variant of kq_quantize. */
KQ_API kq_status kq_ref_fwht_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, uint8_t* q,
                               uint8_t* scales, kq_stream_t stream);

/* kq_e2m1_pack -- the element step of MXFP4 alone: out[k] = code(v[2k]) |
 * code(v[2k+1]) << 4 for already scaled fp32 values (same rounding as
 * kq_quantize).  v device fp32 [n], out device [n/2]; n even. */
KQ_API kq_status kq_e2m1_pack(const float* v, int64_t n, uint8_t* out, kq_stream_t stream);

/* kq_select_variant -- the kernel kq_quantize_n(x, M, d, ..., log2n, ..., mat_dtype,
 * factored, ..., KQ_VAR_AUTO, ...) runs for these sizes, without launching
 * anything: *chosen = KQ_VAR_MMA or KQ_VAR_BUTTERFLY.  has_factored != 0 when the
 * factored form will be passed.  KQ_ERR_INVALID_ARG for a NULL chosen, a negative
 * size, a bad dtype or log2n outside 4..7; KQ_ERR_UNSUPPORTED when no variant
 * serves the combination (16-, 64- and 128-element blocks need fp32 matrices and
 * the factored form).  Host-only: needs no device. */
KQ_API kq_status kq_select_variant(int64_t M, int64_t d, int log2n, kq_dtype mat_dtype, int has_factored,
                                   kq_variant* chosen);

/* ---------------------------------------------------------------- status
 *
 * kq_get_device_error -- synchronises the current device and reports the
 * flags kernels on it have recorded: KQ_ERR_DEVICE_TIMEOUT (a bounded wait ran
 * out), KQ_ERR_SINGULAR (a factor with u == 0), else KQ_OK.  clear != 0 resets
 * the flags.  Returns KQ_ERR_CUDA if the device cannot be read. */
KQ_API kq_status kq_get_device_error(int clear);

/* Description of the last failing CUDA call made by this library on the calling
 * thread (for a KQ_ERR_CUDA status); "no error" if none.  Thread-local storage,
 * valid until the thread's next failing call. */
KQ_API const char* kq_last_error(void);

/* Static, human-readable name of a status code. */
KQ_API const char* kq_status_string(kq_status status);

/* ABI version of this header (major * 100 + minor). */
KQ_API int kq_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KQ_H */
