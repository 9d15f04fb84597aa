// kq_expand.cuh -- set-up kernels: LU parameters -> block matrices / factored form.
//
// "KroQuant: Kronecker-Structured Block Transforms ...", Approach: each 32x32
// block transform is the Kronecker product of five 2x2 unit-determinant LU
// factors (15 parameters per block).  Factor k of block b is F = L U with
// L = [[1,0],[l,1]], U = [[u,v],[0,1/u]], (l,u,v) = params[b][k]; F0 is the
// outermost factor (it acts on the top bit of the index inside the block).
// All set-up arithmetic is fp64 with explicit IEEE operations, rounded once.
#pragma once

#include "kq_common.cuh"

namespace kq {

constexpr int kMaxFactors = 7;  // blocks of up to 128 elements

// F = L U written as the 2x2 matrix product (row r, column c of F is
// L[r][0] U[0][c] + L[r][1] U[1][c], zero terms included, so signed zeros
// follow the same IEEE rules as the product written out).
__device__ __forceinline__ void lu_factor(const float* __restrict__ prm, double F[4]) {
  const double l = prm[0], u = prm[1], v = prm[2];
  const double L[4] = {1.0, 0.0, l, 1.0};
  const double U[4] = {u, v, 0.0, __ddiv_rn(1.0, u)};
#pragma unroll
  for (int r = 0; r < 2; r++)
#pragma unroll
    for (int c = 0; c < 2; c++)
      F[2 * r + c] = __dadd_rn(__dmul_rn(L[2 * r], U[c]), __dmul_rn(L[2 * r + 1], U[2 + c]));
}

// F^-1 = U^-1 L^-1, U^-1 = [[1/u, -v],[0, u]], L^-1 = [[1,0],[-l,1]].
__device__ __forceinline__ void lu_factor_inverse(const float* __restrict__ prm, double F[4]) {
  const double l = prm[0], u = prm[1], v = prm[2];
  const double Ui[4] = {__ddiv_rn(1.0, u), -v, 0.0, u};
  const double Li[4] = {1.0, 0.0, -l, 1.0};
#pragma unroll
  for (int r = 0; r < 2; r++)
#pragma unroll
    for (int c = 0; c < 2; c++)
      F[2 * r + c] = __dadd_rn(__dmul_rn(Ui[2 * r], Li[c]), __dmul_rn(Ui[2 * r + 1], Li[2 + c]));
}

// Round-to-nearest-even of a double to bf16 bits, from the definition: the
// spacing of bf16 values around |a| is 2^(max(E,-126) - 7), E = floor(log2 |a|).
__device__ __forceinline__ uint16_t bf16_rne_from_f64(double a) {
  if (isnan(a)) return 0x7FC0;
  const uint16_t sign = signbit(a) ? 0x8000 : 0;
  const double m = fabs(a);
  if (m == 0.0) return sign;
  if (isinf(m)) return sign | 0x7F80;
  int E = int((__double_as_longlong(m) >> 52) & 0x7FF) - 1023;  // fp64 subnormals: far below bf16
  if (E < -126) E = -126;
  const int qe = E - 7;
  const double n = scalbn(m, -qe);  // exact
  double k = floor(n);
  const double fr = n - k;
  if (fr > 0.5 || (fr == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;
  const float r = float(scalbn(k, qe));  // exact (or +inf past the largest bf16)
  return sign | uint16_t(__float_as_uint(r) >> 16);
}

// One thread per matrix entry of an n x n block matrix, n = 2^log2n:
// K[i][j] = F0[i_top][j_top] (F1 (... F_{log2n-1})), F0 on the most significant
// index bit, assembled from the innermost factor outward.  mode 0: K, 1: K^-1
// (inverse factors), 2: (K^-1)^T (inverse factors, entry (i, j) taken from (j, i):
// the transpose of a Kronecker product is the product of the transposes).
__global__ void expand_kernel(const float* __restrict__ params, int64_t nt, int log2n, int mode, int out_bf16,
                              void* __restrict__ mats) {
  const int64_t gid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int n = 1 << log2n;
  if (gid >= (nt << (2 * log2n))) return;
  const int64_t b = gid >> (2 * log2n);
  const int r = int(gid >> log2n) & (n - 1), c = int(gid) & (n - 1);
  const int i = mode == 2 ? c : r, j = mode == 2 ? r : c;
  const bool inverse = mode != 0;
  double F[kMaxFactors][4];
  bool singular = false;
  for (int k = 0; k < log2n; k++) {
    const float* prm = params + b * 3 * log2n + 3 * k;
    if (prm[1] == 0.0f) singular = true;
    if (inverse)
      lu_factor_inverse(prm, F[k]);
    else
      lu_factor(prm, F[k]);
  }
  double acc = F[log2n - 1][2 * (i & 1) + (j & 1)];
  for (int k = log2n - 2; k >= 0; k--) {
    const int bi = (i >> (log2n - 1 - k)) & 1, bj = (j >> (log2n - 1 - k)) & 1;
    acc = __dmul_rn(F[k][2 * bi + bj], acc);
  }
  if (singular && i == 0 && j == 0) record_error(kDevErrSingular);
  if (out_bf16)
    static_cast<uint16_t*>(mats)[gid] = bf16_rne_from_f64(acc);
  else
    static_cast<float*>(mats)[gid] = __double2float_rn(acc);
}

// Floats per butterfly record of one 32-element block column.
__host__ __device__ constexpr int factored_floats(int log2n) { return log2n == 4 ? 64 : kFactored; }

// One thread per 32-element block column: the butterfly form F_k = M_k diag(a_k, d_k)
// of its transform block(s) of n = 2^log2n elements (log2n 4..7), as the records
// documented with kq_expand_factored_n:
//   log2n 5..7, [48] floats:
//     [0..4]  c_k/a_k and [5..9] b_k/d_k of the five factors acting inside the
//             32-element block (factors log2n-5 .. log2n-1)
//     [10..41] D_j for this block's 32 outputs
//     [42]    upper bound of max|K|   [43] 1 if only the exact path may be used
//     [44]    absolute allowance
//     log2n 6: [45], [46] c/a, b/d of factor 0 (it mixes the two 32-element halves)
//     log2n 7: [45] the coefficient of factor 1 (index bit 5) that this column uses:
//              c/a when the column is the lower one of its pair, else b/d;
//              [46] the same for factor 0 (index bit 6) and the column's 64-element half
//   log2n 4, [64] floats (two 16-element transform blocks h = 0, 1 per column):
//     [0..3] c/a and [4..7] b/d of factors 0..3 of block h = 0, [8..15] those of h = 1
//     [16..47] D_j for the 32 outputs   [48] upper bound of max|K| over both blocks
//     [49] 1 if only the exact path may be used   [50] absolute allowance   [51..63] zero
__device__ void butterfly_factors(const float* __restrict__ prm, int nf, double* a, double* dd, float* lam,
                                  float* bet, bool& exact_only, bool report, double& kmax, double& gain) {
  for (int k = 0; k < nf; k++) {
    if (prm[3 * k + 1] == 0.0f) {
      if (report) record_error(kDevErrSingular);
      exact_only = true;
    }
    double F[4];
    lu_factor(prm + 3 * k, F);
    a[k] = F[0];
    dd[k] = F[3];
    lam[k] = __double2float_rn(__ddiv_rn(F[2], F[0]));
    bet[k] = __double2float_rn(__ddiv_rn(F[1], F[3]));
    // ratios must be finite and moderate for the fp32 butterfly to be usable
    if (!(fabsf(lam[k]) <= 1.8446744e19f) || !(fabsf(bet[k]) <= 1.8446744e19f)) exact_only = true;
    const double mk = fmax(fmax(fabs(F[0]), fabs(F[1])), fmax(fabs(F[2]), fabs(F[3])));
    kmax = __dmul_rn(kmax, mk);
    gain = __dmul_rn(gain, 1.0 + fmax(fabs(double(lam[k])), fabs(double(bet[k]))));
  }
}

__global__ void expand_factored_kernel(const float* __restrict__ params, int64_t nb32, int log2n,
                                       float* __restrict__ out) {
  const int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nb32) return;
  const int rec = factored_floats(log2n);
  float* o = out + b * rec;
  double a[2][kMaxFactors], dd[2][kMaxFactors];
  float lam[2][kMaxFactors], bet[2][kMaxFactors];
  double kmax[2] = {1.0, 1.0}, gain[2] = {1.0, 1.0};
  bool exact_only = false;
  double dmax = 0.0;
  if (log2n == 4) {  // two 16-element transform blocks: 2b and 2b + 1
    for (int h = 0; h < 2; h++)
      butterfly_factors(params + (2 * b + h) * 12, 4, a[h], dd[h], lam[h], bet[h], exact_only, true, kmax[h],
                        gain[h]);
    for (int h = 0; h < 2; h++)
      for (int k = 0; k < 4; k++) {
        o[8 * h + k] = lam[h][k];
        o[8 * h + 4 + k] = bet[h][k];
      }
    for (int j = 0; j < 32; j++) {
      const int h = j >> 4, jj = j & 15;
      double dj = 1.0;
      for (int k = 0; k < 4; k++) dj = __dmul_rn(dj, ((jj >> (3 - k)) & 1) ? dd[h][k] : a[h][k]);
      const float dj32 = __double2float_rn(dj);
      if (!(fabsf(dj32) <= 3.0e38f) || dj32 == 0.0f) exact_only = true;
      o[16 + j] = dj32;
      dmax = fmax(dmax, fabs(double(dj32)));
    }
    const double km = fmax(kmax[0], kmax[1]);
    const float kmf = __fmul_ru(__double2float_ru(km), 1.00000095367431640625f);
    if (!(kmf <= 1.0e30f)) exact_only = true;
    o[48] = kmf;
    o[49] = exact_only ? 1.0f : 0.0f;
    o[50] = __fmul_ru(__double2float_ru(__dmul_rn(dmax, fmax(gain[0], gain[1]))), 2.2420775429197073e-44f);
    for (int i = 51; i < 64; i++) o[i] = 0.0f;
    return;
  }
  const int64_t c = b >> (log2n - 5);                    // transform block
  const int part = int(b & ((1 << (log2n - 5)) - 1));    // which 32 outputs of it
  const int inner0 = log2n - 5;                          // first factor acting inside the 32-block
  butterfly_factors(params + c * 3 * log2n, log2n, a[0], dd[0], lam[0], bet[0], exact_only, part == 0, kmax[0],
                    gain[0]);
  for (int k = inner0; k < log2n; k++) {
    o[k - inner0] = lam[0][k];
    o[5 + k - inner0] = bet[0][k];
  }
  o[45] = o[46] = o[47] = 0.0f;
  if (log2n == 6) {
    o[45] = lam[0][0];
    o[46] = bet[0][0];
  } else if (log2n == 7) {
    o[45] = (part & 1) ? bet[0][1] : lam[0][1];
    o[46] = (part & 2) ? bet[0][0] : lam[0][0];
  }
  for (int j = 0; j < 32; j++) {
    const int jj = part * 32 + j;  // output index inside the transform block
    double dj = 1.0;
    for (int k = 0; k < log2n; k++) dj = __dmul_rn(dj, ((jj >> (log2n - 1 - k)) & 1) ? dd[0][k] : a[0][k]);
    const float dj32 = __double2float_rn(dj);
    if (!(fabsf(dj32) <= 3.0e38f) || dj32 == 0.0f) exact_only = true;
    o[10 + j] = dj32;
    dmax = fmax(dmax, fabs(double(dj32)));
  }
  // upper bound of max|K| (fp64 product error is far below the allowance's margin)
  const float km = __fmul_ru(__double2float_ru(kmax[0]), 1.00000095367431640625f);
  if (!(km <= 1.0e30f)) exact_only = true;
  o[42] = km;
  o[43] = exact_only ? 1.0f : 0.0f;
  // absolute error of results that fall in the fp32 subnormal range: each of the
  // (log2n + 1 <= 8) roundings on an output's path adds at most 2^-150, amplified by
  // at most max|D| * prod_k (1 + max(|c/a|, |b/d|)); 2^-145 leaves a margin.
  o[44] = __fmul_ru(__double2float_ru(__dmul_rn(dmax, gain[0])), 2.2420775429197073e-44f);
}

}  // namespace kq
