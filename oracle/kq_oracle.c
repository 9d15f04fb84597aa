/*
 * kq_oracle.c -- CPU oracle of the KroQuant online activation quantizer.
 *
 * TEST INFRASTRUCTURE ONLY (see kq_oracle.h): plain scalar C in fp64, no
 * blocking, no fusion, no reordering beyond what each definition states.
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (fp64 operations stay single
 * IEEE operations).
 */
#include "kq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define KQO_N 32      /* block length: "each 32-element block" [KQ-abs]        */
#define KQO_NF 5      /* five 2x2 factors, 32 = 2^5 [KQ-sum, Approach]          */

static float f32_from_bf16(uint16_t h) {
  uint32_t w = (uint32_t)h << 16;
  float f;
  memcpy(&f, &w, 4);
  return f;
}

/* [KQ-sum, Approach]: each factor is a 2x2 unit-determinant LU factor.
 * L = [[1,0],[l,1]] (unit lower), U = [[u,v],[0,1/u]] (det 1); F = L U as a
 * plain 2x2 matrix product. */
void kqo_factor(float l, float u, float v, double F[4]) {
  const double L[4] = {1.0, 0.0, (double)l, 1.0};
  const double U[4] = {(double)u, (double)v, 0.0, 1.0 / (double)u};
  for (int r = 0; r < 2; r++)
    for (int c = 0; c < 2; c++) F[2 * r + c] = L[2 * r + 0] * U[0 + c] + L[2 * r + 1] * U[2 + c];
}

/* Inverse of F = L U is U^-1 L^-1 with L^-1 = [[1,0],[-l,1]] and
 * U^-1 = [[1/u,-v],[0,u]] (both triangular, det 1). */
void kqo_factor_inverse(float l, float u, float v, double Fi[4]) {
  const double Li[4] = {1.0, 0.0, -(double)l, 1.0};
  const double Ui[4] = {1.0 / (double)u, -(double)v, 0.0, (double)u};
  for (int r = 0; r < 2; r++)
    for (int c = 0; c < 2; c++) Fi[2 * r + c] = Ui[2 * r + 0] * Li[0 + c] + Ui[2 * r + 1] * Li[2 + c];
}

/* Kronecker product (A (x) B)[i][j] = A[i/nb][j/nb] * B[i%nb][j%nb]. */
void kqo_kron(const double* A, int na, const double* B, int nbd, double* out) {
  const int n = na * nbd;
  for (int i = 0; i < n; i++)
    for (int j = 0; j < n; j++)
      out[i * n + j] = A[(i / nbd) * na + (j / nbd)] * B[(i % nbd) * nbd + (j % nbd)];
}

/* [KQ-sum, Approach]: the 32x32 block transform is the Kronecker product of the
 * five factors, K = F0 (x) (F1 (x) (F2 (x) (F3 (x) F4)))  (F0 outermost).  The
 * inverse is the Kronecker product of the factor inverses, in the same order. */
void kqo_expand_f64(const float* params, int64_t nb, int inverse, double* K) {
  double F[KQO_NF][4];
  double acc[KQO_N * KQO_N], tmp[KQO_N * KQO_N];
  for (int64_t b = 0; b < nb; b++) {
    const float* p = params + b * 3 * KQO_NF;
    for (int k = 0; k < KQO_NF; k++) {
      if (inverse)
        kqo_factor_inverse(p[3 * k + 0], p[3 * k + 1], p[3 * k + 2], F[k]);
      else
        kqo_factor(p[3 * k + 0], p[3 * k + 1], p[3 * k + 2], F[k]);
    }
    /* innermost first: acc = F4, then F3 (x) acc, ..., F0 (x) acc */
    int n = 2;
    memcpy(acc, F[KQO_NF - 1], sizeof(double) * 4);
    for (int k = KQO_NF - 2; k >= 0; k--) {
      kqo_kron(F[k], 2, acc, n, tmp);
      n *= 2;
      memcpy(acc, tmp, sizeof(double) * (size_t)n * (size_t)n);
    }
    memcpy(K + b * KQO_N * KQO_N, acc, sizeof(double) * KQO_N * KQO_N);
  }
}

/* bf16 is 1 sign, 8 exponent, 7 fraction bits.  Round-to-nearest-even of a:
 * q is the spacing of bf16 values around |a| (2^(E-8) in the normal range,
 * 2^-133 below 2^-126); |a|/q is split into integer and fractional parts and
 * rounded to the nearer integer, ties to the even one. */
uint16_t kqo_bf16_from_f64(double a) {
  if (isnan(a)) return 0x7FC0;
  const int neg = signbit(a) ? 1 : 0;
  double m = fabs(a);
  double r;
  if (m == 0.0) {
    r = 0.0;
  } else if (isinf(m)) {
    r = INFINITY;
  } else {
    int E;
    frexp(m, &E); /* m = f 2^E, f in [0.5, 1) */
    if (E < -125) E = -125;
    const double q = ldexp(1.0, E - 8);
    const double n = m / q; /* exact: q is a power of two */
    double lo = floor(n);
    const double frac = n - lo;
    if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) lo += 1.0;
    r = lo * q; /* 2^128 when it overflows: becomes +inf as float below */
  }
  float f = (float)r; /* exact: r is a bf16 value (or 2^128 -> inf) */
  if (neg) f = -f;
  uint32_t w;
  memcpy(&w, &f, 4);
  return (uint16_t)(w >> 16);
}

void kqo_expand(const float* params, int64_t nb, int inverse, int dtype, void* out) {
  const int64_t n = nb * KQO_N * KQO_N;
  double* K = (double*)malloc(sizeof(double) * (size_t)n);
  kqo_expand_f64(params, nb, inverse, K);
  if (dtype == KQO_F32) {
    float* o = (float*)out;
    for (int64_t i = 0; i < n; i++) o[i] = (float)K[i];
  } else {
    uint16_t* o = (uint16_t*)out;
    for (int64_t i = 0; i < n; i++) o[i] = kqo_bf16_from_f64(K[i]);
  }
  free(K);
}

/* [LRQ, Sec. 3.2, eq. 3]: H_2 = (1/sqrt 2)[[1,1],[1,-1]], H_{2^n} = H_2 (x) H_{2^(n-1)}. */
void kqo_hadamard(int n, double* H) {
  const double s = 1.0 / sqrt(2.0);
  const double H2[4] = {s, s, s, -s};
  double* acc = (double*)malloc(sizeof(double) * (size_t)(1 << n) * (size_t)(1 << n));
  double* tmp = (double*)malloc(sizeof(double) * (size_t)(1 << n) * (size_t)(1 << n));
  memcpy(acc, H2, sizeof(H2));
  int m = 2;
  for (int k = 1; k < n; k++) {
    kqo_kron(H2, 2, acc, m, tmp);
    m *= 2;
    memcpy(acc, tmp, sizeof(double) * (size_t)m * (size_t)m);
  }
  memcpy(H, acc, sizeof(double) * (size_t)m * (size_t)m);
  free(acc);
  free(tmp);
}

/* MXFP4 shared scale (E8M0): e = floor(log2 amax) - emax_elem with emax_elem = 2
 * for E2M1, clamped to the E8M0 range [-127, 127]; stored as e + 127.
 * frexp gives amax = f 2^E with f in [0.5,1), so floor(log2 amax) = E - 1. */
int kqo_e8m0(float amax) {
  if (!isfinite(amax)) return 0xFF;
  if (amax == 0.0f) return 0;
  int E;
  frexp((double)amax, &E);
  int e = (E - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e + 127;
}

void kqo_e8m0_many(const float* amax, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = (uint8_t)kqo_e8m0(amax[i]);
}

/* E2M1 magnitudes, in code order 0..7, and the midpoints between neighbours. */
static const double kqo_grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* E2M1 element: round |v| to the nearest grid magnitude; a value exactly on a
 * midpoint goes to the even code (the one whose mantissa bit is 0); above the
 * last midpoint everything saturates to 6.  Bit 3 carries the sign of v. */
int kqo_e2m1(float v) {
  const double a = fabs((double)v);
  int c = 0;
  while (c < 7 && a > 0.5 * (kqo_grid[c] + kqo_grid[c + 1])) c++;
  if (c < 7 && a == 0.5 * (kqo_grid[c] + kqo_grid[c + 1]) && (c & 1)) c++;
  return c | (signbit(v) ? 8 : 0);
}

/* Value of a code: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
 * exponent field 0 is the subnormal 0 / 0.5. */
double kqo_e2m1_value(int code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

void kqo_e2m1_pack(const float* v, int64_t n, uint8_t* out) {
  for (int64_t k = 0; k < n / 2; k++)
    out[k] = (uint8_t)(kqo_e2m1(v[2 * k]) | (kqo_e2m1(v[2 * k + 1]) << 4));
}

static double mat_entry(const void* mats, int dtype, int64_t idx) {
  if (dtype == KQO_F32) return (double)((const float*)mats)[idx];
  return (double)f32_from_bf16(((const uint16_t*)mats)[idx]);
}

/* [KQ-abs]: each 32-element block of the activation gets its own transform;
 * [LRQ, eq. 2]: row-vector form X H.  y_j = sum_i x_i K[i][j]; every product of
 * a bf16 and an fp32/bf16 value is exact in fp64, the sum runs over i in
 * increasing order from +0, and the result is rounded once to fp32. */
void kqo_transform(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                   const void* mats, int dtype, float* y) {
  const int64_t nb = d / KQO_N;
  for (int64_t r = 0; r < M; r++)
    for (int64_t b = 0; b < nb; b++)
      for (int j = 0; j < KQO_N; j++) {
        double acc = 0.0;
        for (int i = 0; i < KQO_N; i++) {
          const double xi = (double)f32_from_bf16(x[r * ldx + b * KQO_N + i]);
          acc += xi * mat_entry(mats, dtype, b * KQO_N * KQO_N + (int64_t)i * KQO_N + j);
        }
        y[r * d + b * KQO_N + j] = (float)acc;
      }
}

/* MXFP4 [KQ-abs "W4A4 (MXFP4e2)"]: per 32 elements one E8M0 scale 2^e with
 * e from the block's largest magnitude, then each element v = y 2^-e (an fp32
 * multiply) is rounded to E2M1; two codes per byte. */
void kqo_mx_quantize(const float* y, int64_t M, int64_t d, uint8_t* q, uint8_t* scales) {
  const int64_t nb = d / KQO_N;
  for (int64_t r = 0; r < M; r++)
    for (int64_t b = 0; b < nb; b++) {
      const float* yb = y + r * d + b * KQO_N;
      uint8_t* qb = q + r * (d / 2) + b * (KQO_N / 2);
      int finite = 1;
      float amax = 0.0f;
      for (int j = 0; j < KQO_N; j++) {
        if (!isfinite(yb[j])) finite = 0;
        else if (fabsf(yb[j]) > amax) amax = fabsf(yb[j]);
      }
      if (!finite) {
        scales[r * nb + b] = 0xFF;
        memset(qb, 0, KQO_N / 2);
        continue;
      }
      const int byte = kqo_e8m0(amax);
      scales[r * nb + b] = (uint8_t)byte;
      const float s = ldexpf(1.0f, 127 - byte); /* 2^-e, a normal fp32 for byte <= 252 */
      float v[KQO_N];
      for (int j = 0; j < KQO_N; j++) v[j] = yb[j] * s;
      kqo_e2m1_pack(v, KQO_N, qb);
    }
}

void kqo_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                  const void* mats, int dtype, uint8_t* q, uint8_t* scales) {
  float* y = (float*)malloc(sizeof(float) * (size_t)(M * d > 0 ? M * d : 1));
  kqo_transform(x, M, d, ldx, mats, dtype, y);
  kqo_mx_quantize(y, M, d, q, scales);
  free(y);
}

/* [KQ-sum, Key results / KQ-abs]: per-channel scaling (SmoothQuant) before
 * MXFP4 is the cheap comparison point; y_j = fp32(x_j * inv_s_j). */
void kqo_smooth_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                         const float* inv_s, uint8_t* q, uint8_t* scales) {
  float* y = (float*)malloc(sizeof(float) * (size_t)(M * d > 0 ? M * d : 1));
  for (int64_t r = 0; r < M; r++)
    for (int64_t c = 0; c < d; c++)
      y[r * d + c] = (float)((double)f32_from_bf16(x[r * ldx + c]) * (double)inv_s[c]);
  kqo_mx_quantize(y, M, d, q, scales);
  free(y);
}

/* [KQ-sum, Key results]: FWHT before MXFP4 is the other comparison point; here
 * the fixed 32x32 normalised Hadamard of eq. 3, rounded once to fp32, applied
 * to every block like a KroQuant block matrix. */
void kqo_fwht_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx,
                       uint8_t* q, uint8_t* scales) {
  const int64_t nb = d / KQO_N;
  double H[KQO_N * KQO_N];
  kqo_hadamard(KQO_NF, H);
  float* mats = (float*)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1) * KQO_N * KQO_N);
  for (int64_t b = 0; b < nb; b++)
    for (int i = 0; i < KQO_N * KQO_N; i++) mats[b * KQO_N * KQO_N + i] = (float)H[i];
  kqo_quantize(x, M, d, ldx, mats, KQO_F32, q, scales);
  free(mats);
}

/* Inverse of the quantizer: yhat_j = value(code_j) 2^(byte-127) (byte 0xFF is
 * NaN); with inv_mats the block transform is undone, xhat = yhat K^-1, which
 * is the activation-side half of eq. 2's invariance. */
void kqo_dequantize(const uint8_t* q, const uint8_t* scales, int64_t M, int64_t d,
                    const void* inv_mats, int dtype, double* out) {
  const int64_t nb = d / KQO_N;
  for (int64_t r = 0; r < M; r++)
    for (int64_t b = 0; b < nb; b++) {
      const int byte = scales[r * nb + b];
      double yh[KQO_N];
      for (int j = 0; j < KQO_N; j++) {
        const uint8_t pair = q[r * (d / 2) + b * (KQO_N / 2) + j / 2];
        const int code = (j & 1) ? (pair >> 4) : (pair & 0xF);
        yh[j] = (byte == 0xFF) ? NAN : kqo_e2m1_value(code) * ldexp(1.0, byte - 127);
      }
      for (int i = 0; i < KQO_N; i++) {
        double v;
        if (inv_mats == NULL) {
          v = yh[i];
        } else {
          v = 0.0;
          for (int j = 0; j < KQO_N; j++)
            v += yh[j] * mat_entry(inv_mats, dtype, b * KQO_N * KQO_N + (int64_t)j * KQO_N + i);
        }
        out[r * d + b * KQO_N + i] = v;
      }
    }
}

/* ---- transform blocks of n = 2^log2n elements ------------------------------------ */

/* [KQ-sum, Approach / Limitations]: the same construction with log2n factors,
 * assembled from the innermost factor outward. */
void kqo_expand_n_f64(const float* params, int64_t nt, int log2n, int inverse, double* K) {
  const int n = 1 << log2n;
  double* acc = (double*)malloc(sizeof(double) * (size_t)n * (size_t)n);
  double* tmp = (double*)malloc(sizeof(double) * (size_t)n * (size_t)n);
  for (int64_t c = 0; c < nt; c++) {
    const float* p = params + c * 3 * log2n;
    double F[4];
    int m = 2;
    if (inverse)
      kqo_factor_inverse(p[3 * (log2n - 1)], p[3 * (log2n - 1) + 1], p[3 * (log2n - 1) + 2], F);
    else
      kqo_factor(p[3 * (log2n - 1)], p[3 * (log2n - 1) + 1], p[3 * (log2n - 1) + 2], F);
    memcpy(acc, F, sizeof(F));
    for (int k = log2n - 2; k >= 0; k--) {
      if (inverse)
        kqo_factor_inverse(p[3 * k], p[3 * k + 1], p[3 * k + 2], F);
      else
        kqo_factor(p[3 * k], p[3 * k + 1], p[3 * k + 2], F);
      kqo_kron(F, 2, acc, m, tmp);
      m *= 2;
      memcpy(acc, tmp, sizeof(double) * (size_t)m * (size_t)m);
    }
    memcpy(K + c * (int64_t)n * n, acc, sizeof(double) * (size_t)n * (size_t)n);
  }
  free(acc);
  free(tmp);
}

void kqo_expand_n(const float* params, int64_t nt, int log2n, int inverse, int dtype, void* out) {
  const int64_t total = nt * ((int64_t)1 << (2 * log2n));
  double* K = (double*)malloc(sizeof(double) * (size_t)(total > 0 ? total : 1));
  kqo_expand_n_f64(params, nt, log2n, inverse, K);
  if (dtype == KQO_F32) {
    float* o = (float*)out;
    for (int64_t i = 0; i < total; i++) o[i] = (float)K[i];
  } else {
    uint16_t* o = (uint16_t*)out;
    for (int64_t i = 0; i < total; i++) o[i] = kqo_bf16_from_f64(K[i]);
  }
  free(K);
}

void kqo_transform_n(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const void* mats, int dtype,
                     int n, float* y) {
  const int64_t nt = d / n;
  for (int64_t r = 0; r < M; r++)
    for (int64_t c = 0; c < nt; c++)
      for (int j = 0; j < n; j++) {
        double acc = 0.0;
        for (int i = 0; i < n; i++) {
          const double xi = (double)f32_from_bf16(x[r * ldx + c * n + i]);
          acc += xi * mat_entry(mats, dtype, c * (int64_t)n * n + (int64_t)i * n + j);
        }
        y[r * d + c * n + j] = (float)acc;
      }
}

void kqo_quantize_n(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const void* mats, int dtype,
                    int n, uint8_t* q, uint8_t* scales) {
  float* y = (float*)malloc(sizeof(float) * (size_t)(M * d > 0 ? M * d : 1));
  kqo_transform_n(x, M, d, ldx, mats, dtype, n, y);
  kqo_mx_quantize(y, M, d, q, scales);
  free(y);
}

/* ---- the consumer: W4A4 product of two MXFP4 operands --------------------------- */

/* Value of element k of an MXFP4 row: its E2M1 code times its block's power of two. */
static double mx_value(const uint8_t* q, const uint8_t* scales, int64_t row, int64_t k, int64_t K) {
  const int byte = scales[row * (K / KQO_N) + k / KQO_N];
  const uint8_t pair = q[row * (K / 2) + k / 2];
  const int code = (k & 1) ? (pair >> 4) : (pair & 0xF);
  if (byte == 0xFF) return NAN;
  return ldexp(kqo_e2m1_value(code), byte - 127);
}

/* [KQ-sum, Approach]; [KQ-abs] W4A4: the plain dot product of every activation row
 * with every weight row, both as MXFP4 values, summed in fp64 in index order. */
void kqo_mx_gemm(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                 const uint8_t* b_scales, int64_t N, int64_t K, double* c) {
  for (int64_t m = 0; m < M; m++)
    for (int64_t n = 0; n < N; n++) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; k++)
        acc += mx_value(a_q, a_scales, m, k, K) * mx_value(b_q, b_scales, n, k, K);
      c[m * N + n] = acc;
    }
}

/* ---- the producer: AdaLN normalisation fused in front of the quantizer ------------ */

/* Pairwise sum in fp32: a[0..n) padded with +0 to a power of two, then neighbours
 * added level by level.  tmp holds at least that power of two. */
static float pairwise_sum_f32(const float* a, int64_t n, float* tmp) {
  int64_t p = 1;
  while (p < n) p *= 2;
  for (int64_t i = 0; i < p; i++) tmp[i] = (i < n) ? a[i] : 0.0f;
  for (int64_t w = p; w > 1; w /= 2)
    for (int64_t j = 0; j < w / 2; j++) tmp[j] = tmp[2 * j] + tmp[2 * j + 1];
  return tmp[0];
}

/* [KQ §Problem], [KQ abstract]: the modulated LayerNorm whose output the quantizer
 * receives, in the step order stated in the header (every operation one IEEE binary32
 * operation: the build keeps fp32 expressions unfused). */
void kqo_adaln(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const uint16_t* shift,
               const uint16_t* scale, int64_t rows_per_group, float eps, uint16_t* h, float* stats) {
  int64_t p = 1;
  while (p < d) p *= 2;
  float* v = (float*)malloc(sizeof(float) * (size_t)(d > 0 ? d : 1));
  float* tmp = (float*)malloc(sizeof(float) * (size_t)p);
  const float df = (float)d;
  for (int64_t r = 0; r < M; r++) {
    for (int64_t i = 0; i < d; i++) v[i] = f32_from_bf16(x[r * ldx + i]);
    const float mu = pairwise_sum_f32(v, d, tmp) / df;
    for (int64_t i = 0; i < d; i++) {
      const float t = v[i] - mu;
      v[i] = t * t;
    }
    const float var = pairwise_sum_f32(v, d, tmp) / df;
    const float rstd = 1.0f / sqrtf(var + eps);
    const int64_t g = r / rows_per_group;
    for (int64_t i = 0; i < d; i++) {
      const float t = f32_from_bf16(x[r * ldx + i]) - mu;
      const float a = 1.0f + f32_from_bf16(scale[g * d + i]);
      const float b = f32_from_bf16(shift[g * d + i]);
      h[r * d + i] = kqo_bf16_from_f64((double)((t * rstd) * a + b));
    }
    if (stats != NULL) {
      stats[2 * r] = mu;
      stats[2 * r + 1] = rstd;
    }
  }
  free(v);
  free(tmp);
}

void kqo_adaln_quantize(const uint16_t* x, int64_t M, int64_t d, int64_t ldx, const uint16_t* shift,
                        const uint16_t* scale, int64_t rows_per_group, float eps, const void* mats,
                        int dtype, uint8_t* q, uint8_t* scales, float* stats) {
  uint16_t* h = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(M * d > 0 ? M * d : 1));
  kqo_adaln(x, M, d, ldx, shift, scale, rows_per_group, eps, h, stats);
  kqo_quantize(h, M, d, d, mats, dtype, q, scales);
  free(h);
}
