// kq_quant.cuh -- fused block-transform + MXFP4 quantizer kernels (sm_100a).
//
// One kernel template, three transforms:
//   MODE_KRON   KroQuant: y = x K_b, K_b = F0 (x) ... (x) F4 ("KroQuant: Kronecker-
//               Structured Block Transforms ...", Approach), applied as a 5-stage
//               butterfly in registers: K_b = (M_0 (x) ... (x) M_4) D_b with
//               M_k = [[1, b_k/d_k],[c_k/a_k, 1]] and D_b diagonal, so each stage
//               is one FMA per element and |M||D| = |K| entry-wise.
//   MODE_FWHT   the fixed normalised Hadamard H_32 (LRQ-DiT eq. 3) in the same
//               form (c/a = 1, b/d = -1, D_j = +-2^-2.5): the FWHT comparison point.
//   MODE_SMOOTH per-channel scaling y_j = x_j s_j: the SmoothQuant comparison point.
//
// Data movement: a CTA owns a column tile of W blocks and walks row tiles of R
// rows.  Each row tile (W*R blocks of 64 B) is fetched by one 3-D TMA load
// (box {32, W, R}, 64-byte swizzle, no multicast) into a ring of shared-memory
// stages; thread t = r*W + c handles block c of row r.  With the 64 B swizzle
// the 16-byte chunk k of block t sits at chunk k ^ ((t >> 1) & 3), which makes
// the four 16-byte shared loads of a warp conflict-free.
//
// Exactness (KRON, FWHT): the fp32 result y_f differs from the definition
// y32 = fp32(sum_i x_i K32[i][j]) by at most E = C * ||x||_1 * max|K| (C covers
// 6 fp32 roundings of the butterfly, the fp32 rounding of the coefficients and
// of K32, and the final rounding, with a factor-two margin).  The scale is taken
// from y_f only when max|y| +- E has one E8M0 exponent, and each code only when
// the values (y_f -+ E) 2^-e round (downward / upward) to the same E2M1 code;
// every other scale or code is recomputed in fp64 in the definition's order,
// so the output equals the definition bit for bit.
#pragma once

#include <float.h>

#include "kq_common.cuh"

namespace kq {

enum Mode { MODE_KRON = 0, MODE_FWHT = 1, MODE_SMOOTH = 2 };

constexpr float kFwhtC = 0.17677669529663688f;      // fp32 nearest to 2^-2.5
constexpr float kKronErrC = 1.9073486328125e-06f;   // 2^-19 = 32 u (14 u needed)
constexpr float kFwhtErrC = 9.5367431640625e-07f;   // 2^-20 = 16 u (7 u needed)
constexpr float kErrAbs = 7.174648137343064e-43f;   // 2^-140: FWHT subnormal-range slack
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s per bounded wait

struct QuantParams {
  const uint16_t* x;      // bf16 bits [M][ldx] (exact path re-reads rows from here)
  int64_t ldx;
  int64_t M;
  int nb;                 // blocks per row (d / 32)
  int W;                  // blocks per column tile
  int R;                  // rows per row tile
  int n_row_tiles;
  int stages;
  int stage_stride;       // bytes between stages (multiple of 1024)
  const float* mats;      // KRON: fp32 [nb][32][32] (exact path)
  const float* factored;  // KRON: [nb][48]
  const float* inv_s;     // SMOOTH: [nb*32]
  uint8_t* q;             // [M][nb*16]
  uint8_t* scales;        // [M][nb]
};

// ---------------------------------------------------------------- exact fp64 path

// y32 of one element: fp32 rounding of sum_i x_i K[i][j], accumulated in fp64 in
// increasing i from +0 (each product is exact in fp64).
template <int MODE>
__device__ __noinline__ float exact_y(const uint16_t* __restrict__ xb, const float* __restrict__ Kb, int j) {
  double acc = 0.0;
#pragma unroll 4
  for (int i = 0; i < kBlock; i++) {
    double kij;
    if (MODE == MODE_FWHT)
      kij = (__popc(i & j) & 1) ? -double(kFwhtC) : double(kFwhtC);
    else
      kij = double(Kb[i * kBlock + j]);
    acc = __dadd_rn(acc, __dmul_rn(double(bf16_to_f32(xb[i])), kij));
  }
  return __double2float_rn(acc);
}

// Whole block in fp64: scale from the exact maximum, then every code.
template <int MODE>
__device__ __noinline__ void exact_block(const uint16_t* __restrict__ xb, const float* __restrict__ Kb,
                                         uint8_t* __restrict__ qb, uint8_t* __restrict__ sb) {
  float y[kBlock];
  bool finite = true;
  float amax = 0.0f;
  for (int j = 0; j < kBlock; j++) {
    y[j] = exact_y<MODE>(xb, Kb, j);
    if (!isfinite(y[j])) finite = false;
    else amax = fmaxf(amax, fabsf(y[j]));
  }
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  int byte = 0xFF;
  if (finite) {
    byte = e8m0_byte(amax);
    const float s = inv_scale_of_byte(byte);
    for (int k = 0; k < 4; k++) {
      const float* v = y + 8 * k;
      w[k] = e2m1x8(__fmul_rn(v[0], s), __fmul_rn(v[1], s), __fmul_rn(v[2], s), __fmul_rn(v[3], s),
                    __fmul_rn(v[4], s), __fmul_rn(v[5], s), __fmul_rn(v[6], s), __fmul_rn(v[7], s));
    }
  }
  *reinterpret_cast<uint4*>(qb) = make_uint4(w[0], w[1], w[2], w[3]);
  *sb = uint8_t(byte);
}

template <int MODE>
__device__ __noinline__ uint32_t exact_code(const uint16_t* __restrict__ xb, const float* __restrict__ Kb, int j,
                                            float s) {
  return e2m1_one(__fmul_rn(exact_y<MODE>(xb, Kb, j), s));
}

// ---------------------------------------------------------------- per-thread coefficients

struct Coef {
  float lam[5];   // c_k / a_k, k = factor index (factor k acts on index bit 4-k)
  float bet[5];   // b_k / d_k
  float D[32];
  float cfac;     // C * max|K|
  float eabs;     // absolute error allowance for subnormal-range results
  bool exact_only;
};

template <int MODE>
__device__ __forceinline__ void load_coef(const QuantParams& p, int b, Coef& c) {
  if (MODE == MODE_KRON) {
    const float4* f = reinterpret_cast<const float4*>(p.factored + int64_t(b) * kFactored);
    float buf[kFactored];
#pragma unroll
    for (int i = 0; i < kFactored / 4; i++) {
      const float4 v = __ldg(f + i);
      buf[4 * i + 0] = v.x;
      buf[4 * i + 1] = v.y;
      buf[4 * i + 2] = v.z;
      buf[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int k = 0; k < 5; k++) {
      c.lam[k] = buf[k];
      c.bet[k] = buf[5 + k];
    }
#pragma unroll
    for (int j = 0; j < 32; j++) c.D[j] = buf[10 + j];
    c.cfac = __fmul_ru(kKronErrC, buf[42]);
    c.eabs = buf[44];
    c.exact_only = buf[43] != 0.0f;
  } else if (MODE == MODE_SMOOTH) {
    const float4* f = reinterpret_cast<const float4*>(p.inv_s + int64_t(b) * kBlock);
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 v = __ldg(f + i);
      c.D[4 * i + 0] = v.x;
      c.D[4 * i + 1] = v.y;
      c.D[4 * i + 2] = v.z;
      c.D[4 * i + 3] = v.w;
    }
    c.cfac = 0.0f;
    c.eabs = 0.0f;
    c.exact_only = false;
  } else {
    c.cfac = kFwhtErrC * kFwhtC;
    c.eabs = kErrAbs;
    c.exact_only = false;
  }
}

// ---------------------------------------------------------------- one block of one row

template <int MODE>
__device__ __forceinline__ void quant_block(const QuantParams& p, const Coef& c, const uint4 (&xr)[4], int64_t row,
                                            int b) {
  uint8_t* qb = p.q + row * int64_t(p.nb) * 16 + int64_t(b) * 16;
  uint8_t* sb = p.scales + row * int64_t(p.nb) + b;
  const uint16_t* xb = p.x + row * p.ldx + int64_t(b) * kBlock;
  const float* Kb = (MODE == MODE_KRON) ? p.mats + int64_t(b) * kBlock * kBlock : nullptr;

  float y[kBlock];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const uint32_t w[4] = {xr[k].x, xr[k].y, xr[k].z, xr[k].w};
#pragma unroll
    for (int h = 0; h < 4; h++) {
      y[8 * k + 2 * h] = bf16lo(w[h]);
      y[8 * k + 2 * h + 1] = bf16hi(w[h]);
    }
  }

  if (MODE == MODE_SMOOTH) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kBlock; j++) {
      y[j] = __fmul_rn(y[j], c.D[j]);  // exactly the definition: one fp32 rounding
      amax = fmax_nan(amax, fabsf(y[j]));
    }
    if (!(amax <= FLT_MAX)) {
      *reinterpret_cast<uint4*>(qb) = make_uint4(0u, 0u, 0u, 0u);
      *sb = 0xFF;
      return;
    }
    const int byte = e8m0_byte(amax);
    const float s = inv_scale_of_byte(byte);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const float* v = y + 8 * k;
      w[k] = e2m1x8(__fmul_rn(v[0], s), __fmul_rn(v[1], s), __fmul_rn(v[2], s), __fmul_rn(v[3], s),
                    __fmul_rn(v[4], s), __fmul_rn(v[5], s), __fmul_rn(v[6], s), __fmul_rn(v[7], s));
    }
    *reinterpret_cast<uint4*>(qb) = make_uint4(w[0], w[1], w[2], w[3]);
    *sb = uint8_t(byte);
    return;
  }

  // ||x||_1, rounded upward so that it bounds the exact norm
  float l1 = 0.0f;
#pragma unroll
  for (int j = 0; j < kBlock; j++) l1 = __fadd_ru(l1, fabsf(y[j]));

  // butterfly: stage on index bit pb applies factor k = 4 - pb
#pragma unroll
  for (int pb = 0; pb < 5; pb++) {
    const float lam = (MODE == MODE_FWHT) ? 1.0f : c.lam[4 - pb];
    const float bet = (MODE == MODE_FWHT) ? -1.0f : c.bet[4 - pb];
#pragma unroll
    for (int i = 0; i < kBlock; i++) {
      if (i & (1 << pb)) continue;
      const int i1 = i | (1 << pb);
      const float x0 = y[i], x1 = y[i1];
      y[i] = __fmaf_rn(lam, x1, x0);
      y[i1] = __fmaf_rn(bet, x0, x1);
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < kBlock; j++) {
    const float dj = (MODE == MODE_FWHT) ? ((__popc(j) & 1) ? -kFwhtC : kFwhtC) : c.D[j];
    y[j] = __fmul_rn(y[j], dj);
    amax = fmax_nan(amax, fabsf(y[j]));
  }

  if (l1 == 0.0f) {  // all inputs are +-0: every y is +0 by definition
    *reinterpret_cast<uint4*>(qb) = make_uint4(0u, 0u, 0u, 0u);
    *sb = 0;
    return;
  }
  const float E = __fmaf_ru(c.cfac, l1, c.eabs);
  bool exact = c.exact_only || !(amax <= FLT_MAX) || !(E <= FLT_MAX);
  const int byte = e8m0_byte(__fadd_ru(amax, E));
  if (!exact && byte != e8m0_byte(fmaxf(__fsub_rd(amax, E), 0.0f))) exact = true;
  if (exact) {
    exact_block<MODE>(xb, Kb, qb, sb);
    return;
  }
  const float s = inv_scale_of_byte(byte);
  const float eb = __fmul_ru(E, s);
  uint32_t cm[4], cp[4];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const float* v = y + 8 * k;
    cm[k] = e2m1x8(__fmaf_rd(v[0], s, -eb), __fmaf_rd(v[1], s, -eb), __fmaf_rd(v[2], s, -eb),
                   __fmaf_rd(v[3], s, -eb), __fmaf_rd(v[4], s, -eb), __fmaf_rd(v[5], s, -eb),
                   __fmaf_rd(v[6], s, -eb), __fmaf_rd(v[7], s, -eb));
    cp[k] = e2m1x8(__fmaf_ru(v[0], s, eb), __fmaf_ru(v[1], s, eb), __fmaf_ru(v[2], s, eb),
                   __fmaf_ru(v[3], s, eb), __fmaf_ru(v[4], s, eb), __fmaf_ru(v[5], s, eb),
                   __fmaf_ru(v[6], s, eb), __fmaf_ru(v[7], s, eb));
  }
  const uint32_t diff = (cm[0] ^ cp[0]) | (cm[1] ^ cp[1]) | (cm[2] ^ cp[2]) | (cm[3] ^ cp[3]);
  if (diff != 0u) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
      uint32_t dm = cm[k] ^ cp[k];
      while (dm) {
        const int nib = (__ffs(dm) - 1) >> 2;
        const uint32_t code = exact_code<MODE>(xb, Kb, 8 * k + nib, s);
        cm[k] = (cm[k] & ~(0xFu << (4 * nib))) | (code << (4 * nib));
        dm &= ~(0xFu << (4 * nib));
      }
    }
  }
  *reinterpret_cast<uint4*>(qb) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
  *sb = uint8_t(byte);
}

// ---------------------------------------------------------------- kernel

template <int MODE>
__global__ void __launch_bounds__(256) quant_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.stages * p.stage_stride);

  const int t = threadIdx.x;
  const int bb = t % p.W, rr = t / p.W;
  const int b = blockIdx.x * p.W + bb;
  const bool has_tile = rr < p.R;
  const bool active = has_tile && b < p.nb;
  const uint32_t stage_bytes = uint32_t(p.W) * uint32_t(p.R) * 64u;
  const int my_tiles = (p.n_row_tiles - int(blockIdx.y) + int(gridDim.y) - 1) / int(gridDim.y);

  Coef c;
  if (active) load_coef<MODE>(p, b, c);

  if (t == 0) {
    s_abort = 0;
    prefetch_tensormap(&tmap);
    for (int s = 0; s < p.stages; s++) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (t == 0) {
    const int first = my_tiles < p.stages ? my_tiles : p.stages;
    for (int s = 0; s < first; s++) {
      const int tile = int(blockIdx.y) + s * int(gridDim.y);
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      tma_load_3d(base + s * p.stage_stride, &tmap, &full[s], 0, int(blockIdx.x) * p.W, tile * p.R);
    }
  }

  const int sw = (t >> 1) & 3;
  int it = 0;
  for (; it < my_tiles; it++) {
    const int s = it % p.stages;
    const uint32_t parity = uint32_t(it / p.stages) & 1u;
    if (!mbar_wait_bounded(&full[s], parity, kWaitLimitNs)) s_abort = 1;
    uint4 xr[4];
    if (has_tile) {
      const uint4* blk = reinterpret_cast<const uint4*>(base + s * p.stage_stride + t * 64);
#pragma unroll
      for (int k = 0; k < 4; k++) xr[k] = blk[k ^ sw];
    }
    __syncthreads();
    if (s_abort) break;
    if (t == 0 && it + p.stages < my_tiles) {
      const int tile = int(blockIdx.y) + (it + p.stages) * int(gridDim.y);
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      tma_load_3d(base + s * p.stage_stride, &tmap, &full[s], 0, int(blockIdx.x) * p.W, tile * p.R);
    }
    const int64_t row = int64_t(int(blockIdx.y) + it * int(gridDim.y)) * p.R + rr;
    if (active && row < p.M) quant_block<MODE>(p, c, xr, row, b);
  }
  if (it < my_tiles && t == 0) {
    // a wait ran out: drain the loads still in flight (bounded) before exiting
    const int last = (it + p.stages < my_tiles) ? it + p.stages : my_tiles;
    for (int k = it; k < last; k++)
      mbar_wait_bounded(&full[k % p.stages], uint32_t(k / p.stages) & 1u, kWaitLimitNs / 4);
  }
}

}  // namespace kq
