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
// stages.  The last warp of the CTA only issues those loads; a stage is refilled
// when every consumer warp has arrived on its "empty" barrier, so consumer
// warps never wait for each other.  Consumer thread t = r*W + c handles block c
// of row r.  With the 64 B swizzle the 16-byte chunk k of block t sits at chunk
// k ^ ((t >> 1) & 3), which makes the four 16-byte shared loads of a warp
// conflict-free.  The butterfly stages on index bits 1..4 run as packed f32x2
// FMAs on element pairs (2m, 2m+1).
//
// Exactness (KRON, FWHT): the fp32 result y_f differs from the definition
// y32 = fp32(sum_i x_i K32[i][j]) by at most E = C * ||x||_1 * max|K|.  KRON:
// 6 roundings on each output's path (5 FMA stages, 1 multiply by D) give 6u;
// the fp32 coefficients (5 ratios and D_j, each rounded once) put the applied
// matrix within 6u of K, K32 is within u of K, and y32 is one more rounding:
// 14u in all (u = 2^-24), against C = 16u.  FWHT: 6 roundings + the final one
// = 7u (its coefficients are exactly the entries of fp32(H32)), against 8u.
// ||x||_1 is summed with upward rounding and max|K| is rounded up.  The scale is taken
// from y_f only when max|y| +- E has one E8M0 exponent, and each code only when
// the values (y_f -+ E) 2^-e round (downward / upward) to the same E2M1 code;
// every other scale or code is recomputed in fp64 in the definition's order,
// so the output equals the definition bit for bit.
#pragma once

#include <float.h>

#include "kq_common.cuh"
#include "kq_mx.cuh"

namespace kq {

enum Mode { MODE_KRON = 0, MODE_FWHT = 1, MODE_SMOOTH = 2 };

constexpr float kKronErrC = 9.5367431640625e-07f;   // 2^-20 = 16 u (14 u needed, see below)
constexpr float kFwhtErrC = 4.76837158203125e-07f;  // 2^-21 = 8 u (7 u needed)
constexpr float kErrAbs = 7.174648137343064e-43f;   // 2^-140: FWHT subnormal-range slack

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
  int cons_warps;         // consumer warps; one more warp issues the TMA loads
  const float* mats;      // KRON: fp32 [nb][32][32] (exact path)
  const float* factored;  // KRON: [nb][48]
  const float* inv_s;     // SMOOTH: [nb*32]
  uint8_t* q;             // [M][nb*16]
  uint8_t* scales;        // [M][nb]
};

// ---------------------------------------------------------------- per-thread coefficients

struct Coef {
  uint64_t lam2[5];  // (c_k/a_k, c_k/a_k); factor k acts on index bit 4-k
  uint64_t bet2[5];  // (b_k/d_k, b_k/d_k)
  uint64_t D2[16];   // (D[2m], D[2m+1]); SMOOTH: the per-channel factors
  float cfac;        // C * max|K|
  float eabs;        // absolute error allowance for subnormal-range results
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
      c.lam2[k] = pk2(buf[k], buf[k]);
      c.bet2[k] = pk2(buf[5 + k], buf[5 + k]);
    }
#pragma unroll
    for (int m = 0; m < 16; m++) c.D2[m] = pk2(buf[10 + 2 * m], buf[11 + 2 * m]);
    c.cfac = __fmul_ru(kKronErrC, buf[42]);
    c.eabs = buf[44];
    c.exact_only = buf[43] != 0.0f;
  } else if (MODE == MODE_SMOOTH) {
    const float4* f = reinterpret_cast<const float4*>(p.inv_s + int64_t(b) * kBlock);
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 v = __ldg(f + i);
      c.D2[2 * i] = pk2(v.x, v.y);
      c.D2[2 * i + 1] = pk2(v.z, v.w);
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
                                            int b, bool act) {
  uint8_t* qb = p.q + row * int64_t(p.nb) * 16 + int64_t(b) * 16;
  uint8_t* sb = p.scales + row * int64_t(p.nb) + b;
  const uint16_t* xb = p.x + row * p.ldx + int64_t(b) * kBlock;
  const float* Kb = (MODE == MODE_KRON) ? p.mats + int64_t(b) * kBlock * kBlock : nullptr;

  float x[kBlock];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const uint32_t w[4] = {xr[k].x, xr[k].y, xr[k].z, xr[k].w};
#pragma unroll
    for (int h = 0; h < 4; h++) {
      x[8 * k + 2 * h] = bf16lo(w[h]);
      x[8 * k + 2 * h + 1] = bf16hi(w[h]);
    }
  }
  uint64_t Y[16];
  float y[kBlock];

  if (MODE == MODE_SMOOTH) {
#pragma unroll
    for (int m = 0; m < 16; m++) Y[m] = mul2_rn(pk2(x[2 * m], x[2 * m + 1]), c.D2[m]);  // one rounding each
#pragma unroll
    for (int m = 0; m < 16; m++) upk2(Y[m], y[2 * m], y[2 * m + 1]);
    const float amax = block_amax(y);
    if (!act) return;
    if (!(amax <= FLT_MAX)) {
      *reinterpret_cast<uint4*>(qb) = make_uint4(0u, 0u, 0u, 0u);
      *sb = 0xFF;
      return;
    }
    const int byte = e8m0_byte(amax);
    const uint64_t S2 = pk2(inv_scale_of_byte(byte), inv_scale_of_byte(byte));
#pragma unroll
    for (int m = 0; m < 16; m++) Y[m] = mul2_rn(Y[m], S2);
    *reinterpret_cast<uint4*>(qb) = make_uint4(codes8(Y), codes8(Y + 4), codes8(Y + 8), codes8(Y + 12));
    *sb = uint8_t(byte);
    return;
  }

  // ||x||_1 rounded upward (four partial sums for ILP)
  float l1p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int j = 0; j < kBlock; j++) l1p[j & 3] = __fadd_ru(l1p[j & 3], fabsf(x[j]));
  const float l1 = __fadd_ru(__fadd_ru(l1p[0], l1p[1]), __fadd_ru(l1p[2], l1p[3]));

  // stage on index bit 0 (factor 4), scalar: the pair partners share a register pair
  {
    float l4 = 1.0f, b4 = -1.0f;
    if (MODE == MODE_KRON) {
      float t0;
      upk2(c.lam2[4], l4, t0);
      upk2(c.bet2[4], b4, t0);
    }
#pragma unroll
    for (int m = 0; m < 16; m++) {
      const float x0 = x[2 * m], x1 = x[2 * m + 1];
      if (MODE == MODE_FWHT) {
        x[2 * m] = __fadd_rn(x0, x1);
        x[2 * m + 1] = __fsub_rn(x1, x0);
      } else {
        x[2 * m] = __fmaf_rn(l4, x1, x0);
        x[2 * m + 1] = __fmaf_rn(b4, x0, x1);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 16; m++) Y[m] = pk2(x[2 * m], x[2 * m + 1]);
  // stages on index bits 1..4 (factors 3..0) on packed pairs
#pragma unroll
  for (int pb = 1; pb < 5; pb++) {
#pragma unroll
    for (int m = 0; m < 16; m++) {
      if (m & (1 << (pb - 1))) continue;
      const int m1 = m | (1 << (pb - 1));
      const uint64_t y0 = Y[m], y1 = Y[m1];
      if (MODE == MODE_FWHT) {
        Y[m] = add2_rn(y0, y1);
        Y[m1] = sub2_rn(y1, y0);
      } else {
        Y[m] = fma2_rn(c.lam2[4 - pb], y1, y0);
        Y[m1] = fma2_rn(c.bet2[4 - pb], y0, y1);
      }
    }
  }
  // diagonal: D_j (FWHT: +-2^-2.5 with the sign of (-1)^popcount(j))
#pragma unroll
  for (int m = 0; m < 16; m++) {
    if (MODE == MODE_FWHT) {
      const float sg = (__popc(m) & 1) ? -kFwhtC : kFwhtC;
      Y[m] = mul2_rn(pk2(sg, -sg), Y[m]);
    } else {
      Y[m] = mul2_rn(c.D2[m], Y[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < 16; m++) upk2(Y[m], y[2 * m], y[2 * m + 1]);
  const float amax = block_amax(y);

  constexpr int KSRC = (MODE == MODE_FWHT) ? KSRC_FWHT : KSRC_F32;
  // l1 is an upward-rounded fp32 sum of |x| without flushing: 0 exactly when all inputs are +-0
  certify_store(Y, amax, l1, l1 == 0.0f, c.cfac, c.eabs, c.exact_only, act, qb, sb,
                [&](bool need) { warp_exact_pass<KSRC>(need, xb, Kb, qb, sb); });
}

// ---------------------------------------------------------------- kernel

template <int MODE>
__global__ void __launch_bounds__(256, 2) quant_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.stages * p.stage_stride);
  uint64_t* empty = full + p.stages;

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const uint32_t stage_bytes = uint32_t(p.W) * uint32_t(p.R) * 64u;
  const int my_tiles = (p.n_row_tiles - int(blockIdx.y) + int(gridDim.y) - 1) / int(gridDim.y);

  if (t == 0) {
    for (int s = 0; s < p.stages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(p.cons_warps));
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == p.cons_warps) {  // producer warp: one thread issues every TMA load
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      int it = 0;
      for (; it < my_tiles; it++) {
        const int s = it % p.stages;
        if (it >= p.stages && !mbar_wait_bounded(&empty[s], uint32_t(it / p.stages - 1) & 1u, kWaitLimitNs)) break;
        const int tile = int(blockIdx.y) + it * int(gridDim.y);
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        tma_load_3d(base + s * p.stage_stride, &tmap, &full[s], 0, int(blockIdx.x) * p.W, tile * p.R);
      }
      if (it < my_tiles) {  // consumers stopped: let the loads still in flight land before exiting
        for (int k = (it > p.stages ? it - p.stages : 0); k < it; k++)
          mbar_wait_bounded(&full[k % p.stages], uint32_t(k / p.stages) & 1u, kWaitLimitNs / 4);
      }
    }
    return;
  }

  const int bb = t % p.W, rr = t / p.W;
  const int b = blockIdx.x * p.W + bb;
  const bool has_tile = rr < p.R;
  const bool active = has_tile && b < p.nb;
  Coef c = {};
  if (active) load_coef<MODE>(p, b, c);

  const int sw = (t >> 1) & 3;
  for (int it = 0; it < my_tiles; it++) {
    const int s = it % p.stages;
    if (!mbar_wait_bounded(&full[s], uint32_t(it / p.stages) & 1u, kWaitLimitNs)) break;
    uint4 xr[4] = {};
    if (has_tile) {
      const uint4* blk = reinterpret_cast<const uint4*>(base + s * p.stage_stride + t * 64);
#pragma unroll
      for (int k = 0; k < 4; k++) xr[k] = blk[k ^ sw];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const int64_t row = int64_t(int(blockIdx.y) + it * int(gridDim.y)) * p.R + rr;
    // every lane takes part (the exact path is warp-cooperative); only real blocks store
    quant_block<MODE>(p, c, xr, row, b, active && row < p.M);
  }
}

}  // namespace kq
