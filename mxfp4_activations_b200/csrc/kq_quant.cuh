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
// Data movement: a tile is 8 block columns x 32 rows (16 KB of bf16), fetched by
// one 3-D TMA load (box {32 elements, 32 rows, 8 blocks}, 64-byte swizzle, no
// multicast) into a ring of shared-memory stages; in shared memory the tile is
// [block column][row][64 B].  A CTA owns one group of 8 block columns and walks
// a stride of row tiles.  Its last warp only issues the loads; a stage is
// refilled when every consumer warp has arrived on its "empty" barrier, so
// consumer warps never wait for each other.  Consumer warp w holds block
// columns 4(w&1)..4(w&1)+3 and rows 8(w>>1)..8(w>>1)+7 of each tile: lane l
// takes column 4(w&1) + l/8 and row 8(w>>1) + l%8.  Eight lanes share a column,
// so the per-column coefficients are read from a shared table by broadcast loads
// (four distinct addresses per warp, in distinct banks) instead of living in
// registers, and the four 16-byte shared loads of a block stay conflict-free
// under the swizzle (chunk k of 64-byte row t sits at chunk k ^ ((t >> 1) & 3)).
// Each row's four blocks give 64 contiguous bytes of codes per warp store.
// The butterfly stages on index bits 1..4 run as packed f32x2 FMAs on element
// pairs (2m, 2m+1).
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
constexpr float kKronErrC64 = 1.9073486328125e-06f; // 2^-19 = 32 u for 64-element blocks (16 u needed)
constexpr float kFwhtErrC = 4.76837158203125e-07f;  // 2^-21 = 8 u (7 u needed)
constexpr float kErrAbs = 7.174648137343064e-43f;   // 2^-140: FWHT subnormal-range slack

// Tile geometry (see "Data movement" above).
constexpr int kQCols = 8;                        // block columns per tile
constexpr int kQRows = 32;                       // rows per tile
constexpr int kQConsWarps = 8;                   // consumer warps (4 columns x 8 rows each)
constexpr int kQThreads = (kQConsWarps + 1) * 32;  // + the TMA producer warp
constexpr int kQStageBytes = kQCols * kQRows * 64;  // 16 KB
constexpr int kQStages = 4;
// Shared coefficient table, one record of kQCoef floats per block column:
//   [4s .. 4s+3]  (lam, lam, bet, bet) of the stage on index bit s+1 (factor 3-s), s = 0..3
//   [16 .. 47]    D_0 .. D_31 (SMOOTH: the 32 per-channel factors)
//   [48 .. 51]    lam and bet of factor 4 (index bit 0), C * max|K| (+inf: exact path
//                 only), absolute allowance
//   [52 .. 53]    lam and bet of the factor that mixes the two 32-element halves of a
//                 64-element transform block (64-element blocks only)
constexpr int kQCoef = 56;

struct QuantParams {
  const uint16_t* x;      // bf16 bits [M][ldx] (exact path re-reads rows from here)
  int64_t ldx;
  int64_t M;
  int nb;                 // blocks per row (d / 32)
  int n_row_tiles;        // ceil(M / 32)
  int coef_offset;        // bytes from the stage ring to the coefficient table (kQStages * kQStageBytes)
  const float* mats;      // KRON: fp32 [nb][32][32] (exact path)
  const float* factored;  // KRON: [nb][48]
  const float* inv_s;     // SMOOTH: [nb*32]
  uint8_t* q;             // [M][nb*16]
  uint8_t* scales;        // row-major [M][nb], or tiled (scale_index)
};

// Entry f of the coefficient record of block column b (fp32 bits as read by
// the consumer warps).
template <int MODE, int NT>
__device__ __forceinline__ float coef_entry(const QuantParams& p, int b, int f) {
  if (MODE == MODE_KRON) {
    const float* fb = p.factored + int64_t(b) * kFactored;
    if (f < 16) {
      const int k = 3 - (f >> 2);                  // factor of this stage
      return __ldg(fb + ((f & 2) ? 5 + k : k));    // bet_k = b/d, lam_k = c/a
    }
    if (f < 48) return __ldg(fb + 10 + (f - 16));  // D
    if (f == 48) return __ldg(fb + 4);
    if (f == 49) return __ldg(fb + 9);
    if (f == 50)
      return __ldg(fb + 43) != 0.0f ? __int_as_float(0x7F800000)
                                    : __fmul_ru(NT == 64 ? kKronErrC64 : kKronErrC, __ldg(fb + 42));
    if (f == 51) return __ldg(fb + 44);
    if (NT == 64 && f == 52) return __ldg(fb + 45);
    if (NT == 64 && f == 53) return __ldg(fb + 46);
    return 0.0f;
  }
  if (MODE == MODE_SMOOTH) return (f >= 16 && f < 48) ? __ldg(p.inv_s + int64_t(b) * kBlock + (f - 16)) : 0.0f;
  return 0.0f;
}

// ---------------------------------------------------------------- one block of one row
//
// cf: shared-memory address of this block column's coefficient record.  NT = 64:
// the block is one half of a 64-element transform block whose other half is held
// by lane ^ 8 (same row, neighbouring column); `upper` marks the second half.
template <int MODE, int NT>
__device__ __forceinline__ void quant_block(uint32_t cf, const uint4 (&xr)[4], bool act, uint8_t* qb, uint8_t* sb,
                                            const uint16_t* xb, const float* Kb, bool upper) {
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
    for (int i = 0; i < 8; i++) {
      const uint4 dv = lds128(cf + 64 + 16 * i);
      Y[2 * i] = mul2_rn(pk2(x[4 * i], x[4 * i + 1]), pk2(__uint_as_float(dv.x), __uint_as_float(dv.y)));
      Y[2 * i + 1] = mul2_rn(pk2(x[4 * i + 2], x[4 * i + 3]), pk2(__uint_as_float(dv.z), __uint_as_float(dv.w)));
    }
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
  float l1 = __fadd_ru(__fadd_ru(l1p[0], l1p[1]), __fadd_ru(l1p[2], l1p[3]));
  // every output of a 64-element block depends on all 64 inputs
  if (NT == 64) {
    l1 = __fadd_ru(l1, __shfl_xor_sync(0xFFFFFFFFu, l1, 8));
    // factor 0 of a 64-element block, applied first (the Kronecker factors act on
    // different index bits and commute): x_lo + lam x_hi in the lower half, x_hi +
    // bet x_lo in the upper one, element by element, with the partner half's inputs
    // taken from lane ^ 8 as raw bf16 pairs (16 shuffles)
    const uint4 cx = lds128(cf + 208);
    const float cc = upper ? __uint_as_float(cx.y) : __uint_as_float(cx.x);
    const uint64_t C2 = pk2(cc, cc);
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const uint32_t w[4] = {xr[k].x, xr[k].y, xr[k].z, xr[k].w};
#pragma unroll
      for (int h = 0; h < 4; h++) {
        const uint32_t pw = __shfl_xor_sync(0xFFFFFFFFu, w[h], 8);
        const uint64_t X = fma2_rn(C2, pk2(bf16lo(pw), bf16hi(pw)), pk2(x[8 * k + 2 * h], x[8 * k + 2 * h + 1]));
        upk2(X, x[8 * k + 2 * h], x[8 * k + 2 * h + 1]);
      }
    }
  }

  float cfac, eabs;
  // stage on index bit 0 (factor 4), scalar: the pair partners share a register pair
  {
    float l4 = 1.0f, b4 = -1.0f;
    if (MODE == MODE_KRON) {
      const uint4 s0 = lds128(cf + 192);
      l4 = __uint_as_float(s0.x);
      b4 = __uint_as_float(s0.y);
      cfac = __uint_as_float(s0.z);
      eabs = __uint_as_float(s0.w);
    } else {
      cfac = kFwhtErrC * kFwhtC;
      eabs = kErrAbs;
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
    uint64_t L2 = 0, B2 = 0;
    if (MODE == MODE_KRON) {
      const uint4 c = lds128(cf + 16 * (pb - 1));
      L2 = pk2(__uint_as_float(c.x), __uint_as_float(c.y));
      B2 = pk2(__uint_as_float(c.z), __uint_as_float(c.w));
    }
#pragma unroll
    for (int m = 0; m < 16; m++) {
      if (m & (1 << (pb - 1))) continue;
      const int m1 = m | (1 << (pb - 1));
      const uint64_t y0 = Y[m], y1 = Y[m1];
      if (MODE == MODE_FWHT) {
        Y[m] = add2_rn(y0, y1);
        Y[m1] = sub2_rn(y1, y0);
      } else {
        Y[m] = fma2_rn(L2, y1, y0);
        Y[m1] = fma2_rn(B2, y0, y1);
      }
    }
  }
  // diagonal: D_j (FWHT: +-2^-2.5 with the sign of (-1)^popcount(j))
  if (MODE == MODE_FWHT) {
#pragma unroll
    for (int m = 0; m < 16; m++) {
      const float sg = (__popc(m) & 1) ? -kFwhtC : kFwhtC;
      Y[m] = mul2_rn(pk2(sg, -sg), Y[m]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const uint4 dv = lds128(cf + 64 + 16 * i);
      Y[2 * i] = mul2_rn(pk2(__uint_as_float(dv.x), __uint_as_float(dv.y)), Y[2 * i]);
      Y[2 * i + 1] = mul2_rn(pk2(__uint_as_float(dv.z), __uint_as_float(dv.w)), Y[2 * i + 1]);
    }
  }
#pragma unroll
  for (int m = 0; m < 16; m++) upk2(Y[m], y[2 * m], y[2 * m + 1]);
  const float amax = block_amax(y);

  constexpr int KSRC = (MODE == MODE_FWHT) ? KSRC_FWHT : KSRC_F32;
  // l1 is an upward-rounded fp32 sum of |x| without flushing: 0 exactly when all inputs are +-0
  // cfac = +inf marks a column whose butterfly form is unusable: every block exact
  certify_store(Y, amax, l1, l1 == 0.0f, cfac, eabs, !(cfac <= FLT_MAX), act, qb, sb,
                [&](bool need) { warp_exact_pass<KSRC, NT>(need, xb, Kb, qb, sb); });
}

// ---------------------------------------------------------------- kernel

// TILED: scales in the 128 x 4 tiled layout of block-scaled GEMMs (a template
// parameter, so the row-major store costs nothing extra).  NT: transform block of
// 32 or 64 elements (KRON only; 64 needs an even number of block columns).
template <int MODE, int TILED, int NT>
__global__ void __launch_bounds__(kQThreads, 3) quant_kernel(const __grid_constant__ CUtensorMap tmap, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // [kQCols][kQCoef] after the stages; the offset comes from the host (kept out of
  // the compile-time address arithmetic, which otherwise costs the loop a register)
  float* coef = reinterpret_cast<float*>(base + p.coef_offset);
  uint64_t* full = reinterpret_cast<uint64_t*>(coef + kQCols * kQCoef);
  uint64_t* empty = full + kQStages;

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int col0 = int(blockIdx.x) * kQCols;
  const int my_tiles = (p.n_row_tiles - int(blockIdx.y) + int(gridDim.y) - 1) / int(gridDim.y);

  if (t == 0) {
    for (int s = 0; s < kQStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(kQConsWarps));
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream

  if (warp == kQConsWarps) {  // producer warp: one thread issues every TMA load
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      int it = 0;
      for (; it < my_tiles; it++) {
        const int s = it % kQStages;
        if (it >= kQStages && !mbar_wait_bounded(&empty[s], uint32_t(it / kQStages - 1) & 1u, kWaitLimitNs))
          break;
        const int tile = int(blockIdx.y) + it * int(gridDim.y);
        mbar_arrive_expect_tx(&full[s], uint32_t(kQStageBytes));
        tma_load_3d(base + s * kQStageBytes, &tmap, &full[s], 0, tile * kQRows, col0);
      }
      grid_launch_dependents();  // every load issued: the next grid may start its prologue
      if (it < my_tiles) {  // consumers stopped: let the loads still in flight land before exiting
        for (int k = (it > kQStages ? it - kQStages : 0); k < it; k++)
          mbar_wait_bounded(&full[k % kQStages], uint32_t(k / kQStages) & 1u, kWaitLimitNs / 4);
      }
    }
    return;
  }

  // coefficient table of this CTA's columns (consumer warps only; the producer
  // is already streaming the first tiles)
  if (MODE != MODE_FWHT) {
    constexpr int kN = kQCols * kQCoef;
    constexpr int kPer = (kN + kQConsWarps * 32 - 1) / (kQConsWarps * 32);
    float v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = t + i * kQConsWarps * 32;
      const int c = e / kQCoef;
      v[i] = (e < kN && col0 + c < p.nb) ? coef_entry<MODE, NT>(p, col0 + c, e - c * kQCoef) : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = t + i * kQConsWarps * 32;
      if (e < kN) coef[e] = v[i];
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kQConsWarps * 32) : "memory");
  }

  const int cl = (warp & 1) * 4 + (lane >> 3);  // block column inside the tile
  const int rl = (warp >> 1) * 8 + (lane & 7);  // row inside the tile
  const int b = col0 + cl;
  const bool col_ok = b < p.nb;
  const int bc = col_ok ? b : 0;
  const uint32_t cf = smem_addr(coef + cl * kQCoef);
  const uint32_t xoff = uint32_t(cl * kQRows + rl) * 64u;
  const int sw = (rl >> 1) & 3;
  const uint32_t sbase = smem_addr(base);
  // exact path: this block's columns of its transform matrix ([nt][NT][NT]), and
  // the transform block's first input
  const float* Kb = (MODE == MODE_KRON)
                        ? p.mats + int64_t(bc / (NT / kBlock)) * NT * NT + (bc % (NT / kBlock)) * kBlock
                        : nullptr;
  const int bx = bc - bc % (NT / kBlock);  // first block column of the transform block
  const bool upper = (bc % (NT / kBlock)) != 0;
  // per-tile pointer steps: gridDim.y row tiles of kQRows rows
  const int64_t row_step = int64_t(gridDim.y) * kQRows;
  int64_t row = int64_t(blockIdx.y) * kQRows + rl;

  for (int it = 0; it < my_tiles; it++, row += row_step) {
    const int s = it % kQStages;  // compile-time ring size: no integer division per block
    if (!mbar_wait_bounded(&full[s], uint32_t(it / kQStages) & 1u, kWaitLimitNs)) break;
    uint4 xr[4];
    const uint32_t blk = sbase + uint32_t(s) * kQStageBytes + xoff;
#pragma unroll
    for (int k = 0; k < 4; k++) xr[k] = lds128(blk + uint32_t((k ^ sw) << 4));
    stage_release(&empty[s], lane);
    const bool act = col_ok && row < p.M;
    const int64_t rowc = act ? row : 0;
    uint8_t* qb = p.q + rowc * int64_t(p.nb) * 16 + int64_t(bc) * 16;
    uint8_t* sb = p.scales + scale_index(rowc, bc, p.nb, TILED);
    const uint16_t* xb = p.x + rowc * p.ldx + int64_t(bx) * kBlock;
    // every lane takes part (the exact path is warp-cooperative); only real blocks store
    quant_block<MODE, NT>(cf, xr, act, qb, sb, xb, Kb, upper);
  }
}

}  // namespace kq
