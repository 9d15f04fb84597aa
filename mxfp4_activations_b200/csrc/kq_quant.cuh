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
// Work mapping.  The [M][nb] grid of 32-element blocks is cut into "lanes": lane
// v owns block column c = v % nb and the rows r0 = v / nb, r0 + k, r0 + 2k, ...
// (k rows in flight, k * nb lanes).  Thread t takes lane t, so a thread keeps one
// block column for its whole life: its butterfly coefficients (or per-channel
// factors) are loaded once into registers and no per-block coefficient traffic
// remains.  Consecutive threads hold consecutive block columns of one row, so a
// warp reads 2 KB of contiguous input and writes 512 contiguous bytes of codes and
// 32 contiguous scale bytes per row step.  When nb exceeds the threads of one
// wave, threads walk several lanes.
//
// Data movement.  Each thread streams its own blocks through a private ring of
// kSStages 64-byte slots in shared memory with asynchronous copies (cp.async, four
// 16-byte pieces per block): kSStages - 1 blocks are in flight while one is
// computed, without holding registers.  Piece k of thread t's slot sits at 16-byte
// position k ^ ((t >> 1) & 3), so the four 16-byte reads of a block are free of
// bank conflicts across each group of eight threads.
//
// A row step stores every block's fast result; the rare blocks that the fp32 bound
// cannot certify (below) are then recomputed exactly by the whole warp, which
// overwrites their fast results.
//
// Exactness (KRON, FWHT): the fp32 result y_f differs from the definition
// y32 = fp32(sum_i x_i K32[i][j]) by at most E = C * ||x||_1 * max|K|.  KRON:
// 6 roundings on each output's path (5 FMA stages, 1 multiply by D) give 6u;
// the fp32 coefficients (5 ratios and D_j, each rounded once) put the applied
// matrix within 6u of K, K32 is within u of K, and y32 is one more rounding:
// 14u in all (u = 2^-24) to first order; with the second-order terms of those products
// of (1 + u) factors, 14u + 109u^2, against C = 14u (1 + 2^-16).  FWHT: 6 roundings + the final one
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

constexpr float kKronErrC = 8.344777597812936e-07f; // 14 u (1 + 2^-16), exact in fp32 (14 u + 109 u^2 needed, see above; 12 u for 16-element blocks)
constexpr float kKronErrC64 = 1.9073486328125e-06f; // 2^-19 = 32 u for 64- and 128-element blocks (16 u, 18 u needed)
constexpr float kFwhtErrC = 4.76837158203125e-07f;  // 2^-21 = 8 u (7 u needed)
constexpr float kErrAbs = 7.174648137343064e-43f;   // 2^-140: FWHT subnormal-range slack

constexpr int kSThreads = 256;    // threads per CTA
constexpr int kSCtasPerSm = 2;    // resident CTAs per SM the register budget is written for
constexpr int kSStages = 4;       // 64-byte slots per thread (blocks in flight + 1)
constexpr int kSSmemBytes = kSStages * kSThreads * 64;
constexpr int kDTableBytes = 32 * kBlock * 4;  // D of the 32 block columns a grouped CTA covers
// Dynamic shared memory of quant_kernel: the rings, and with ADALN each thread's staged h
// block (64 bytes) for the warp-cooperative exact path.
// GROUPED adds the CTA's table of D (32 block columns x 32 fp32).
__host__ __device__ constexpr int quant_smem_bytes(bool adaln, bool grouped = false) {
  return kSSmemBytes + (adaln ? kSThreads * 64 : 0) + (grouped ? kDTableBytes : 0);
}

// The AdaLN modulation of one block, every step one IEEE binary32 operation rounded to
// nearest: h_i = bf16( ((x_i - mu) * rstd) * (1 + scale_i) + shift_i ).  X: the block's
// inputs as packed pairs (elements 2j, 2j+1); sv, hv: its 32 scale and shift values (bf16
// bits, 16-byte pieces in element order); hw: h as bf16 pairs.  Packed steps are used only
// where no multiply feeds a packed add (the compiler fuses such a pair into one FMA); the
// add of the shift is the scalar __fadd_rn, which it never contracts.
__device__ __forceinline__ void modulate(const uint64_t (&X)[16], float mu, float rstd, const uint4 (&sv)[4],
                                         const uint4 (&hv)[4], uint32_t (&hw)[16]) {
  const uint64_t MU = pk2(mu, mu), RS = pk2(rstd, rstd), ONE = pk2(1.0f, 1.0f);
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const uint32_t s4[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w}, b4[4] = {hv[k].x, hv[k].y, hv[k].z, hv[k].w};
#pragma unroll
    for (int m = 0; m < 4; m++) {
      const int j = 4 * k + m;
      const uint64_t A = add2_rn(ONE, pk2(bf16lo(s4[m]), bf16hi(s4[m])));
      float v0, v1;
      upk2(mul2_rn(mul2_rn(sub2_rn(X[j], MU), RS), A), v0, v1);
      const float h0 = __fadd_rn(v0, bf16lo(b4[m])), h1 = __fadd_rn(v1, bf16hi(b4[m]));
      uint32_t out;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(h1), "f"(h0));
      hw[j] = out;
    }
  }
}

struct QuantParams {
  const uint16_t* x;      // bf16 bits [M][ldx]
  int64_t ldx;
  int64_t M;
  int64_t k;              // rows in flight per lane pass (row step of a lane)
  int64_t lanes;          // k * nb (every lane: one block column, rows r0 + i k)
  int64_t threads;        // threads that take lanes (lane v is taken by thread v % threads)
  int64_t n_iter;         // row steps per lane: ceil(M / k)
  int passes;             // lanes per thread: ceil(lanes / threads)
  int nb;                 // blocks per row (d / 32)
  int cg;                 // grouped layout (quant_kernel GROUPED): column groups of 32, nb / 32
  const float* mats;      // KRON: fp32 [nb/(NT/32)][NT][NT] (exact path)
  const float* factored;  // KRON: [nb][48]
  const float* inv_s;     // SMOOTH: [nb*32]
  uint8_t* q;             // [M][nb*16]
  uint8_t* scales;        // row-major [M][nb], or tiled (scale_index)
  // ADALN (the quantizer behind an AdaLN-modulated LayerNorm, kq_adaln.cuh): the input
  // of row r's blocks is h = bf16(((x - mu) * rstd) * (1 + scale[g]) + shift[g]),
  // g = r / rows_per_group, with (mu, rstd) = stats[r] from the statistics pass
  const float* stats;     // [M][2]
  const uint16_t* shift;  // bf16 bits [G][nb * 32]
  const uint16_t* scale;  // bf16 bits [G][nb * 32]
  int64_t rows_per_group;
};

// Coefficients of one block column, held in registers by the thread that owns it.
struct ColCoef {
  float l4, b4;         // stage on index bit 0 (factor 4): lam, bet
  uint64_t L[4], B[4];  // stages on index bits 1..4 (factors 3..0): (lam, lam), (bet, bet)
  uint64_t D[16];       // (D_2m, D_2m+1); SMOOTH: the per-channel factors
  float cfac;           // C * max|K| (+inf: the column takes the exact path only)
  float eabs;           // absolute allowance (results in the fp32 subnormal range)
  float mix;            // 64-element blocks: lam (lower half) or bet (upper half) of F0;
                        // 128-element blocks: this column's coefficient of the factor on index bit 5
  float mix2;           // 128-element blocks: this column's coefficient of the factor on index bit 6
  float l16[2], b16[2];        // 16-element blocks: stage on index bit 0 of each half
  uint64_t L16[3][2], B16[3][2];  // 16-element blocks: stages on index bits 1..3 of each half
};

// Offset of column c's first output column in its transform matrix array, and the
// first block column of its transform block (n = 16: the column's two 16 x 16
// matrices; n >= 32: one n x n matrix per n / 32 columns).
template <int NT>
__device__ __forceinline__ int64_t kmat_offset(int c) {
  constexpr int g = NT >= kBlock ? NT / kBlock : 1;  // block columns per transform block
  if (NT == 16) return int64_t(c) * 512;
  return int64_t(c / g) * NT * NT + (c % g) * kBlock;
}
template <int NT>
__device__ __forceinline__ int first_column(int c) {
  constexpr int g = NT >= kBlock ? NT / kBlock : 1;
  return c - c % g;
}

template <int MODE, int NT>
__device__ __forceinline__ void load_coef(const QuantParams& p, int c, ColCoef& cf) {
  cf.l4 = 1.0f;
  cf.b4 = -1.0f;
  cf.cfac = kFwhtErrC * kFwhtC;
  cf.eabs = kErrAbs;
  cf.mix = cf.mix2 = 0.0f;
#pragma unroll
  for (int s = 0; s < 4; s++) cf.L[s] = cf.B[s] = 0;
  if (MODE == MODE_KRON && NT == 16) {
    const float4* fb = reinterpret_cast<const float4*>(p.factored + int64_t(c) * 64);
    float r[64];
#pragma unroll
    for (int i = 0; i < 16; i++) {
      const float4 v = __ldg(fb + i);
      r[4 * i] = v.x;
      r[4 * i + 1] = v.y;
      r[4 * i + 2] = v.z;
      r[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int h = 0; h < 2; h++) {
      cf.l16[h] = r[8 * h + 3];  // factor 3 acts on index bit 0
      cf.b16[h] = r[8 * h + 7];
#pragma unroll
      for (int s = 0; s < 3; s++) {  // stage on bit s+1 uses factor 2-s
        cf.L16[s][h] = pk2(r[8 * h + 2 - s], r[8 * h + 2 - s]);
        cf.B16[s][h] = pk2(r[8 * h + 6 - s], r[8 * h + 6 - s]);
      }
    }
#pragma unroll
    for (int m = 0; m < 16; m++) cf.D[m] = pk2(r[16 + 2 * m], r[17 + 2 * m]);
    cf.cfac = r[49] != 0.0f ? __int_as_float(0x7F800000) : __fmul_ru(kKronErrC, r[48]);
    cf.eabs = r[50];
  } else if (MODE == MODE_KRON) {
    const float4* fb = reinterpret_cast<const float4*>(p.factored + int64_t(c) * kFactored);
    float r[kFactored];
#pragma unroll
    for (int i = 0; i < kFactored / 4; i++) {
      const float4 v = __ldg(fb + i);
      r[4 * i] = v.x;
      r[4 * i + 1] = v.y;
      r[4 * i + 2] = v.z;
      r[4 * i + 3] = v.w;
    }
    cf.l4 = r[4];
    cf.b4 = r[9];
#pragma unroll
    for (int s = 0; s < 4; s++) {  // stage on bit s+1 uses factor 3-s
      cf.L[s] = pk2(r[3 - s], r[3 - s]);
      cf.B[s] = pk2(r[8 - s], r[8 - s]);
    }
#pragma unroll
    for (int m = 0; m < 16; m++) cf.D[m] = pk2(r[10 + 2 * m], r[11 + 2 * m]);
    cf.cfac = r[43] != 0.0f ? __int_as_float(0x7F800000) : __fmul_ru(NT >= 64 ? kKronErrC64 : kKronErrC, r[42]);
    cf.eabs = r[44];
    if (NT == 64) cf.mix = (c & 1) ? r[46] : r[45];
    if (NT == 128) {
      cf.mix = r[45];
      cf.mix2 = r[46];
    }
  } else if (MODE == MODE_SMOOTH) {
    const float4* sp = reinterpret_cast<const float4*>(p.inv_s + int64_t(c) * kBlock);
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 v = __ldg(sp + i);
      cf.D[2 * i] = pk2(v.x, v.y);
      cf.D[2 * i + 1] = pk2(v.z, v.w);
    }
  }
}

// Asynchronous copy of one block (64 bytes at p, 16-byte aligned) into the slot
// whose 16-byte pieces are at slot + ((k ^ sw) << 4); completes with the thread's
// next commit group.
__device__ __forceinline__ void copy_block_async(uint32_t slot, int sw, const uint16_t* p) {
#pragma unroll
  for (int k = 0; k < 4; k++)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(slot + uint32_t((k ^ sw) << 4)), "l"(p + 8 * k)
                 : "memory");
}
__device__ __forceinline__ void copy_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's commit groups are still in flight.
template <int N>
__device__ __forceinline__ void copy_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The 64 bytes of a landed slot as 16 words: word h holds elements 2h (low half)
// and 2h+1 (high half) of the block.
__device__ __forceinline__ void read_slot(uint32_t slot, int sw, uint32_t (&w)[16]) {
#pragma unroll
  for (int k = 0; k < 4; k++) {
    const uint4 v = lds128(slot + uint32_t((k ^ sw) << 4));
    w[4 * k] = v.x;
    w[4 * k + 1] = v.y;
    w[4 * k + 2] = v.z;
    w[4 * k + 3] = v.w;
  }
}

// ---------------------------------------------------------------- one block of one row
//
// NT = 16: the block holds two 16-element transform blocks (its halves).  NT = 64:
// the block is one half of a 64-element transform block whose other half is held
// by lane ^ 1 (same row, neighbouring column).  NT = 128: a quarter of a 128-element
// transform block, the others held by lanes ^ 1, ^ 2 and ^ 3 (bits 5 and 6 of the
// index inside the transform block are bits 0 and 1 of the lane).
// act marks the lanes whose block is real.  Stores the fast result of a real
// block and returns whether it must be recomputed exactly (never for SMOOTH, whose
// fp32 product is the definition itself).
// DSH: D comes from the CTA's shared table (grouped layout), this lane's entries at
// shared address dsh + 512 i (i = 0..7, 16 bytes each: D_4i .. D_4i+3), not from cf.D.
template <int MODE, int NT, bool DSH = false>
__device__ __forceinline__ bool quant_block(const ColCoef& cf, const uint32_t (&w)[16], bool act, uint8_t* qb,
                                            uint8_t* sb, uint32_t dsh = 0u) {
  float x[kBlock];
#pragma unroll
  for (int h = 0; h < 16; h++) {
    x[2 * h] = bf16lo(w[h]);
    x[2 * h + 1] = bf16hi(w[h]);
  }
  uint64_t Y[16];
  float y[kBlock];

  if (MODE == MODE_SMOOTH) {
#pragma unroll
    for (int m = 0; m < 16; m++) Y[m] = mul2_rn(pk2(x[2 * m], x[2 * m + 1]), cf.D[m]);
#pragma unroll
    for (int m = 0; m < 16; m++) upk2(Y[m], y[2 * m], y[2 * m + 1]);
    const float amax = block_amax(y);
    if (!act) return false;
    if (!(amax <= FLT_MAX)) {
      *reinterpret_cast<uint4*>(qb) = make_uint4(0u, 0u, 0u, 0u);
      *sb = 0xFF;
      return false;
    }
    const int byte = e8m0_byte(amax);
    const uint64_t S2 = pk2(inv_scale_of_byte(byte), inv_scale_of_byte(byte));
#pragma unroll
    for (int m = 0; m < 16; m++) Y[m] = mul2_rn(Y[m], S2);
    *reinterpret_cast<uint4*>(qb) = make_uint4(codes8(Y), codes8(Y + 4), codes8(Y + 8), codes8(Y + 12));
    *sb = uint8_t(byte);
    return false;
  }

  // ||x||_1 rounded upward (four partial sums for ILP)
  float l1p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int j = 0; j < kBlock; j++) l1p[j & 3] = __fadd_ru(l1p[j & 3], fabsf(x[j]));
  float l1 = __fadd_ru(__fadd_ru(l1p[0], l1p[1]), __fadd_ru(l1p[2], l1p[3]));
  if (NT >= 64) {
    // every output of the transform block depends on all of its inputs
    l1 = __fadd_ru(l1, __shfl_xor_sync(0xFFFFFFFFu, l1, 1));
    if (NT == 128) l1 = __fadd_ru(l1, __shfl_xor_sync(0xFFFFFFFFu, l1, 2));
    // the factor on index bit 5 (64-element blocks: factor 0; 128: factor 1), applied
    // first (the Kronecker factors act on different index bits and commute): x_lo +
    // lam x_hi in the lower column, x_hi + bet x_lo in the upper one, element by
    // element, with the partner column's inputs taken from lane ^ 1 as raw bf16
    // pairs (16 shuffles)
    const uint64_t C2 = pk2(cf.mix, cf.mix);
#pragma unroll
    for (int h = 0; h < 16; h++) {
      const uint32_t pw = __shfl_xor_sync(0xFFFFFFFFu, w[h], 1);
      const uint64_t X = fma2_rn(C2, pk2(bf16lo(pw), bf16hi(pw)), pk2(x[2 * h], x[2 * h + 1]));
      upk2(X, x[2 * h], x[2 * h + 1]);
    }
    if (NT == 128) {
      // factor 0 (index bit 6) with the 64-element half held by lanes ^ 2, on the
      // fp32 results of the step above (32 shuffles)
      const uint64_t C4 = pk2(cf.mix2, cf.mix2);
#pragma unroll
      for (int h = 0; h < 16; h++) {
        const float p0 = __shfl_xor_sync(0xFFFFFFFFu, x[2 * h], 2);
        const float p1 = __shfl_xor_sync(0xFFFFFFFFu, x[2 * h + 1], 2);
        const uint64_t X = fma2_rn(C4, pk2(p0, p1), pk2(x[2 * h], x[2 * h + 1]));
        upk2(X, x[2 * h], x[2 * h + 1]);
      }
    }
  }

  // stage on index bit 0 (factor 4; 16-element blocks: factor 3 of each half),
  // scalar: the pair partners share a register pair
#pragma unroll
  for (int m = 0; m < 16; m++) {
    const float x0 = x[2 * m], x1 = x[2 * m + 1];
    if (MODE == MODE_FWHT) {
      x[2 * m] = __fadd_rn(x0, x1);
      x[2 * m + 1] = __fsub_rn(x1, x0);
    } else if (NT == 16) {
      x[2 * m] = __fmaf_rn(cf.l16[m >> 3], x1, x0);
      x[2 * m + 1] = __fmaf_rn(cf.b16[m >> 3], x0, x1);
    } else {
      x[2 * m] = __fmaf_rn(cf.l4, x1, x0);
      x[2 * m + 1] = __fmaf_rn(cf.b4, x0, x1);
    }
  }
#pragma unroll
  for (int m = 0; m < 16; m++) Y[m] = pk2(x[2 * m], x[2 * m + 1]);
  // stages on index bits 1..4 (factors 3..0; 16-element blocks: bits 1..3, factors
  // 2..0 of each half) on packed pairs
#pragma unroll
  for (int pb = 1; pb < (NT == 16 ? 4 : 5); pb++) {
#pragma unroll
    for (int m = 0; m < 16; m++) {
      if (m & (1 << (pb - 1))) continue;
      const int m1 = m | (1 << (pb - 1));
      const uint64_t y0 = Y[m], y1 = Y[m1];
      if (MODE == MODE_FWHT) {
        Y[m] = add2_rn(y0, y1);
        Y[m1] = sub2_rn(y1, y0);
      } else if (NT == 16) {
        Y[m] = fma2_rn(cf.L16[pb - 1][m >> 3], y1, y0);
        Y[m1] = fma2_rn(cf.B16[pb - 1][m >> 3], y0, y1);
      } else {
        Y[m] = fma2_rn(cf.L[pb - 1], y1, y0);
        Y[m1] = fma2_rn(cf.B[pb - 1], y0, y1);
      }
    }
  }
  // diagonal: D_j (FWHT: +-2^-2.5 with the sign of (-1)^popcount(j))
#pragma unroll
  for (int m = 0; m < 16; m++) {
    if (MODE == MODE_FWHT) {
      const float sg = (__popc(m) & 1) ? -kFwhtC : kFwhtC;
      Y[m] = mul2_rn(pk2(sg, -sg), Y[m]);
    } else if (DSH) {
      if ((m & 1) == 0) {
        const uint4 v = lds128(dsh + uint32_t(m / 2) * 512u);
        Y[m] = mul2_rn((uint64_t(v.y) << 32) | v.x, Y[m]);
        Y[m + 1] = mul2_rn((uint64_t(v.w) << 32) | v.z, Y[m + 1]);
      }
    } else {
      Y[m] = mul2_rn(cf.D[m], Y[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < 16; m++) upk2(Y[m], y[2 * m], y[2 * m + 1]);
  const float amax = block_amax(y);

  // l1 is an upward-rounded fp32 sum of |x| without flushing: 0 exactly when all inputs are +-0
  // cfac = +inf marks a column whose butterfly form is unusable: every block exact
  return certify_store(Y, amax, l1, l1 == 0.0f, cf.cfac, cf.eabs, !(cf.cfac <= FLT_MAX), act, qb, sb);
}

// ---------------------------------------------------------------- kernel

// One row step of a lane: wait for the block of ring slot `slot` (offset of the
// stage from the thread's slot base), refill the slot read one step earlier with
// the block kSStages - 1 rows ahead, quantize, and recompute exactly every block
// of the warp that the fp32 bound could not certify.
// ADALN: the block is modulated first (QuantParams); st holds this row's (mu, rstd) and
// is replaced by the next row step's, loaded one step ahead; hst is this thread's 64-byte
// staging of h in shared memory.
template <int MODE, int TILED, int NT, bool ADALN = false, bool GROUPED = false>
__device__ __forceinline__ void row_step(const QuantParams& p, const ColCoef& cf, uint32_t cbase, int sw,
                                         uint32_t slot, uint32_t refill, bool lane_ok, int c, int64_t r, int64_t f,
                                         int64_t f_end, int64_t f_ahead, const uint16_t* xr, const uint16_t* xi,
                                         float2& st, uint16_t* hst, uint32_t dsh) {
  const bool act = lane_ok && f < f_end;
  uint4 sv[4], hv[4];
  if (ADALN) {
    // this row's modulation vectors (cached: every row of a group reads the same ones)
    const int64_t g = act ? r / p.rows_per_group : 0;
    const uint4* ps = reinterpret_cast<const uint4*>(p.scale + (g * p.nb + c) * kBlock);
    const uint4* ph = reinterpret_cast<const uint4*>(p.shift + (g * p.nb + c) * kBlock);
#pragma unroll
    for (int k = 0; k < 4; k++) {
      sv[k] = __ldg(ps + k);
      hv[k] = __ldg(ph + k);
    }
  }
  copy_wait<kSStages - 2>();  // this step's block has landed
  uint32_t cur[16];
  read_slot(cbase + slot, sw, cur);
  if (lane_ok && f + f_ahead < f_end) copy_block_async(cbase + refill, sw, xi);
  copy_commit();
  const int64_t fc = act ? f : c;
  uint8_t* qb = p.q + fc * 16;
  uint8_t* sb = p.scales + (TILED ? scale_index(act ? r : 0, c, p.nb, 1) : fc);
  if (ADALN) {
    const float2 sr = st;
    const int64_t rn = r + p.k;  // the lane's next row
    if (lane_ok && rn < p.M) st = __ldg(reinterpret_cast<const float2*>(p.stats) + rn);
    uint64_t X[16];
#pragma unroll
    for (int j = 0; j < 16; j++) X[j] = pk2(bf16lo(cur[j]), bf16hi(cur[j]));
    modulate(X, sr.x, sr.y, sv, hv, cur);
    uint4* hs = reinterpret_cast<uint4*>(hst);
#pragma unroll
    for (int k = 0; k < 4; k++) hs[k] = make_uint4(cur[4 * k], cur[4 * k + 1], cur[4 * k + 2], cur[4 * k + 3]);
    const bool need = quant_block<MODE, NT, GROUPED>(cf, cur, act, qb, sb, dsh);
    if (__any_sync(0xFFFFFFFFu, need)) {
      __syncwarp();  // every lane's staged h is visible to the warp
      warp_exact_pass<KSRC_F32, NT, false>(need, hst, p.mats + kmat_offset<NT>(c), qb, sb);
    }
    return;
  }
  const bool need = quant_block<MODE, NT, GROUPED>(cf, cur, act, qb, sb, dsh);
  if (MODE != MODE_SMOOTH && __any_sync(0xFFFFFFFFu, need)) {
    // rare: the transform block's first input and this block's columns of its matrix
    const uint16_t* xb = xr - (c - first_column<NT>(c)) * kBlock;
    const float* Kb = (MODE == MODE_KRON) ? p.mats + kmat_offset<NT>(c) : nullptr;
    constexpr int KSRC = (MODE == MODE_FWHT) ? KSRC_FWHT : KSRC_F32;
    warp_exact_pass<KSRC, NT>(need, xb, Kb, qb, sb);
  }
}

// TILED: scales in the 128 x 4 tiled layout of block-scaled GEMMs (a template
// parameter, so the row-major store costs nothing extra).  NT: transform block of
// 16, 32, 64 or 128 elements (KRON only; n > 32 needs d % n == 0).
// ADALN (KRON, 32-element blocks only): the quantizer of kq_adaln_quantize's two-kernel
// form, on h formed from x, the statistics pass's (mu, rstd) and the modulation vectors.
// GROUPED (KRON, 32-element blocks, nb % 32 == 0): CTA b covers the 32 block columns of
// group b % cg for 8 row residues, warp w taking residue (b / cg) 8 + w and lane l column
// 32 (b % cg) + l, so the 8 warps share their columns' D, which one warp puts in a
// shared table once (32 fewer live registers per thread), and their matrices for the
// exact pass.  One lane pass per thread (passes = 1).
template <int MODE, int TILED, int NT, bool ADALN = false, bool GROUPED = false>
__global__ void __launch_bounds__(kSThreads, kSCtasPerSm) quant_kernel(const __grid_constant__ QuantParams p) {
  static_assert(!ADALN || (MODE == MODE_KRON && NT == kBlock), "the AdaLN prologue serves KroQuant's 32-element blocks");
  static_assert(!GROUPED || (MODE == MODE_KRON && NT == kBlock), "the grouped layout serves KroQuant's 32-element blocks");
  static_assert(kSStages == 4, "the row loop below is written for a ring of four slots");
  extern __shared__ __align__(128) uint8_t ring[];
  const int64_t t = int64_t(blockIdx.x) * kSThreads + threadIdx.x;
  const int sw = (threadIdx.x >> 1) & 3;
  const uint32_t cbase = smem_addr(ring) + threadIdx.x * 64u;
  uint16_t* hst = reinterpret_cast<uint16_t*>(ring + kSSmemBytes) + threadIdx.x * kBlock;  // ADALN only
  // GROUPED: this lane's column in the CTA's D table
  const uint32_t dsh = smem_addr(ring) + uint32_t(quant_smem_bytes(ADALN)) + (threadIdx.x & 31) * 16u;
  constexpr uint32_t kStage = kSThreads * 64u;  // bytes between the stages of one thread's ring
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  for (int pass = 0; pass < p.passes; pass++) {
    bool lane_ok;
    int c;
    int64_t r0;
    if (GROUPED) {
      const int64_t rr = int64_t(blockIdx.x / unsigned(p.cg)) * (kSThreads / 32) + (threadIdx.x >> 5);
      lane_ok = rr < p.k;
      c = int(blockIdx.x % unsigned(p.cg)) * 32 + (threadIdx.x & 31);
      r0 = lane_ok ? rr : 0;
    } else {
      const int64_t v = t + int64_t(pass) * p.threads;
      lane_ok = t < p.threads && v < p.lanes;
      const int64_t vc = lane_ok ? v : 0;
      c = int(vc % p.nb);
      r0 = vc / p.nb;
    }
    const int64_t xstep = p.k * p.ldx;
    const int64_t fstep = p.k * int64_t(p.nb);
    const int64_t f_end = p.M * int64_t(p.nb);  // row r is real iff its flat index r nb + c < f_end
    const uint16_t* xr = p.x + r0 * p.ldx + int64_t(c) * kBlock;  // this lane's block in row r
    int64_t r = r0;                                                   // row of the step
    int64_t f = r0 * int64_t(p.nb) + c;                               // flat block index of row r
    // the first kSStages - 1 blocks of the lane go in flight before anything else
#pragma unroll
    for (int s = 0; s < kSStages - 1; s++) {
      if (lane_ok && f + s * fstep < f_end) copy_block_async(cbase + s * kStage, sw, xr + s * xstep);
      copy_commit();
    }
    if (pass == 0) grid_launch_dependents();
    ColCoef cf;
    load_coef<MODE, NT>(p, c, cf);
    if (GROUPED) {
      // every warp of the CTA has the same 32 columns: warp 0 fills the table
      if (threadIdx.x < 32) {
#pragma unroll
        for (int m = 0; m < 16; m += 2)
          asm volatile("st.shared.v2.b64 [%0], {%1, %2};" ::"r"(dsh + uint32_t(m / 2) * 512u), "l"(cf.D[m]),
                       "l"(cf.D[m + 1])
                       : "memory");
      }
      __syncthreads();
    }
    float2 st = make_float2(0.0f, 0.0f);  // ADALN: (mu, rstd) of the lane's current row
    if (ADALN && lane_ok && r0 < p.M) st = __ldg(reinterpret_cast<const float2*>(p.stats) + r0);
    const int64_t f_ahead = (kSStages - 1) * fstep;
    const uint16_t* xi = xr + (kSStages - 1) * xstep;  // next block to put in flight
    // two row steps per trip: step i uses stage i & 3, so the pair (i, i + 1) uses
    // stages (h, h + 1) with h = 0 or 2 and refills (h + 3, h) & 3
    uint32_t h = 0;
    for (int64_t i = 0; i < p.n_iter; i += 2) {
      row_step<MODE, TILED, NT, ADALN, GROUPED>(p, cf, cbase, sw, h, (h + 3 * kStage) & (4 * kStage - 1), lane_ok,
                                                c, r, f, f_end, f_ahead, xr, xi, st, hst, dsh);
      if (i + 1 < p.n_iter)
        row_step<MODE, TILED, NT, ADALN, GROUPED>(p, cf, cbase, sw, h + kStage, h, lane_ok, c, r + p.k, f + fstep,
                                                  f_end, f_ahead, xr + xstep, xi + xstep, st, hst, dsh);
      h ^= 2 * kStage;
      r += 2 * p.k;
      f += 2 * fstep;
      xr += 2 * xstep;
      xi += 2 * xstep;
    }
    copy_wait<0>();  // no copy of this pass still writes the ring
  }
}

}  // namespace kq
