// kq_mx.cuh -- the MXFP4 step shared by the quantizer kernels: block maximum,
// E2M1 codes, and the certified selection between the fast fp32 result and an
// exact fp64 recomputation.
//
// MXFP4 ("W4A4 (MXFP4e2)" in the KroQuant abstract): one E8M0 scale 2^e per 32
// elements with e = floor(log2 max|y|) - 2 (OCP MX rule for E2M1), clamped to
// [-127, 127]; each element v = y 2^-e is rounded to E2M1 (nearest, ties to
// even, saturating at 6, sign kept).  A block with a non-finite y gets scale
// byte 0xFF and zero codes; an all-zero input block is +0 everywhere.
#pragma once

#include <float.h>

#include "kq_common.cuh"

namespace kq {

constexpr float kFwhtC = 0.17677669529663688f;    // fp32 nearest to 2^-2.5
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per bounded wait

// Byte index of the scale of block column b of row `row` (nb block columns):
// row-major, or the 128 x 4 tiled layout of block-scaled tensor-core GEMMs
// (tile (row/128, b/4) of 512 bytes, stored tile row by tile row; inside it
// 16*(row%32) + 4*((row/32)%4) + b%4).
__device__ __forceinline__ int64_t scale_index(int64_t row, int b, int nb, int tiled) {
  if (!tiled) return row * int64_t(nb) + b;
  const int64_t tile = (row >> 7) * int64_t((nb + 3) >> 2) + (b >> 2);
  return tile * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (b & 3);
}

// Where the exact path reads K[i][j] from.
enum KSource { KSRC_F32 = 0, KSRC_BF16 = 1, KSRC_FWHT = 2 };

// max_j |y_j| with NaN propagation: for each residue r = j mod 4, the eight
// elements r, r+4, ..., r+28 through three-input maxima, then the four results.
__device__ __forceinline__ float block_amax(const float (&y)[kBlock]) {
  float a[4];
#pragma unroll
  for (int r = 0; r < 4; r++) {
    float m = fmax3_nan(fabsf(y[r]), fabsf(y[r + 4]), fabsf(y[r + 8]));
    m = fmax3_nan(m, fabsf(y[r + 12]), fabsf(y[r + 16]));
    m = fmax3_nan(m, fabsf(y[r + 20]), fabsf(y[r + 24]));
    a[r] = fmax_nan(m, fabsf(y[r + 28]));
  }
  return fmax_nan(fmax3_nan(a[0], a[1], a[2]), a[3]);
}

// E2M1 codes of the 8 values held in pairs Y[4k .. 4k+3].
__device__ __forceinline__ uint32_t codes8(const uint64_t* Y) {
  float v[8];
#pragma unroll
  for (int h = 0; h < 4; h++) upk2(Y[h], v[2 * h], v[2 * h + 1]);
  return e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
}

// ---------------------------------------------------------------- exact fp64 path
//
// Only blocks whose scale or some code the fp32 bound cannot certify come here.
// Every load of a chunk is issued before its arithmetic, so that one L2 round
// trip serves 32 rows of the recomputation.

// K[i][j] of a block matrix whose rows are `ld` entries apart.
template <int KSRC>
__device__ __forceinline__ float k_entry(const void* __restrict__ Kb, int i, int j, int ld) {
  if (KSRC == KSRC_FWHT) return (__popc(i & j) & 1) ? -kFwhtC : kFwhtC;
  if (KSRC == KSRC_BF16) return bf16_to_f32(__ldg(static_cast<const unsigned short*>(Kb) + i * ld + j));
  return __ldg(static_cast<const float*>(Kb) + i * ld + j);
}

// Exact recomputation of one 32-element output block by the whole warp: lane j
// computes y32_j = fp32( sum_{i < NT} x_i K[i][j] ) in fp64, summing in
// increasing i from +0 (each product of a bf16 and an fp32 or bf16 value is
// exact in fp64).  xb: the NT inputs of the transform block; Kb: column 0 of this
// block's 32 outputs in the NT x NT matrix (rows NT entries apart).  NT = 16: xb is
// the 32-element block, which holds two transform blocks, and Kb their two 16 x 16
// matrices; lane j sums over the 16 inputs of its own half.  Rows of K are
// loaded 32 at a time, each row one coalesced 128-byte load across the warp; x is
// a broadcast load.  The block's scale then comes from the exact maximum and
// every code from the exact value, and lane `owner` stores them.  Must be called
// by all 32 lanes with the same arguments (taken from the owner lane).
// XG: x is in global memory (read-only path); otherwise a generic pointer, which may
// point into shared memory.
template <int KSRC, int NT, bool XG = true>
__device__ __forceinline__ void exact_block_warp(const uint16_t* __restrict__ xb, const void* __restrict__ Kb,
                                              uint8_t* __restrict__ qb, uint8_t* __restrict__ sb, int owner) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
  if (NT == 16) {
    // two 16-element transform blocks: lane j sums over its half's 16 inputs,
    // with the half's 16 x 16 matrix (Kb: the first of the column's two)
    const int h = lane >> 4;
    float kc[16];
#pragma unroll
    for (int i = 0; i < 16; i++) kc[i] = k_entry<KSRC>(Kb, h * 16 + i, lane & 15, 16);
    const uint4* px = reinterpret_cast<const uint4*>(xb + 16 * h);
    uint32_t xw[8];
#pragma unroll
    for (int k = 0; k < 2; k++) {
      const uint4 v = XG ? __ldg(px + k) : px[k];
      xw[4 * k] = v.x;
      xw[4 * k + 1] = v.y;
      xw[4 * k + 2] = v.z;
      xw[4 * k + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 16; i++) {
      const float xi = (i & 1) ? bf16hi(xw[i >> 1]) : bf16lo(xw[i >> 1]);
      acc = __fma_rn(double(xi), double(kc[i]), acc);
    }
  }
#pragma unroll 1
  for (int i0 = 0; i0 < (NT == 16 ? 0 : NT); i0 += kBlock) {
    float kc[kBlock];
#pragma unroll
    for (int i = 0; i < kBlock; i++) kc[i] = k_entry<KSRC>(Kb, i0 + i, lane, NT);
    const uint4* px = reinterpret_cast<const uint4*>(xb + i0);
    uint32_t xw[16];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const uint4 v = XG ? __ldg(px + k) : px[k];
      xw[4 * k] = v.x;
      xw[4 * k + 1] = v.y;
      xw[4 * k + 2] = v.z;
      xw[4 * k + 3] = v.w;
    }
    // every product is exact in fp64, so the fused multiply-add rounds exactly as
    // the addition of the product would
#pragma unroll
    for (int i = 0; i < kBlock; i++) {
      const float xi = (i & 1) ? bf16hi(xw[i >> 1]) : bf16lo(xw[i >> 1]);
      acc = __fma_rn(double(xi), double(kc[i]), acc);
    }
  }
  const float y = __double2float_rn(acc);
  const bool finite = __all_sync(0xFFFFFFFFu, isfinite(y));
  float m = fabsf(y);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  int byte = 0xFF;
  uint32_t code = 0u;
  if (finite) {
    byte = e8m0_byte(m);
    code = e2m1_one(__fmul_rn(y, inv_scale_of_byte(byte)));
  }
  // nibble j of word j/8; OR across each group of eight lanes
  uint32_t w = code << (4 * (lane & 7));
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 4);
  const uint32_t w0 = __shfl_sync(0xFFFFFFFFu, w, 0), w1 = __shfl_sync(0xFFFFFFFFu, w, 8);
  const uint32_t w2 = __shfl_sync(0xFFFFFFFFu, w, 16), w3 = __shfl_sync(0xFFFFFFFFu, w, 24);
  if (lane == owner) {
    *reinterpret_cast<uint4*>(qb) = make_uint4(w0, w1, w2, w3);
    *sb = uint8_t(byte);
  }
}

// Every lane whose block needs the exact path hands it to the whole warp, one
// block at a time.  Called by all 32 lanes.
template <int KSRC, int NT = kBlock, bool XG = true>
__device__ __forceinline__ void warp_exact_pass(bool need, const uint16_t* xb, const void* Kb, uint8_t* qb,
                                                uint8_t* sb) {
  uint32_t pending = __ballot_sync(0xFFFFFFFFu, need);
  while (pending) {
    const int src = __ffs(pending) - 1;
    pending &= pending - 1;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(
        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(xb), src));
    const void* ks = reinterpret_cast<const void*>(
        __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(Kb), src));
    uint8_t* qs = reinterpret_cast<uint8_t*>(__shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(qb), src));
    uint8_t* ss = reinterpret_cast<uint8_t*>(__shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(sb), src));
    exact_block_warp<KSRC, NT, XG>(xs, ks, qs, ss, src);
  }
}

// The certified MXFP4 step of one block.  Y holds the fast fp32 y as pairs,
// amax = max|y| (NaN-propagating), and E = cfac * l1 + eabs bounds |y - y32|
// for every element, y32 being the definition's value; zero_block is the exact
// test that every input of the block is +-0 (then y = +0 when every matrix entry
// is finite).  exact_only sends every block, zero or not, to the exact path.  The
// scale is taken from amax only when amax - E and amax + E (directed rounding)
// give the same E8M0 byte; each code only when (y - E) 2^-e rounded down and
// (y + E) 2^-e rounded up give the same E2M1 code.  For a real block (act) the
// fast codes and scale are stored either way; the return value says whether the
// block is uncertain, in which case the caller must recompute it exactly and
// store over them (warp_exact_pass).  Keeping the recomputation out of this step
// leaves nothing of it on the per-block path but one vote.
__device__ __forceinline__ bool certify_store(const uint64_t (&Y)[16], float amax, float l1, bool zero_block,
                                              float cfac, float eabs, bool exact_only, bool act, uint8_t* qb,
                                              uint8_t* sb) {
  // zero_block: all inputs +-0, so every y is +0 by definition (byte 0, codes 0)
  const float E = __fmaf_ru(cfac, l1, eabs);
  bool exact = exact_only || !(amax <= FLT_MAX) || !(E <= FLT_MAX);
  const int byte = e8m0_byte(__fadd_ru(amax, E));
  if (byte != e8m0_byte(fmaxf(__fsub_rd(amax, E), 0.0f))) exact = true;
  const float s = inv_scale_of_byte(exact ? 0 : byte);
  const float eb = __fmul_ru(E, s);
  const uint64_t S2 = pk2(s, s), NE2 = pk2(-eb, -eb), PE2 = pk2(eb, eb);
  // eight elements at a time: the lower and upper bounds of each group are
  // converted while the other groups' pairs stay in registers
  uint32_t cm[4], cp[4];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    uint64_t V[4];
#pragma unroll
    for (int m = 0; m < 4; m++) V[m] = fma2_rd(Y[4 * k + m], S2, NE2);
    cm[k] = codes8(V);
#pragma unroll
    for (int m = 0; m < 4; m++) V[m] = fma2_ru(Y[4 * k + m], S2, PE2);
    cp[k] = codes8(V);
  }
  const uint32_t diff = (cm[0] ^ cp[0]) | (cm[1] ^ cp[1]) | (cm[2] ^ cp[2]) | (cm[3] ^ cp[3]);
  if (act) {
    const uint32_t keep = zero_block ? 0u : 0xFFFFFFFFu;
    *reinterpret_cast<uint4*>(qb) = make_uint4(cm[0] & keep, cm[1] & keep, cm[2] & keep, cm[3] & keep);
    *sb = uint8_t(zero_block ? 0 : byte);
  }
  // a block with an uncertain scale or an uncertain code is recomputed exactly;
  // with exact_only (matrix entries possibly non-finite) so is an all-zero block
  return act && (exact_only || (!zero_block && (exact || diff != 0u)));
}

}  // namespace kq
