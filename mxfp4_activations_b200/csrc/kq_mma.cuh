// kq_mma.cuh -- tensor-core (tcgen05) variant of the KroQuant quantizer.
//
// "KroQuant: Kronecker-Structured Block Transforms ...", Approach: the 32x32
// block transform is "applied as a single tensor-core GEMM per block" (the
// abstract: "the block-local structure runs as small tensor-core GEMMs").  Here
// each 32-element block of 128 rows is one UMMA chain: D[128 x 32] (fp32, in
// tensor memory) = X_b[128 x 32] (bf16, shared memory, K-major, 64-byte swizzle)
// x K_b[32 x 32] (bf16, shared memory, N-major, 64-byte swizzle).  For fp32
// matrices K_b is split exactly into three bf16 parts, K = hi + mid + lo
// (hi = bf16(K), mid = bf16(K - hi), lo = K - hi - mid), and the three products
// accumulate in the same tensor-memory columns, so the tensor core sees K32
// exactly; for bf16 matrices one part.
//
// CTA roles (a CTA owns a group of two 32-element block columns and a stride of
// 128-row tiles; three CTAs share an SM, 128 tensor-memory columns each; ten
// warps per CTA keep every SM sub-partition's register file within bounds):
//   warp 0      TMA producer: one 3-D load per tile (box {32, 128, 2}: each row
//               reads 128 contiguous bytes), no multicast; it starts streaming
//               while the other warps build the B operands
//   warp 1      allocates the tensor memory; one lane issues the UMMAs (2 or 6 per
//               block) and commits each tile to an mbarrier
//   warps 2-9   epilogue: warp w handles block (w-2)/4 of the tile for tensor-memory
//               lanes 32*(w%4)..+31.  As soon as the tile has landed it reads its
//               row's inputs from the staged tile (L1 bound and zero test) while the
//               UMMAs run; the stage is released by every epilogue warp plus a
//               commit of the UMMAs that read it.  Then tcgen05.ld of 32 fp32
//               columns per row, release of the accumulator buffer, and the
//               certified MXFP4 step shared with the butterfly kernel (kq_mx.cuh);
//               its rare exact recomputation re-reads x and K from global memory.
// Three tile stages and two accumulator buffers per CTA keep load, MMA and
// epilogue overlapped.  Every wait is bounded; on a timeout the CTA drains what it issued,
// frees its tensor memory and exits with the device error flag set.
#pragma once

#include <cuda_bf16.h>

#include "kq_common.cuh"
#include "kq_mx.cuh"

namespace kq {

constexpr int kMmaRows = 128;                        // UMMA M (rows per tile)
constexpr int kMmaWb = 2;                            // blocks per tile
constexpr int kMmaStages = 3;                        // tile stages
constexpr int kMmaAccBufs = 2;                       // accumulator buffers
constexpr int kMmaAccCols = kMmaWb * 32;             // columns per buffer
constexpr int kMmaTmemCols = kMmaAccBufs * kMmaAccCols;  // 128 of the SM's 512
constexpr int kMmaCtasPerSm = 3;
static_assert(kMmaTmemCols * kMmaCtasPerSm <= 512, "co-resident CTAs must fit the tensor memory");
static_assert((kMmaTmemCols & (kMmaTmemCols - 1)) == 0 && kMmaTmemCols >= 32, "tcgen05.alloc takes a power of 2 >= 32");
constexpr int kMmaEpiWarps = 4 * kMmaWb;             // one warp per (block, lane quarter)
constexpr int kMmaThreads = (2 + kMmaEpiWarps) * 32; // 320
constexpr int kMmaATileBytes = kMmaRows * 64;        // 8 KB per block of a tile
constexpr int kMmaAStageBytes = kMmaWb * kMmaATileBytes;  // 16 KB per tile
constexpr int kMmaBBytes = 32 * 64;                  // one 32x32 bf16 matrix
// Error allowance of the tensor-core sum, derived (not measured):
//   E = (C max|K| + kMmaErrL1) ||x||_1 + kMmaErrAbsK max|K| + kMmaErrAbs  >=  |y_fast - fp32(x K)|.
// Model: one kind::f16 UMMA (K = 16) forms d + sum of 16 products; every bf16 x bf16
// product is exact in fp32, and the 16 additions may run in any order, each rounded
// or truncated to at least 24 significant bits (relative error below 2u, u = 2^-24).
// Then |error| <= g (|d| + sum |p|) with g = 16 (2u) / (1 - 32u).  A block chains J
// UMMAs from d = 0 (J = 2 for bf16 K; J = 6 for fp32 K split exactly into three bf16
// parts, whose magnitudes add up to at most (1 + 2^-6) |K|), so the chain's error is
// at most J g (1 + g)^J sum_i |x_i| |K_ij|, and the definition's own rounding of y
// adds u |y|.  With sum_i |x_i||K_ij| <= ||x||_1 max|K|:
//   bf16 K: 2 g (1 + g)^2 + u < 65.1u  -> C = 66u
//   fp32 K: 6 g (1 + g)^6 (1 + 2^-6) + u < 196.1u -> C = 198u.
// Absolute terms for a tensor core that flushes fp32 subnormals: flushed K parts lose
// at most 3 x 2^-126 per unit of ||x||_1 (kMmaErrL1 = 2^-124); flushed subnormal
// inputs at most 32 x 2^-126 x (1 + 2^-6) max|K| (kMmaErrAbsK = 2^-120); flushed
// subnormal products and partial sums at most 2 x 96 x 2^-126 (kMmaErrAbs = 2^-118).
// A fast result that overflowed is non-finite and always takes the exact path.
// (Measured on B200 the worst error was 11u and 5.3u: the bound holds with room.)
constexpr float kMmaErrC_F32 = 1.1801719665527344e-05f;  // 198u
constexpr float kMmaErrC_BF16 = 3.933906555175781e-06f;  // 66u
constexpr float kMmaErrL1 = 4.701977403289208e-38f;      // 2^-124
constexpr float kMmaErrAbsK = 7.52316384526264e-37f;     // 2^-120
constexpr float kMmaErrAbs = 3.009265538105056e-36f;     // 2^-118

// UMMA instruction descriptor, kind::f16: D fp32, A and B bf16, A K-major,
// B N-major, N = 32, M = 128.
constexpr uint32_t kMmaIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((32u >> 3) << 17) |
                               ((128u >> 4) << 24);

struct MmaParams {
  const uint16_t* x;   // bf16 bits [M][ldx] (exact path)
  int64_t ldx;
  int64_t M;
  int nb;
  int n_row_tiles;
  int nsplit;          // 3 for fp32 matrices, 1 for bf16
  const void* mats;    // [nb][32][32] fp32 or bf16
  uint8_t* q;
  uint8_t* scales;     // row-major [M][nb], or tiled (scale_index)
};

// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), version 1, layout 4 = 64-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(4) << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kMmaIdesc), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; j++) v[j] = __uint_as_float(r[j]);
}

// Byte offset of element (row, col) of a [rows][32] bf16 tile with 64-byte
// rows under the 64-byte swizzle (16-byte chunk index ^= (row >> 1) & 3).
__device__ __forceinline__ uint32_t sw64_offset(int row, int col) {
  return uint32_t(row) * 64u + ((uint32_t(col >> 3) ^ (uint32_t(row >> 1) & 3u)) << 4) + uint32_t(col & 7) * 2u;
}

// Upper bound of sum_i |x_i| for the 32 bf16 values of one 64-byte row held as
// four 16-byte chunks: signs cleared, a tree of packed bf16 additions (each
// rounding to nearest: relative error at most 2^-8 per level, four levels plus
// one upward fp32 addition), then scaled up by 1 + 2^-5 > 1 / (1 - 2^-8)^4.
// Sums that land in the subnormal range may lose up to 2^-126 per addition;
// the absolute allowance kMmaErrAbsK max|K| covers that (C max|K| 2^-122 is far smaller).
__device__ __forceinline__ float l1_upper_bf16(const uint4 (&v)[4]) {
  uint32_t w[16];
#pragma unroll
  for (int k = 0; k < 4; k++) {
    w[4 * k] = v[k].x & 0x7FFF7FFFu;
    w[4 * k + 1] = v[k].y & 0x7FFF7FFFu;
    w[4 * k + 2] = v[k].z & 0x7FFF7FFFu;
    w[4 * k + 3] = v[k].w & 0x7FFF7FFFu;
  }
#pragma unroll
  for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
    for (int i = 0; i < n; i++) {
      uint32_t r;
      asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w[i]), "r"(w[i + n]));
      w[i] = r;
    }
  const float s = __fadd_ru(bf16lo(w[0]), bf16hi(w[0]));
  return __fmul_ru(s, 1.03125f);
}

template <int KSRC, int TILED>
__global__ void __launch_bounds__(kMmaThreads, kMmaCtasPerSm) quant_mma_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                   const MmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = base;                                   // [stages][Wb][128][64 B]
  uint8_t* b_smem = base + kMmaStages * kMmaAStageBytes;    // [Wb][nsplit][32][64 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_smem + kMmaWb * 3 * kMmaBBytes);
  uint64_t* full_a = bars;                                  // [stages]  TMA landed
  uint64_t* empty_a = bars + kMmaStages;                    // [stages]  epilogue read x, UMMAs done
  uint64_t* mma_full = bars + 2 * kMmaStages;               // [bufs]    accumulators ready
  uint64_t* tmem_empty = bars + 2 * kMmaStages + kMmaAccBufs;  // [bufs] accumulators read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMmaStages + 2 * kMmaAccBufs);
  uint32_t* kmax_bits = tmem_slot + 1;                      // [Wb] max |K| per block, as fp32 bits

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int group = blockIdx.x;
  const int my_tiles = (p.n_row_tiles - int(blockIdx.y) + int(gridDim.y) - 1) / int(gridDim.y);

  if (t == 0) {
    for (int s = 0; s < kMmaStages; s++) {
      mbar_init(&full_a[s], 1);
      mbar_init(&empty_a[s], kMmaEpiWarps + 1);  // every epilogue warp + the MMA commit
    }
    for (int i = 0; i < kMmaAccBufs; i++) {
      mbar_init(&mma_full[i], 1);
      mbar_init(&tmem_empty[i], kMmaEpiWarps);
    }
    fence_mbar_init();
  }
  if (t < kMmaWb) kmax_bits[t] = 0u;
  __syncthreads();
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream

  if (warp >= 1) {
    // B operands, built by the MMA and epilogue warps while the producer streams
    // A: this group's matrices split into bf16 parts in the 64-byte-swizzled
    // N-major layout; every load is issued before the first store.  max |K| per
    // block is reduced per warp, then one shared atomic.
    constexpr int kSetupThreads = kMmaThreads - 32;
    constexpr int kPer = (kMmaWb * 1024 + kSetupThreads - 1) / kSetupThreads;
    const int tt = t - 32;
    float kv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = tt + i * kSetupThreads;
      const int b = group * kMmaWb + (e >> 10);
      kv[i] = 0.0f;
      if (e < kMmaWb * 1024 && b < p.nb) {
        const int64_t idx = int64_t(b) * 1024 + (e & 1023);
        kv[i] = (KSRC == KSRC_BF16) ? bf16_to_f32(__ldg(static_cast<const unsigned short*>(p.mats) + idx))
                                    : __ldg(static_cast<const float*>(p.mats) + idx);
      }
    }
    uint32_t kloc[kMmaWb] = {};
#pragma unroll
    for (int i = 0; i < kPer; i++) {
      const int e = tt + i * kSetupThreads;
      if (e >= kMmaWb * 1024) continue;
      const int bw = e >> 10, r = (e >> 5) & 31, c = e & 31;
      const float kf = kv[i];
#pragma unroll
      for (int k = 0; k < kMmaWb; k++)
        if (k == bw) kloc[k] = max(kloc[k], __float_as_uint(kf) & 0x7FFFFFFFu);
      const uint32_t off = sw64_offset(r, c);
      uint8_t* mb = b_smem + bw * p.nsplit * kMmaBBytes;
      if (p.nsplit == 1) {
        *reinterpret_cast<__nv_bfloat16*>(mb + off) = __float2bfloat16_rn(kf);
      } else {
        const __nv_bfloat16 hi = __float2bfloat16_rn(kf);
        const float r1 = __fsub_rn(kf, __bfloat162float(hi));
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = __fsub_rn(r1, __bfloat162float(mid));
        *reinterpret_cast<__nv_bfloat16*>(mb + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(mb + kMmaBBytes + off) = mid;
        *reinterpret_cast<__nv_bfloat16*>(mb + 2 * kMmaBBytes + off) = __float2bfloat16_rn(r2);
      }
    }
#pragma unroll
    for (int k = 0; k < kMmaWb; k++) {
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, kloc[k]);
      if (lane == 0 && m != 0u) atomicMax(&kmax_bits[k], m);
    }
    if (warp == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                   "r"(uint32_t(kMmaTmemCols))
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B writes -> tensor core
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(kSetupThreads) : "memory");
    tc_fence_after();
  }
  const uint32_t tmem = warp >= 1 ? *tmem_slot : 0u;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      int it = 0;
      for (; it < my_tiles; it++) {
        const int s = it % kMmaStages;
        if (it >= kMmaStages &&
            !mbar_wait_bounded(&empty_a[s], uint32_t(it / kMmaStages - 1) & 1u, kWaitLimitNs))
          break;
        const int tile = int(blockIdx.y) + it * int(gridDim.y);
        mbar_arrive_expect_tx(&full_a[s], uint32_t(kMmaAStageBytes));
        tma_load_3d(a_smem + s * kMmaAStageBytes, &tmap, &full_a[s], 0, tile * kMmaRows, group * kMmaWb);
      }
      grid_launch_dependents();  // every load issued: the next grid may start its prologue
      if (it < my_tiles) {
        for (int k = (it > kMmaStages ? it - kMmaStages : 0); k < it; k++)
          mbar_wait_bounded(&full_a[k % kMmaStages], uint32_t(k / kMmaStages) & 1u, kWaitLimitNs / 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t b_base = smem_addr(b_smem);
      int it = 0;
      for (; it < my_tiles; it++) {
        const int s = it % kMmaStages, buf = it % kMmaAccBufs;
        if (!mbar_wait_bounded(&full_a[s], uint32_t(it / kMmaStages) & 1u, kWaitLimitNs)) break;
        if (it >= kMmaAccBufs &&
            !mbar_wait_bounded(&tmem_empty[buf], uint32_t(it / kMmaAccBufs - 1) & 1u, kWaitLimitNs))
          break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(a_smem + s * kMmaAStageBytes);
#pragma unroll
        for (int bw = 0; bw < kMmaWb; bw++) {
          const uint32_t d = tmem + uint32_t(buf * kMmaAccCols + bw * 32);
          for (int sp = 0; sp < p.nsplit; sp++) {
#pragma unroll
            for (int kh = 0; kh < 2; kh++) {
              const uint64_t ad = umma_desc(a_base + bw * kMmaATileBytes + kh * 32, 16, 512);
              const uint64_t bd = umma_desc(b_base + (bw * p.nsplit + sp) * kMmaBBytes + kh * 1024, 2048, 512);
              umma_bf16(d, ad, bd, (sp | kh) != 0 ? 1u : 0u);
            }
          }
        }
        umma_commit(&mma_full[buf]);
        umma_commit(&empty_a[s]);  // the stage is free for the producer once these UMMAs have read it
      }
      if (it > 0) {  // the last commit must have landed before tensor memory is freed
        const int k = it - 1;
        mbar_wait_bounded(&mma_full[k % kMmaAccBufs], uint32_t(k / kMmaAccBufs) & 1u, kWaitLimitNs / 4);
      }
      // the stage-release commits of the last tiles arrive asynchronously too: let
      // them land before the CTA's shared memory can be reused
      for (int k = (it > kMmaStages ? it - kMmaStages : 0); k < it; k++)
        mbar_wait_bounded(&empty_a[k % kMmaStages], uint32_t(k / kMmaStages) & 1u, kWaitLimitNs / 4);
    }
  } else {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;            // tensor-memory lane quarter
    const int bw = (warp - 2) >> 2;    // block of the tile
    const int rr = q * 32 + lane;      // row inside the tile
    const int sw = (rr >> 1) & 3;
    const int b = group * kMmaWb + bw;
    const bool col_ok = b < p.nb;
    const int bc = col_ok ? b : 0;
    const float kmax = __uint_as_float(kmax_bits[bw]);
    const float cfac = __fmaf_ru(KSRC == KSRC_BF16 ? kMmaErrC_BF16 : kMmaErrC_F32, kmax, kMmaErrL1);
    const float eabs = __fmaf_ru(kMmaErrAbsK, kmax, kMmaErrAbs);
    const void* Kb = (KSRC == KSRC_BF16)
                         ? static_cast<const void*>(static_cast<const uint16_t*>(p.mats) + int64_t(bc) * 1024)
                         : static_cast<const void*>(static_cast<const float*>(p.mats) + int64_t(bc) * 1024);
    for (int it = 0; it < my_tiles; it++) {
      const int s = it % kMmaStages, buf = it % kMmaAccBufs;
      // this row's inputs as soon as the tile has landed, overlapping the UMMAs:
      // L1 upper bound and exact zero test
      if (!mbar_wait_bounded(&full_a[s], uint32_t(it / kMmaStages) & 1u, kWaitLimitNs)) break;
      const uint4* xs = reinterpret_cast<const uint4*>(a_smem + s * kMmaAStageBytes + bw * kMmaATileBytes + rr * 64);
      float l1;
      bool zero_block;
      {
        uint4 xv[4];
#pragma unroll
        for (int k = 0; k < 4; k++) xv[k] = xs[k ^ sw];
        l1 = l1_upper_bf16(xv);
        uint32_t nz = 0u;
#pragma unroll
        for (int k = 0; k < 4; k++) nz |= xv[k].x | xv[k].y | xv[k].z | xv[k].w;
        zero_block = (nz & 0x7FFF7FFFu) == 0u;
      }
      stage_release(&empty_a[s], lane);
      if (!mbar_wait_bounded(&mma_full[buf], uint32_t(it / kMmaAccBufs) & 1u, kWaitLimitNs)) break;
      tc_fence_after();
      float y[32];
      tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(buf * kMmaAccCols + bw * 32), y);
      // the accumulators are no longer needed: release them before the math
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty[buf]);
      const int64_t row = int64_t(int(blockIdx.y) + it * int(gridDim.y)) * kMmaRows + rr;
      const bool act = col_ok && row < p.M;
      const int64_t rowc = act ? row : 0;
      uint64_t Y[16];
#pragma unroll
      for (int m2 = 0; m2 < 16; m2++) Y[m2] = pk2(y[2 * m2], y[2 * m2 + 1]);
      const float amax = block_amax(y);
      uint8_t* qb = p.q + rowc * int64_t(p.nb) * 16 + int64_t(bc) * 16;
      uint8_t* sb = p.scales + scale_index(rowc, bc, p.nb, TILED);
      const uint16_t* xb = p.x + rowc * p.ldx + int64_t(bc) * kBlock;
      const bool need = certify_store(Y, amax, l1, zero_block, cfac, eabs, !(cfac <= FLT_MAX), act, qb, sb);
      if (__any_sync(0xFFFFFFFFu, need)) warp_exact_pass<KSRC>(need, xb, Kb, qb, sb);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(uint32_t(kMmaTmemCols))
                 : "memory");
  }
}

}  // namespace kq
