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
// CTA roles (one CTA per 128-row tile x 4-block column group at a time):
//   warp 0     TMA producer: one 3-D load per tile (box {32, 128, 4}), no multicast
//   warp 1     allocates 256 tensor-memory columns, one lane issues the UMMAs
//              (2 or 6 per block) and commits them to an mbarrier
//   warps 2-9  epilogue: tcgen05.ld of 32 fp32 columns per row, the row's L1
//              norm from the staged tile, then the certified MXFP4 step shared
//              with the butterfly kernel (kq_mx.cuh).  Warp w reads tensor-memory
//              lanes 32*(w%4)..+31; warps w and w+4 take alternate blocks.
// Two A-tile stages and two accumulator buffers overlap load, MMA and epilogue.
// Every wait is bounded; on a timeout the CTA drains what it issued, frees its
// tensor memory and exits with the device error flag set.
#pragma once

#include <cuda_bf16.h>

#include "kq_common.cuh"
#include "kq_mx.cuh"

namespace kq {

constexpr int kMmaRows = 128;                        // UMMA M (rows per tile)
constexpr int kMmaWb = 4;                            // blocks per tile
constexpr int kMmaStages = 2;                        // A-tile stages
constexpr int kMmaAccCols = kMmaWb * 32;             // tensor-memory columns per accumulator buffer
constexpr int kMmaTmemCols = 2 * kMmaAccCols;        // two buffers: 256 columns
constexpr int kMmaEpiWarps = 8;
constexpr int kMmaThreads = (2 + kMmaEpiWarps) * 32; // 320
constexpr int kMmaATileBytes = kMmaRows * 64;        // 8 KB per block per tile
constexpr int kMmaAStageBytes = kMmaWb * kMmaATileBytes;
constexpr int kMmaBBytes = 32 * 64;                  // one 32x32 bf16 matrix
// Error allowance of the tensor-core sum relative to sum_i |x_i| max|K| (see
// DESIGN: accumulation-order model, checked on the device by the parity tests).
constexpr float kMmaErrC = 1.52587890625e-05f;       // 2^-16
constexpr float kMmaErrAbs = 7.703719777548943e-34f; // 2^-110: flushed subnormal partial sums

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
  uint8_t* scales;
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

template <int KSRC>
__global__ void __launch_bounds__(kMmaThreads, 2) quant_mma_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                   const MmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_smem = base;                                            // [stages][Wb][128][64 B]
  uint8_t* b_smem = base + kMmaStages * kMmaAStageBytes;             // [Wb][nsplit][32][64 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(b_smem + kMmaWb * 3 * kMmaBBytes);
  uint64_t* full_a = bars;                   // [stages]  TMA landed
  uint64_t* empty_a = bars + kMmaStages;     // [stages]  epilogue done with the tile
  uint64_t* mma_full = bars + 2 * kMmaStages;       // [2] accumulators ready
  uint64_t* tmem_empty = bars + 2 * kMmaStages + 2; // [2] accumulators read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMmaStages + 4);
  uint32_t* kmax_bits = tmem_slot + 1;       // [Wb] max |K| per block, as fp32 bits

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int group = blockIdx.x;
  const int my_tiles = (p.n_row_tiles - int(blockIdx.y) + int(gridDim.y) - 1) / int(gridDim.y);

  if (t == 0) {
    for (int s = 0; s < kMmaStages; s++) {
      mbar_init(&full_a[s], 1);
      mbar_init(&empty_a[s], kMmaEpiWarps);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&mma_full[b], 1);
      mbar_init(&tmem_empty[b], kMmaEpiWarps);
    }
    fence_mbar_init();
  }
  if (t < kMmaWb) kmax_bits[t] = 0u;
  __syncthreads();

  // B operands: this group's matrices, split into bf16 parts, written in the
  // 64-byte-swizzled N-major layout the descriptors describe.
  for (int e = t; e < kMmaWb * 1024; e += kMmaThreads) {
    const int bw = e >> 10, i = (e >> 5) & 31, j = e & 31;
    const int b = group * kMmaWb + bw;
    float kf = 0.0f;
    if (b < p.nb) {
      const int64_t idx = int64_t(b) * 1024 + (e & 1023);
      kf = (KSRC == KSRC_BF16) ? bf16_to_f32(static_cast<const uint16_t*>(p.mats)[idx])
                               : static_cast<const float*>(p.mats)[idx];
    }
    atomicMax(&kmax_bits[bw], __float_as_uint(fabsf(kf)) & 0x7FFFFFFFu);
    const uint32_t off = sw64_offset(i, j);
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(uint32_t(kMmaTmemCols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B writes -> tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

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
      if (it < my_tiles) {
        for (int k = (it > kMmaStages ? it - kMmaStages : 0); k < it; k++)
          mbar_wait_bounded(&full_a[k % kMmaStages], uint32_t(k / kMmaStages) & 1u, kWaitLimitNs / 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer
    if (lane == 0) {
      int it = 0;
      for (; it < my_tiles; it++) {
        const int s = it % kMmaStages, buf = it & 1;
        if (!mbar_wait_bounded(&full_a[s], uint32_t(it / kMmaStages) & 1u, kWaitLimitNs)) break;
        if (it >= 2 && !mbar_wait_bounded(&tmem_empty[buf], uint32_t(it / 2 - 1) & 1u, kWaitLimitNs)) break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(a_smem + s * kMmaAStageBytes);
        const uint32_t b_base = smem_addr(b_smem);
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
      }
      if (it > 0) {  // the last commit must have landed before tensor memory is freed
        const int k = it - 1;
        mbar_wait_bounded(&mma_full[k & 1], uint32_t(k / 2) & 1u, kWaitLimitNs / 4);
      }
    }
  } else {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int half = (warp - 2) >> 2;       // which alternate blocks
    const int rr = q * 32 + lane;           // row inside the tile
    for (int it = 0; it < my_tiles; it++) {
      const int s = it % kMmaStages, buf = it & 1;
      if (!mbar_wait_bounded(&mma_full[buf], uint32_t(it / 2) & 1u, kWaitLimitNs)) break;
      tc_fence_after();
      const int64_t row = int64_t(int(blockIdx.y) + it * int(gridDim.y)) * kMmaRows + rr;
      const uint8_t* a_stage = a_smem + s * kMmaAStageBytes;
#pragma unroll 1
      for (int bw = half; bw < kMmaWb; bw += 2) {
        const int b = group * kMmaWb + bw;
        const bool act = row < p.M && b < p.nb;
        float y[32];
        tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(buf * kMmaAccCols + bw * 32), y);
        // ||x||_1 of this row's block from the staged tile, rounded upward
        const uint4* xs = reinterpret_cast<const uint4*>(a_stage + bw * kMmaATileBytes + rr * 64);
        const int sw = (rr >> 1) & 3;
        float l1p[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const uint4 v = xs[k ^ sw];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; h++) {
            l1p[h] = __fadd_ru(l1p[h], fabsf(bf16lo(w[h])));
            l1p[h] = __fadd_ru(l1p[h], fabsf(bf16hi(w[h])));
          }
        }
        const float l1 = __fadd_ru(__fadd_ru(l1p[0], l1p[1]), __fadd_ru(l1p[2], l1p[3]));
        uint64_t Y[16];
#pragma unroll
        for (int m = 0; m < 16; m++) Y[m] = pk2(y[2 * m], y[2 * m + 1]);
        const float amax = block_amax(y);
        const float cfac = __fmul_ru(kMmaErrC, __uint_as_float(kmax_bits[bw]));
        const int64_t rowc = act ? row : 0;
        const int bc = act ? b : 0;
        const uint16_t* xb = p.x + rowc * p.ldx + int64_t(bc) * kBlock;
        const void* Kb = (KSRC == KSRC_BF16)
                             ? static_cast<const void*>(static_cast<const uint16_t*>(p.mats) + int64_t(bc) * 1024)
                             : static_cast<const void*>(static_cast<const float*>(p.mats) + int64_t(bc) * 1024);
        certify_store<KSRC>(Y, amax, l1, cfac, kMmaErrAbs, false, act, xb, Kb,
                            p.q + rowc * int64_t(p.nb) * 16 + int64_t(bc) * 16, p.scales + rowc * int64_t(p.nb) + bc);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tmem_empty[buf]);
        mbar_arrive(&empty_a[s]);
      }
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
