// kq_gemm.cuh -- W4A4 MXFP4 GEMM on the 5th-generation tensor cores (tcgen05,
// kind::mxf4 with block scaling), the consumer of the quantizer's output.
//
// "KroQuant: Kronecker-Structured Block Transforms ...", lead summary: W4A4
// MXFP4 inference; the activations are quantized with K_b and the weights with
// K_b^-T, so C = A_q . B_q^T approximates x . w^T.  Here
//   C[m][n] = sum_k value(A[m][k]) 2^(SA[m][k/32] - 127) value(B[n][k]) 2^(SB[n][k/32] - 127)
// with A [M][K] and B [N][K] as packed E2M1 codes (element 2j in the low nibble of
// byte j) and SA, SB as E8M0 scales in the 128 x 4 tiled layout that
// kq_quantize writes with KQ_SCALES_MMA_TILED.  The fp32 sum is the tensor core's.
//
// One CTA computes one 128 x 128 tile of C.  Warp 0 streams K in stages of 128
// elements: a 2-D TMA load of 128 rows x 64 bytes of A and of B (64-byte
// swizzle, no multicast) and two 512-byte bulk copies of the stage's scale tiles.
// One lane of warp 1 copies each stage's scale tiles into tensor memory
// (tcgen05.cp 32x128b, replicated to the four lane quarters, which is the layout
// the block-scaled MMA reads: lane quarter q finds the scales of its rows in word
// q, the k-block in the byte) and issues two MMAs of K = 64 per stage into one
// 128 x 128 fp32 accumulator in tensor memory.  Warps 2..5 then read the
// accumulator (one row per thread) and store C.  Every wait is bounded.
#pragma once

#include <cuda_bf16.h>

#include "kq_common.cuh"
#include "kq_mx.cuh"

namespace kq {

constexpr int kGmTile = 128;                  // rows of A and of B per tile (M = N = 128 per MMA)
constexpr int kGmKStage = 128;                // K elements per stage (64 bytes of codes per row)
constexpr int kGmStages = 6;               // 104 KB of stages: two CTAs per SM
constexpr int kGmABytes = kGmTile * 64;       // 8 KB of A codes per stage
constexpr int kGmBBytes = kGmTile * 64;       // 8 KB of B codes per stage
constexpr int kGmSfBytes = 512;               // one 128 x 4 scale tile
constexpr int kGmStageBytes = kGmABytes + kGmBBytes + 2 * kGmSfBytes;
constexpr int kGmThreads = 6 * 32;            // TMA warp, MMA warp, 4 epilogue warps
constexpr int kGmTmemCols = 256;              // accumulator 0..127; stage s scales of A at 128 + 8s, of B at 132 + 8s
constexpr int kGmSmemBytes = 1024 + kGmStages * kGmStageBytes + 256;

// Instruction descriptor of tcgen05.mma kind::mxf4 (block-scaled): A and B E2M1
// (format 1), K-major, E8M0 scales (bit 23), N = 128 (bits 17..22 hold N >> 3),
// M = 128 (bits 24..28 hold M >> 4), K = 64 (bit 31 clear); the byte of the
// scale word each operand starts from goes in bits 29..30 (A) and 4..5 (B).
__host__ __device__ constexpr uint32_t gemm_idesc(uint32_t sfa_byte, uint32_t sfb_byte) {
  return (sfb_byte << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) |
         (sfa_byte << 29);
}

struct GemmParams {
  const uint8_t* sa;  // tiled scales of A
  const uint8_t* sb;  // tiled scales of B
  void* c;
  int64_t M, N, K;
  int64_t ldc;        // elements between rows of C
  int c_bf16;
  int n_ktiles;       // ceil(K / 128)
  int k_tail_blocks;  // 32-element blocks in the last stage (1..4)
  int c_vec;          // C rows 16-byte aligned: full tiles store 16 bytes at a time
};

// Shared-memory matrix descriptor (sm_100): start, leading and stride byte offsets
// (16-byte units), descriptor version 1 (bit 46), layout type in bits 61..63.
__device__ __forceinline__ uint64_t gemm_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(layout) << 61);
}

__device__ __forceinline__ uint32_t bf16x2_bits(uint32_t lo, uint32_t hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(smem_dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

__global__ void __launch_bounds__(kGmThreads, 1) mxf4_gemm_kernel(const __grid_constant__ CUtensorMap tma_a,
                                                                  const __grid_constant__ CUtensorMap tma_b,
                                                                  const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kGmStages * kGmStageBytes);
  uint64_t* empty = full + kGmStages;
  uint64_t* acc_full = empty + kGmStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = int(blockIdx.x) * kGmTile, m0 = int(blockIdx.y) * kGmTile;
  const int64_t tile_row_a = m0 / kGmTile, tile_row_b = n0 / kGmTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(uint32_t(kGmTmemCols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();  // operands may come from the previous kernel in the stream

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tma_a);
      prefetch_tensormap(&tma_b);
      int kt = 0;
      for (; kt < p.n_ktiles; kt++) {
        const int s = kt % kGmStages;
        if (kt >= kGmStages && !mbar_wait_bounded(&empty[s], uint32_t(kt / kGmStages - 1) & 1u, kWaitLimitNs)) break;
        uint8_t* st = base + s * kGmStageBytes;
        mbar_arrive_expect_tx(&full[s], uint32_t(kGmStageBytes));
        tma_load_2d(st, &tma_a, &full[s], kt * 64, m0);
        tma_load_2d(st + kGmABytes, &tma_b, &full[s], kt * 64, n0);
        bulk_load(st + kGmABytes + kGmBBytes, p.sa + (tile_row_a * p.n_ktiles + kt) * kGmSfBytes, kGmSfBytes, &full[s]);
        bulk_load(st + kGmABytes + kGmBBytes + kGmSfBytes, p.sb + (tile_row_b * p.n_ktiles + kt) * kGmSfBytes,
                  kGmSfBytes, &full[s]);
      }
      grid_launch_dependents();
      // let copies still in flight land before the CTA can exit
      for (int k = (kt > kGmStages ? kt - kGmStages : 0); k < kt; k++)
        mbar_wait_bounded(&full[k % kGmStages], uint32_t(k / kGmStages) & 1u, kWaitLimitNs / 4);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int kt = 0;
      for (; kt < p.n_ktiles; kt++) {
        const int s = kt % kGmStages;
        if (!mbar_wait_bounded(&full[s], uint32_t(kt / kGmStages) & 1u, kWaitLimitNs)) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        uint8_t* stp = base + s * kGmStageBytes;
        const uint32_t st = smem_addr(stp);
        if (kt == p.n_ktiles - 1 && p.k_tail_blocks < 4) {
          // K ends inside this stage: the codes past it arrive as zeros (TMA fill), but
          // their scale bytes are padding the quantizer never wrote and may hold 0xFF
          // (NaN), which would turn 0 x scale into NaN.  Give them the finite byte 0.
          uint8_t* sf = stp + kGmABytes + kGmBBytes;
          for (int r = 0; r < 2 * kGmTile; r++)
            for (int c = p.k_tail_blocks; c < 4; c++) sf[(r >> 7) * kGmSfBytes + 16 * (r & 31) + 4 * ((r >> 5) & 3) + c] = 0;
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        const uint32_t sfa_col = tmem + 128 + 8 * s, sfb_col = sfa_col + 4;
        // scale tiles: 32 rows of 16 bytes, no swizzle (core matrices of 8 rows x 16 bytes
        // stacked every 128 bytes); each row lands in one lane of every lane quarter
        const uint64_t sda = gemm_sdesc(st + kGmABytes + kGmBBytes, 128, 128, 0);
        const uint64_t sdb = gemm_sdesc(st + kGmABytes + kGmBBytes + kGmSfBytes, 128, 128, 0);
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sfa_col), "l"(sda) : "memory");
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sfb_col), "l"(sdb) : "memory");
#pragma unroll
        for (int kh = 0; kh < 2; kh++) {
          // K-major 64-byte-swizzled rows of 64 bytes: 8-row groups 512 bytes apart,
          // K = 64 codes = 32 bytes per MMA
          const uint64_t ad = gemm_sdesc(st + kh * 32, 16, 512, 4);
          const uint64_t bd = gemm_sdesc(st + kGmABytes + kh * 32, 16, 512, 4);
          const uint32_t byte = uint32_t(2 * kh);  // k-blocks 2kh and 2kh + 1 of the stage
          const uint32_t idesc = gemm_idesc(byte, byte);
          const uint32_t accumulate = (kt > 0 || kh > 0) ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                  tmem),
              "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate), "r"(sfa_col | (byte << 30)), "r"(sfb_col | (byte << 30))
              : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_addr(&empty[s]))
                     : "memory");
      }
      if (ok)
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_addr(acc_full))
                     : "memory");
      // the stage-release commits arrive asynchronously: let them land before exit
      for (int k = (kt > kGmStages ? kt - kGmStages : 0); k < kt; k++)
        mbar_wait_bounded(&empty[k % kGmStages], uint32_t(k / kGmStages) & 1u, kWaitLimitNs / 4);
      if (ok) mbar_wait_bounded(acc_full, 0u, kWaitLimitNs / 4);
    }
  } else {
    // ------------------------------------------------ epilogue: one row of the tile per thread
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const int row = q * 32 + lane;
    if (mbar_wait_bounded(acc_full, 0u, kWaitLimitNs)) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int64_t m = int64_t(m0) + row;
#pragma unroll 1
      for (int c0 = 0; c0 < kGmTile; c0 += 32) {
        uint32_t v[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
            "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
              "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
              "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(tmem + (uint32_t(q * 32) << 16) + uint32_t(c0)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (m < p.M) {
          if (p.c_vec && n0 + kGmTile <= p.N) {
            if (p.c_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + m * p.ldc + n0 + c0);
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 w;
                w.x = bf16x2_bits(v[j], v[j + 1]);
                w.y = bf16x2_bits(v[j + 2], v[j + 3]);
                w.z = bf16x2_bits(v[j + 4], v[j + 5]);
                w.w = bf16x2_bits(v[j + 6], v[j + 7]);
                dst[j / 8] = w;
              }
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.c) + m * p.ldc + n0 + c0);
#pragma unroll
              for (int j = 0; j < 32; j += 4) dst[j / 4] = make_uint4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j++) {
              const int64_t n = int64_t(n0) + c0 + j;
              if (n >= p.N) break;
              if (p.c_bf16)
                static_cast<__nv_bfloat16*>(p.c)[m * p.ldc + n] = __float2bfloat16_rn(__uint_as_float(v[j]));
              else
                static_cast<float*>(p.c)[m * p.ldc + n] = __uint_as_float(v[j]);
            }
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(uint32_t(kGmTmemCols))
                 : "memory");
  }
}

}  // namespace kq
