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
constexpr int kGmStages = 5;                  // 85 KB of stages + 16 KB of output staging: two CTAs per SM
constexpr int kGmABytes = kGmTile * 64;       // 8 KB of A codes per stage
constexpr int kGmBBytes = kGmTile * 64;       // 8 KB of B codes per stage
constexpr int kGmSfBytes = 512;               // one 128 x 4 scale tile
constexpr int kGmStageBytes = kGmABytes + kGmBBytes + 2 * kGmSfBytes;
constexpr int kGmThreads = 6 * 32;            // TMA warp, MMA warp, 4 epilogue warps
constexpr int kGmTmemCols = 256;              // accumulator 0..127; stage s scales of A at 128 + 8s, of B at 132 + 8s
// Output staging: each epilogue warp owns 4 KB of shared memory that feeds TMA tensor
// stores of 32 rows x 32 columns: two 2 KB buffers of 64-byte rows for bf16, one 4 KB
// buffer of 128-byte rows for fp32.
constexpr int kEpiWarpBytes = 4096;
constexpr int kEpiBytes = 4 * kEpiWarpBytes;
constexpr int kGmSmemBytes = 1024 + kGmStages * kGmStageBytes + kEpiBytes + 256;

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
  int c_tma;          // C is written by TMA tensor stores (16-byte aligned rows)
  int n_ktiles;       // ceil(K / 128)
  int k_tail_blocks;  // 32-element blocks in the last stage (1..4)
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

// 32 consecutive 32-bit columns of this thread's tensor-memory lane, without waiting:
// the registers are valid after tcgen05.wait::ld.
__device__ __forceinline__ void tmem_ld32x32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's tensor-memory lane (waits for them).
__device__ __forceinline__ void tmem_ld32x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Non-blocking test of an mbarrier phase (acquire semantics when it reports completion).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// TMA tensor store from shared memory, tracked by this thread's bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_addr(smem_src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Where an epilogue writes C.
struct GemmOut {
  void* c;
  int64_t M, N, ldc;
  int bf16;
  int tma;
};

// One warp's 32 rows x 32 columns of C (row row0 + lane, columns col0..col0+31) from
// fp32 bits in registers.  With the tensor map: through the warp's swizzled staging
// buffer (64- or 128-byte swizzle, matching the map) to a TMA tensor store, which
// clips rows and columns past C; a buffer is refilled once the store issued from it
// has read it.  Without: plain stores with bounds checks.
__device__ __forceinline__ void epi_chunk(const GemmOut& o, const CUtensorMap* cmap, uint8_t* bufs, int& nbuf,
                                          const uint32_t (&v)[32], int lane, int64_t row0, int64_t col0) {
  if (row0 >= o.M || col0 >= o.N) return;  // warp-uniform: nothing of the chunk lies in C
  if (o.tma) {
    uint8_t* buf = o.bf16 ? bufs + (nbuf & 1) * 2048 : bufs;
    if (lane == 0) {
      if (o.bf16)
        bulk_wait_read<1>();
      else
        bulk_wait_read<0>();
    }
    __syncwarp();
    if (o.bf16) {
      uint8_t* row = buf + lane * 64;
      const int sw = (lane >> 1) & 3;
#pragma unroll
      for (int j = 0; j < 4; j++)
        *reinterpret_cast<uint4*>(row + 16 * (j ^ sw)) =
            make_uint4(bf16x2_bits(v[8 * j], v[8 * j + 1]), bf16x2_bits(v[8 * j + 2], v[8 * j + 3]),
                       bf16x2_bits(v[8 * j + 4], v[8 * j + 5]), bf16x2_bits(v[8 * j + 6], v[8 * j + 7]));
    } else {
      uint8_t* row = buf + lane * 128;
      const int sw = lane & 7;
#pragma unroll
      for (int j = 0; j < 8; j++)
        *reinterpret_cast<uint4*>(row + 16 * (j ^ sw)) = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(cmap, buf, int(col0), int(row0));
      bulk_commit();
    }
    nbuf++;
  } else {
    const int64_t m = row0 + lane;
    if (m < o.M) {
#pragma unroll
      for (int j = 0; j < 32; j++) {
        const int64_t n = col0 + j;
        if (n >= o.N) break;
        if (o.bf16)
          static_cast<__nv_bfloat16*>(o.c)[m * o.ldc + n] = __float2bfloat16_rn(__uint_as_float(v[j]));
        else
          static_cast<float*>(o.c)[m * o.ldc + n] = __uint_as_float(v[j]);
      }
    }
  }
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
                                                                  const __grid_constant__ CUtensorMap tma_c,
                                                                  const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = base + kGmStages * kGmStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiBytes);
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
    // ------------------------------------------------ epilogue: warp w reads lane quarter w % 4
    const int q = warp & 3;  // tensor-memory lane quarter this warp may access
    const GemmOut o{p.c, p.M, p.N, p.ldc, p.c_bf16, p.c_tma};
    uint8_t* bufs = epi + (warp - 2) * kEpiWarpBytes;
    int nbuf = 0;
    if (mbar_wait_bounded(acc_full, 0u, kWaitLimitNs)) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
      for (int c0 = 0; c0 < kGmTile; c0 += 32) {
        uint32_t v[32];
        tmem_ld32x32(tmem + (uint32_t(q * 32) << 16) + uint32_t(c0), v);
        epi_chunk(o, &tma_c, bufs, nbuf, v, lane, int64_t(m0) + q * 32, int64_t(n0) + c0);
      }
    }
    if (lane == 0) bulk_wait<0>();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(uint32_t(kGmTmemCols))
                 : "memory");
  }
}


// ---------------------------------------------------------------------------------------
// Two-SM variant (tcgen05 cta_group::2): a cluster of two CTAs on the two SMs of a TPC
// computes 256 x 256 tiles of C.  CTA r of the pair holds rows 128r..128r+127 of the
// tile's A rows and of its B rows in its own shared memory; the pair's MMAs
// (M = 256, N = 256, K = 64), issued by CTA 0, read both halves, and CTA r's tensor
// memory accumulates its 128 rows of C against all 256 columns.  Per SM this moves
// half the operand bytes per flop of the one-SM kernel.  Scales: each CTA stages its
// own 128 rows of A scales and the scales of all 256 B rows; one tcgen05.cp of the
// pair copies every CTA's stage into its own tensor memory.  The kernel is
// persistent: the clusters walk the tiles (row band by row band), the stage ring
// runs on across tiles, and the epilogue hands the accumulator back to the MMA
// issuer as soon as it has read it (bf16 output, kept packed in registers) so the
// next tile's products overlap the previous tile's stores.  Needs K % 128 == 0.
//
// Synchronisation.  full[s] lives in CTA 0: its producer expects the stage bytes of
// both CTAs, and the TMA loads of both (cta_group::2 form, no multicast) complete
// on it.  empty[s] and acc_full exist in both CTAs; the MMA issuer's commits arrive
// on both (tcgen05.commit multicast to the pair).  acc_empty lives in CTA 0 and
// counts the epilogue warps of both CTAs.  A cluster barrier follows the barrier
// set-up and precedes the release of tensor memory.

constexpr int kG2EpiWarps = 8;                               // two per lane quarter, 128 columns each
constexpr int kG2Threads = (2 + kG2EpiWarps) * 32;

// Stage geometry of the two-SM kernel for KS K-elements per stage (128 or 256): rows
// of KS/2 bytes of codes with the matching swizzle (64 or 128 bytes), KS/128 scale
// tiles of 128 x 4 per 128 rows.
template <int KS>
struct G2Cfg {
  static constexpr int kRowBytes = KS / 2;
  static constexpr int kTiles = KS / 128;                    // scale tiles per 128 rows per stage
  static constexpr int kMmas = KS / 64;                      // K = 64 per MMA
  static constexpr int kABytes = 128 * kRowBytes;
  static constexpr int kBBytes = 128 * kRowBytes;
  static constexpr int kSfaOff = kABytes + kBBytes;          // A scales of this CTA's 128 rows
  static constexpr int kSfbOff = kSfaOff + 512 * kTiles;     // B scales of all 256 rows
  static constexpr int kStageBytes = kSfbOff + 1024 * kTiles;
  static constexpr int kStages = KS == 128 ? 8 : 5;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kG2EpiWarps * kEpiWarpBytes + 256;
  static constexpr int kSfCols = 12 * kTiles;                // per stage: 4 per A tile, 8 per B tile pair
  static constexpr uint32_t kLayout = KS == 128 ? 4u : 2u;   // 64- or 128-byte swizzle
  static constexpr uint32_t kSbo = 8 * kRowBytes;            // 8-row core-matrix group
  static_assert(kStageBytes % kSbo == 0, "stages must keep the swizzle atoms aligned");
  static_assert(256 + kStages * kSfCols <= 512, "scale columns must fit beside the accumulator");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

constexpr int kG2TmemCols = 512;                             // accumulator 0..255, scales from 256

// M = 256 (cta_group::2), N = 256, otherwise as gemm_idesc.
__host__ __device__ constexpr uint32_t gemm2_idesc(uint32_t sf_byte) {
  return (sf_byte << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | (1u << 23) | ((256u >> 4) << 24) |
         (sf_byte << 29);
}

struct Gemm2Params {
  void* c;
  int64_t M, N;
  int64_t ldc;
  int c_bf16;
  int c_tma;     // C is written by TMA tensor stores (16-byte aligned rows)
  int n_ktiles;  // K / KS
  int n_ctiles;  // K / 128: scale tiles per 128 rows
  int tiles_m;   // ceil(M / 256)
  int tiles_n;   // ceil(N / 256)
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared-memory address, in the cluster window, of the same variable in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
  return a;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// 2-D TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier that may sit in the peer CTA of the pair (cluster-window address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t cluster_bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void pair_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"(uint16_t(3))
      : "memory");
}

// One stage's scale tiles from both CTAs' shared memory into their tensor memory:
// A tile c to sfa + 4c, B tiles of tile column c (rows 0..127, 128..255) to sfb + 8c
// and sfb + 8c + 4.  Scale tiles are 32 rows of 16 bytes, no swizzle (core matrices of
// 8 rows x 16 bytes stacked every 128 bytes); each row lands in one lane of every
// lane quarter.
template <class C>
__device__ __forceinline__ void pair_scale_copies(uint64_t sfa_desc, uint64_t sfb_desc, uint32_t sfa_col,
                                                  uint32_t sfb_col) {
  // sfa_desc / sfb_desc: descriptors of the stage's first A and B scale tiles; tiles are
  // 512 bytes (32 in the descriptor's 16-byte address units) apart
#pragma unroll
  for (int c = 0; c < C::kTiles; c++) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(sfa_col + 4 * c),
                 "l"(sfa_desc + uint64_t(32 * c))
                 : "memory");
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(sfb_col + 8 * c),
                 "l"(sfb_desc + uint64_t(32 * c))
                 : "memory");
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(sfb_col + 8 * c + 4),
                 "l"(sfb_desc + uint64_t(32 * (C::kTiles + c)))
                 : "memory");
  }
}

template <int KS>
__global__ void __launch_bounds__(kG2Threads, 1)
    mxf4_gemm2_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                      const __grid_constant__ CUtensorMap tma_sa, const __grid_constant__ CUtensorMap tma_sb,
                      const __grid_constant__ CUtensorMap tma_c, const Gemm2Params p) {
  using C = G2Cfg<KS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = base + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kG2EpiWarps * kEpiWarpBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_clusters = int(gridDim.x) / 2, cid = int(blockIdx.x) / 2;
  const int n_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kG2EpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(uint32_t(kG2TmemCols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anything can arrive on them
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      prefetch_tensormap(&tma_a);
      prefetch_tensormap(&tma_b);
      prefetch_tensormap(&tma_sa);
      prefetch_tensormap(&tma_sb);
      const uint32_t full0 = cluster_addr(&full[0], 0);
      int it = 0;
      bool ok = true;
      for (int t = cid; t < n_tiles && ok; t += n_clusters) {
        const int tm = t / p.tiles_n, tn = t % p.tiles_n;
        const int arow = tm * 256 + 128 * int(rank), brow = tn * 256 + 128 * int(rank);
        const int sfa_tile = tm * 2 + int(rank), sfb_tile = tn * 2;
        for (int kt = 0; kt < p.n_ktiles; kt++, it++) {
          const int s = it % C::kStages;
          if (it >= C::kStages && !mbar_test(&empty[s], uint32_t(it / C::kStages - 1) & 1u) &&
              (*abort_flag || !mbar_wait_bounded(&empty[s], uint32_t(it / C::kStages - 1) & 1u, kWaitLimitNs))) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = base + s * C::kStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], uint32_t(2 * C::kStageBytes));
          const uint32_t bar = full0 + uint32_t(s) * 8u;
          const int ct = C::kTiles * kt;  // first scale tile column of the stage
          tma_load_2d_pair(st, &tma_a, bar, kt * C::kRowBytes, arow);
          tma_load_2d_pair(st + C::kABytes, &tma_b, bar, kt * C::kRowBytes, brow);
          tma_load_2d_pair(st + C::kSfaOff, &tma_sa, bar, 0, 2 * (sfa_tile * p.n_ctiles + ct));
          tma_load_2d_pair(st + C::kSfbOff, &tma_sb, bar, 0, 2 * (sfb_tile * p.n_ctiles + ct));
          tma_load_2d_pair(st + C::kSfbOff + 512 * C::kTiles, &tma_sb, bar, 0,
                           2 * ((sfb_tile + 1) * p.n_ctiles + ct));
        }
      }
      grid_launch_dependents();
      // the pair's MMAs read this CTA's last stages: wait for their release
      for (int k = (it > C::kStages ? it - C::kStages : 0); k < it; k++)
        mbar_wait_bounded(&empty[k % C::kStages], uint32_t(k / C::kStages) & 1u, kWaitLimitNs / 4);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (CTA 0 of the pair)
    if (rank == 0 && lane == 0) {
      int it = 0, tl = 0;
      bool ok = true;
      // Descriptors of stage 0; another stage or K step differs only in the start-address
      // field (16-byte units, below 2^14 for every address in this CTA's shared memory),
      // so they are formed once and offset by an add.
      const uint32_t st0 = smem_addr(base);
      const uint64_t a_desc0 = gemm_sdesc(st0, 16, C::kSbo, C::kLayout);
      const uint64_t b_desc0 = gemm_sdesc(st0 + C::kABytes, 16, C::kSbo, C::kLayout);
      const uint64_t sfa_desc0 = gemm_sdesc(st0 + C::kSfaOff, 128, 128, 0);
      const uint64_t sfb_desc0 = gemm_sdesc(st0 + C::kSfbOff, 128, 128, 0);
      constexpr uint64_t kStageUnits = uint64_t(C::kStageBytes >> 4);
      for (int t = cid; t < n_tiles && ok; t += n_clusters, tl++) {
        if (tl > 0 && (*abort_flag || !mbar_wait_bounded(acc_empty, uint32_t(tl - 1) & 1u, kWaitLimitNs))) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // The issuing thread is held by the tensor pipe while it issues a stage, so
        // the next stage's barrier is tested (without blocking) before that, and the
        // full wait with its time-outs runs only when the test found it incomplete.
        bool ready = mbar_test(&full[it % C::kStages], uint32_t(it / C::kStages) & 1u);
        for (int kt = 0; kt < p.n_ktiles; kt++, it++) {
          const int s = it % C::kStages;
          if (!ready &&
              (*abort_flag || !mbar_wait_bounded(&full[s], uint32_t(it / C::kStages) & 1u, kWaitLimitNs))) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          ready = kt + 1 < p.n_ktiles &&
                  mbar_test(&full[(it + 1) % C::kStages], uint32_t((it + 1) / C::kStages) & 1u);
          const uint64_t so = kStageUnits * uint64_t(s);
          const uint32_t sfa_col = tmem + 256 + uint32_t(C::kSfCols * s), sfb_col = sfa_col + 4 * C::kTiles;
          pair_scale_copies<C>(sfa_desc0 + so, sfb_desc0 + so, sfa_col, sfb_col);
#pragma unroll
          for (int j = 0; j < C::kMmas; j++) {
            const uint64_t ad = a_desc0 + so + uint64_t(2 * j);  // K step j: 32 bytes further
            const uint64_t bd = b_desc0 + so + uint64_t(2 * j);
            const uint32_t byte = uint32_t(2 * (j & 1));
            const uint32_t accumulate = (kt > 0 || j > 0) ? 1u : 0u;
            const uint32_t sfa = (sfa_col + 4 * (j >> 1)) | (byte << 30);
            const uint32_t sfb = (sfb_col + 8 * (j >> 1)) | (byte << 30);
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                    tmem),
                "l"(ad), "l"(bd), "r"(gemm2_idesc(byte)), "r"(accumulate), "r"(sfa), "r"(sfb)
                : "memory");
          }
          pair_commit(&empty[s]);
        }
        if (!ok) break;
        pair_commit(acc_full);
      }
      for (int k = (it > C::kStages ? it - C::kStages : 0); k < it; k++)
        mbar_wait_bounded(&empty[k % C::kStages], uint32_t(k / C::kStages) & 1u, kWaitLimitNs / 4);
      if (ok && tl > 0) mbar_wait_bounded(acc_empty, uint32_t(tl - 1) & 1u, kWaitLimitNs / 4);
    }
  } else {
    // ------------------------------------------------ epilogue (both CTAs): warp w reads lane quarter w % 4,
    // columns 128 h .. 128 h + 127 with h = (w - 2) / 4
    const int q = warp & 3, h = (warp - 2) >> 2;
    const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + uint32_t(128 * h);
    const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
    const GemmOut o{p.c, p.M, p.N, p.ldc, p.c_bf16, p.c_tma};
    uint8_t* bufs = epi + (warp - 2) * kEpiWarpBytes;
    int nbuf = 0;
    int tl = 0;
    for (int t = cid; t < n_tiles; t += n_clusters, tl++) {
      if (*abort_flag || !mbar_wait_bounded(acc_full, uint32_t(tl) & 1u, kWaitLimitNs)) {
        *abort_flag = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int tm = t / p.tiles_n, tn = t % p.tiles_n;
      const int64_t row0 = int64_t(tm) * 256 + 128 * int(rank) + q * 32;
      const int64_t col0 = int64_t(tn) * 256 + 128 * h;
      // drain this warp's 32 x 128 block of the accumulator at once, then hand the
      // accumulator back so the next tile's products overlap these stores
      uint32_t v[4][32];
#pragma unroll
      for (int c = 0; c < 4; c++) tmem_ld32x32_nowait(tbase + uint32_t(32 * c), v[c]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
#pragma unroll
      for (int c = 0; c < 4; c++) epi_chunk(o, &tma_c, bufs, nbuf, v[c], lane, row0, col0 + 32 * c);
    }
    if (lane == 0) bulk_wait<0>();
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  cluster_sync_all();  // no CTA of the pair leaves while the other may still touch its memory
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(uint32_t(kG2TmemCols))
                 : "memory");
  }
}

}  // namespace kq
