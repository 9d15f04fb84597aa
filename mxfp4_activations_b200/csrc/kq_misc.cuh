// kq_misc.cuh -- dequantize (with optional inverse block transform) and the bare
// E2M1 element step.
#pragma once

#include <cuda_bf16.h>

#include "kq_common.cuh"

namespace kq {

// E2M1 magnitude of code bits 2..0 (exponent bias 1, one mantissa bit).
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = (e == 0u) ? 0.5f * float(m) : __uint_as_float((e + 126u) << 23) * (1.0f + 0.5f * float(m));
  return (code & 8u) ? -mag : mag;
}

// 2^(byte - 127) for byte in [0, 254] (2^-127 is an fp32 subnormal); NaN for 0xFF.
__device__ __forceinline__ float scale_of_byte(uint32_t byte) {
  if (byte == 0xFFu) return __uint_as_float(0x7FC00000u);
  if (byte == 0u) return __uint_as_float(0x00400000u);
  return __uint_as_float(byte << 23);
}

constexpr int kDqWarps = 8;  // warps per CTA of dequant_kernel
constexpr int kDqRows = 8;   // rows a warp has in flight

// CTA (b, g) handles block column b; its warp w takes the rows (g*8 + w)*8 + i,
// i < 8, then steps by gridDim.y*64 rows; lane l computes element l of each row:
// yhat_l = value(code_l) * 2^(byte-127).  The codes and scales of a warp's eight
// rows are loaded before any of them is used.  With inv (fp32 or bf16
// [nb][32][32]), lane i keeps column i of block b's inverse in registers (loaded
// once, one coalesced row of the matrix per step) and forms xhat_i = sum_j yhat_j
// inv[j][i] with fp32 FMAs in j order from +0, the row's yhat broadcast through
// shared memory.  Each row's 32 outputs are one contiguous store of the warp.
// INV: an inverse is applied (a template parameter, so the plain decode keeps few
// registers and many warps in flight).
template <int INV>
__global__ void __launch_bounds__(kDqWarps * 32, INV ? 2 : 3) dequant_kernel(
    const uint8_t* __restrict__ q, const uint8_t* __restrict__ scales, int64_t M, int nb,
    const void* __restrict__ inv, int inv_bf16, void* __restrict__ out, int out_bf16) {
  __shared__ __align__(16) float ys[kDqWarps][kBlock];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  float kcol[kBlock];
  if (INV) {
#pragma unroll
    for (int j = 0; j < kBlock; j++) {
      const int64_t off = (int64_t(b) * kBlock + j) * kBlock + lane;
      kcol[j] = inv_bf16 ? bf16_to_f32(static_cast<const uint16_t*>(inv)[off]) : static_cast<const float*>(inv)[off];
    }
  }
  const int64_t d = int64_t(nb) * kBlock;
  const int64_t step = int64_t(gridDim.y) * kDqWarps * kDqRows;
  for (int64_t r0 = (int64_t(blockIdx.y) * kDqWarps + warp) * kDqRows; r0 < M; r0 += step) {
    uint32_t w[kDqRows];
    uint32_t sc[kDqRows];
#pragma unroll
    for (int i = 0; i < kDqRows; i++) {
      const int64_t r = r0 + i < M ? r0 + i : r0;
      const int64_t g = r * nb + b;
      w[i] = reinterpret_cast<const uint32_t*>(q + g * 16)[lane >> 3];
      sc[i] = scales[g];
    }
#pragma unroll
    for (int i = 0; i < kDqRows; i++) {
      if (r0 + i >= M) break;
      const float yh = __fmul_rn(e2m1_value((w[i] >> (4 * (lane & 7))) & 0xFu), scale_of_byte(sc[i]));
      float xo = yh;
      if (INV) {
        ys[warp][lane] = yh;
        __syncwarp();
        const float4* yv = reinterpret_cast<const float4*>(ys[warp]);
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < kBlock / 4; k++) {
          const float4 v = yv[k];
          acc = __fmaf_rn(v.x, kcol[4 * k], acc);
          acc = __fmaf_rn(v.y, kcol[4 * k + 1], acc);
          acc = __fmaf_rn(v.z, kcol[4 * k + 2], acc);
          acc = __fmaf_rn(v.w, kcol[4 * k + 3], acc);
        }
        __syncwarp();  // the row's yhat is read by every lane before the next row overwrites it
        xo = acc;
      }
      const int64_t o = (r0 + i) * d + int64_t(b) * kBlock + lane;
      if (out_bf16)
        static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(xo);
      else
        static_cast<float*>(out)[o] = xo;
    }
  }
}

// out[k] = code(v[2k]) | code(v[2k+1]) << 4; one thread per 8 values, tail by pairs.
__global__ void e2m1_pack_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out) {
  const int64_t n8 = n / 8;
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < n8; g += int64_t(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(v)[2 * g];
    const float4 c = reinterpret_cast<const float4*>(v)[2 * g + 1];
    reinterpret_cast<uint32_t*>(out)[g] = e2m1x8(a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w);
  }
  if (blockIdx.x == 0) {
    for (int64_t k = n8 * 4 + threadIdx.x; k < n / 2; k += blockDim.x)
      out[k] = uint8_t(e2m1_one(v[2 * k]) | (e2m1_one(v[2 * k + 1]) << 4));
  }
}

}  // namespace kq
