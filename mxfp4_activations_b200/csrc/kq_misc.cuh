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

// One thread per (row, block): yhat = value(code) * 2^(byte-127); with inv
// (fp32 or bf16 [nb][32][32]) xhat_i = sum_j yhat_j inv[j][i], fp32 FMAs in j order.
__global__ void dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scales, int64_t M,
                               int nb, const void* __restrict__ inv, int inv_bf16, void* __restrict__ out,
                               int out_bf16) {
  const int64_t total = M * nb;
  for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < total;
       g += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = g / nb;
    const int b = int(g - row * nb);
    const uint4 cw = *reinterpret_cast<const uint4*>(q + g * 16);
    const float sc = scale_of_byte(scales[g]);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    float yh[32];
#pragma unroll
    for (int k = 0; k < 4; k++)
#pragma unroll
      for (int n = 0; n < 8; n++) yh[8 * k + n] = __fmul_rn(e2m1_value((words[k] >> (4 * n)) & 0xFu), sc);
    float xo[32];
    if (inv == nullptr) {
#pragma unroll
      for (int i = 0; i < 32; i++) xo[i] = yh[i];
    } else {
#pragma unroll
      for (int i = 0; i < 32; i++) xo[i] = 0.0f;
      for (int j = 0; j < 32; j++) {
        const int64_t off = (int64_t(b) * 32 + j) * 32;
#pragma unroll
        for (int i = 0; i < 32; i++) {
          const float kji = inv_bf16 ? bf16_to_f32(static_cast<const uint16_t*>(inv)[off + i])
                                     : static_cast<const float*>(inv)[off + i];
          xo[i] = __fmaf_rn(yh[j], kji, xo[i]);
        }
      }
    }
    if (out_bf16) {
      uint32_t pk[16];
#pragma unroll
      for (int h = 0; h < 16; h++) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(xo[2 * h], xo[2 * h + 1]);
        pk[h] = *reinterpret_cast<const uint32_t*>(&v);
      }
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + g * 32);
#pragma unroll
      for (int h = 0; h < 4; h++) o[h] = make_uint4(pk[4 * h], pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
    } else {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + g * 32);
#pragma unroll
      for (int h = 0; h < 8; h++) o[h] = make_float4(xo[4 * h], xo[4 * h + 1], xo[4 * h + 2], xo[4 * h + 3]);
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
