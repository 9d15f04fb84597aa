// kq_lib.cu -- C ABI of libkq (declared in include/kq.h): argument checks,
// launch configuration and tensor-map set-up for the sm_100a kernels.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "kq.h"
#include "kq_common.cuh"
#include "kq_adaln.cuh"
#include "kq_expand.cuh"
#include "kq_gemm.cuh"
#include "kq_misc.cuh"
#include "kq_mma.cuh"
#include "kq_quant.cuh"

namespace {

constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

cudaStream_t as_cuda(kq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Description of the last failing CUDA call on this thread (kq_last_error).
thread_local char g_last_error[256] = "no error";

kq_status cuda_fail(const char* what, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", what, cudaGetErrorString(e), int(e));
  cudaGetLastError();  // do not leave a stale error for the next call
  return KQ_ERR_CUDA;
}

kq_status launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KQ_OK : cuda_fail(what, e);
}

// ---- per-device facts, cached
struct DeviceInfo {
  std::once_flag once;
  int sms = 0;
  int smem_optin = 0;
  int smem_per_sm = 0;
  bool ok = false;
};
DeviceInfo g_dev[kMaxDevices];

const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&]() {
    d.ok = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess;
  });
  return d.ok ? &d : nullptr;
}

// ---- cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// ---- launch with programmatic stream serialization: the kernel may start its
// prologue while the previous kernel in the stream finishes; it waits for that
// kernel's completion (griddepcontrol.wait) before reading global memory.
template <typename... Args>
kq_status launch_pdl(void (*kern)(Args...), dim3 grid, int threads, int smem, cudaStream_t stream, const char* what,
                     const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(unsigned(threads));
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  return e == cudaSuccess ? launch_status(what) : cuda_fail(what, e);
}

// ---- launch of the butterfly / comparison quantizer kernels

// Resident CTAs per SM of a kernel launched with `threads` threads and `smem`
// bytes of dynamic shared memory (the occupancy query, cached per kernel and device).
kq_status resident_ctas(const void* kern, int threads, int smem, int devid, int* out) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({kern, devid});
  if (it != cache.end()) {
    *out = it->second;
    return KQ_OK;
  }
  int per_sm = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
  if (per_sm < 1) return cuda_fail("occupancy: no resident CTA", cudaErrorInvalidConfiguration);
  cache[{kern, devid}] = per_sm;
  *out = per_sm;
  return KQ_OK;
}

// Lane layout of the streaming quantizer: every lane owns one block column and
// walks rows r0, r0 + k, ...; one wave of resident threads takes the lanes.
// k is the largest row count that fits the wave, then lowered to the smallest
// value with the same number of row steps (same makespan, fewer threads).  When
// the block columns alone exceed the wave, k = 1 and threads walk several lanes.
void lane_layout(int64_t M, int64_t nb, int64_t slots, kq::QuantParams& p) {
  if (nb <= slots) {
    int64_t k = slots / nb;
    if (k > M) k = M;
    const int64_t n_iter = (M + k - 1) / k;
    k = (M + n_iter - 1) / n_iter;
    p.k = k;
    p.n_iter = n_iter;
    p.lanes = k * nb;
    p.threads = p.lanes;
    p.passes = 1;
  } else {
    p.k = 1;
    p.n_iter = M;
    p.lanes = nb;
    p.threads = slots;
    p.passes = int((nb + slots - 1) / slots);
  }
}

// The AdaLN fields of the quantizer's ADALN form (kq_adaln_quantize given stats).
struct AdaLnInput {
  const float* stats = nullptr;
  const uint16_t* shift = nullptr;
  const uint16_t* scale = nullptr;
  int64_t rows_per_group = 1;
};

template <int MODE, int TILED, int NT, bool ADALN, bool GROUPED>
kq_status launch_quant_impl(const void* x, int64_t M, int64_t d, int64_t ldx, const float* mats,
                            const float* factored, const float* inv_s, uint8_t* q, uint8_t* scales,
                            cudaStream_t stream, const AdaLnInput& ada) {
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  int devid = 0;
  cudaGetDevice(&devid);
  const int64_t nb = d / 32;
  void (*kern)(const kq::QuantParams) = kq::quant_kernel<MODE, TILED, NT, ADALN, GROUPED>;
  constexpr int smem = kq::quant_smem_bytes(ADALN, GROUPED);
  static std::atomic<int> attr_set[kMaxDevices];
  if (!attr_set[devid].load()) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
    attr_set[devid].store(1);
  }
  int per_sm = 0;
  kq_status st = resident_ctas(reinterpret_cast<const void*>(kern), kq::kSThreads, smem, devid, &per_sm);
  if (st != KQ_OK) return st;

  kq::QuantParams p;
  p.stats = ada.stats;
  p.shift = ada.shift;
  p.scale = ada.scale;
  p.rows_per_group = ada.rows_per_group;
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.M = M;
  p.nb = int(nb);
  p.mats = mats;
  p.factored = factored;
  p.inv_s = inv_s;
  p.q = q;
  p.scales = scales;
  p.cg = 0;
  int64_t grid = 0;
  if (GROUPED) {
    // CTAs of 8 row residues x one group of 32 columns: fill the resident slots once
    // (at least one CTA row), then lower the residue count k to the smallest with the same
    // number of row steps, as lane_layout does
    constexpr int64_t kWarps = kq::kSThreads / 32;
    const int64_t cg = nb / 32;
    const int64_t krow = std::max<int64_t>(1, int64_t(dev->sms) * per_sm / cg);
    int64_t k = std::min<int64_t>(krow * kWarps, M);
    p.n_iter = (M + k - 1) / k;
    k = (M + p.n_iter - 1) / p.n_iter;
    p.cg = int(cg);
    p.k = k;
    p.lanes = k * nb;
    p.passes = 1;
    grid = (k + kWarps - 1) / kWarps * cg;
    p.threads = grid * kq::kSThreads;
  } else {
    lane_layout(M, nb, int64_t(dev->sms) * per_sm * kq::kSThreads, p);
    grid = (p.threads + kq::kSThreads - 1) / kq::kSThreads;
  }
  return launch_pdl(kern, dim3(unsigned(grid)), kq::kSThreads, smem, stream, "quant_kernel launch", p);
}

// Row steps per thread from which the grouped layout is taken.  Measured back to back at
// M = 4608: 24 steps (d = 12288) 37.4 against 38.1 us; 6 steps (d = 3072) 17.9 against
// 17.0 us, where the layout's start (the shared table's fill and one barrier) is not
// amortised.  The AdaLN form was slower grouped at both widths (105.5 against 102.2 us).
constexpr int64_t kGroupedMinSteps = 16;

// The butterfly / comparison quantizer kernels.  KroQuant with 32-element blocks takes the
// grouped layout when d is a multiple of 1024 (whole groups of 32 block columns) and each
// thread walks at least kGroupedMinSteps rows.
template <int MODE, int TILED, int NT = 32, bool ADALN = false>
kq_status launch_quant(const void* x, int64_t M, int64_t d, int64_t ldx, const float* mats, const float* factored,
                       const float* inv_s, uint8_t* q, uint8_t* scales, cudaStream_t stream,
                       const AdaLnInput& ada = AdaLnInput()) {
  if constexpr (MODE == kq::MODE_KRON && NT == 32 && !ADALN) {
    const int64_t nb = d / 32;
    const DeviceInfo* dev = device_info();
    if (nb % 32 == 0 && dev != nullptr) {
      int devid = 0;
      cudaGetDevice(&devid);
      void (*gkern)(const kq::QuantParams) = kq::quant_kernel<MODE, TILED, NT, false, true>;
      constexpr int gsmem = kq::quant_smem_bytes(false, true);
      static std::atomic<int> gattr_set[kMaxDevices];
      if (!gattr_set[devid].load()) {  // before the occupancy query, which counts the shared memory
        const cudaError_t e = cudaFuncSetAttribute(gkern, cudaFuncAttributeMaxDynamicSharedMemorySize, gsmem);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
        gattr_set[devid].store(1);
      }
      int per_sm = 0;
      const kq_status st = resident_ctas(reinterpret_cast<const void*>(gkern), kq::kSThreads, gsmem, devid, &per_sm);
      if (st != KQ_OK) return st;
      const int64_t krow = std::max<int64_t>(1, int64_t(dev->sms) * per_sm / (nb / 32));
      const int64_t k = std::min<int64_t>(krow * (kq::kSThreads / 32), M);
      if ((M + k - 1) / k >= kGroupedMinSteps)
        return launch_quant_impl<MODE, TILED, NT, ADALN, true>(x, M, d, ldx, mats, factored, inv_s, q, scales,
                                                               stream, ada);
    }
  }
  return launch_quant_impl<MODE, TILED, NT, ADALN, false>(x, M, d, ldx, mats, factored, inv_s, q, scales, stream,
                                                          ada);
}

// Row-tile stride for a grid of ncol column groups on sms SMs holding per_sm
// CTAs each: fill the resident slots once, then balance the row tiles.
int64_t row_stride(int64_t ncol, int64_t nrt, int sms, int per_sm) {
  const int64_t slots = int64_t(sms) * per_sm;
  int64_t gy = slots / ncol;
  if (gy < 1) gy = 1;
  if (gy > nrt) gy = nrt;
  // same makespan (row tiles per CTA) with fewer CTAs: drop the surplus
  const int64_t per = (nrt + gy - 1) / gy;
  gy = (nrt + per - 1) / per;
  if (gy > 65535) gy = 65535;
  return gy;
}

// Tensor-core variant: 128-row x 4-block tiles, one CTA per 4-block column group
// and row-tile stride, two CTAs per SM (256 tensor-memory columns each).
kq_status launch_quant_mma(const void* x, int64_t M, int64_t d, int64_t ldx, const void* mats, bool mats_bf16,
                           uint8_t* q, uint8_t* scales, int sf_tiled, cudaStream_t stream) {
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
  const int nb = int(d / 32);
  CUtensorMap tmap;
  const cuuint64_t gdim[3] = {32, cuuint64_t(M), cuuint64_t(nb)};
  const cuuint64_t gstride[2] = {cuuint64_t(ldx) * 2, 64};
  const cuuint32_t box[3] = {32, cuuint32_t(kq::kMmaRows), cuuint32_t(kq::kMmaWb)};
  const cuuint32_t estride[3] = {1, 1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cuda_fail("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
  const int smem = 1024 + kq::kMmaStages * kq::kMmaAStageBytes + kq::kMmaWb * 3 * kq::kMmaBBytes + 256;
  if (smem > dev->smem_optin) return KQ_ERR_UNSUPPORTED;
  const int which = (mats_bf16 ? 1 : 0) + (sf_tiled ? 2 : 0);
  static void (*const kernels[4])(const CUtensorMap, const kq::MmaParams) = {
      kq::quant_mma_kernel<kq::KSRC_F32, 0>, kq::quant_mma_kernel<kq::KSRC_BF16, 0>,
      kq::quant_mma_kernel<kq::KSRC_F32, 1>, kq::quant_mma_kernel<kq::KSRC_BF16, 1>};
  auto kern = kernels[which];
  static std::atomic<int> attr_set[4][kMaxDevices];
  int devid = 0;
  cudaGetDevice(&devid);
  if (!attr_set[which][devid].load()) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
    attr_set[which][devid].store(1);
  }
  kq::MmaParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.M = M;
  p.nb = nb;
  const int64_t nrt = (M + kq::kMmaRows - 1) / kq::kMmaRows;
  if (nrt > int64_t(INT32_MAX) / 2 || nb > 2147483647) return KQ_ERR_SHAPE;
  p.n_row_tiles = int(nrt);
  p.nsplit = mats_bf16 ? 1 : 3;
  p.mats = mats;
  p.q = q;
  p.scales = scales;
  // Resident CTAs per SM.  The runtime's occupancy query reports one CTA per SM
  // for any kernel that touches tensor memory (it cannot know how many columns
  // the kernel allocates), so the count comes from the kernel's own budget:
  // kMmaCtasPerSm x 128 tensor-memory columns <= 512, registers capped by the
  // launch bound, and the shared memory checked here.
  const int per_sm = (smem + 1024) * kq::kMmaCtasPerSm <= dev->smem_per_sm ? kq::kMmaCtasPerSm : 1;
  const int64_t ngroups = (nb + kq::kMmaWb - 1) / kq::kMmaWb;
  const int64_t gy = row_stride(ngroups, nrt, dev->sms, per_sm);
  return launch_pdl(kern, dim3(unsigned(ngroups), unsigned(gy)), kq::kMmaThreads, smem, stream,
                    "quant_mma_kernel launch", tmap, p);
}

// Which GEMM kernel serves a shape: the two-SM persistent kernel needs K % 128 == 0
// and pays off once its 256 x 256 tiles give every SM pair work; smaller products
// take the one-SM kernel's 128 x 128 tiles.  KQ_GEMM=1sm|2sm (read once) overrides
// the choice where both apply.
int gemm_env() {
  static const int v = []() {
    const char* e = std::getenv("KQ_GEMM");
    if (e == nullptr) return 0;
    if (std::strcmp(e, "1sm") == 0) return 1;
    if (std::strcmp(e, "2sm") == 0) return 2;
    if (std::strcmp(e, "2sm128") == 0) return 3;
    return 0;
  }();
  return v;
}

bool gemm_uses_pair(int64_t M, int64_t N, int64_t K, int sms) {
  if (K % 128 != 0) return false;
  const int e = gemm_env();
  if (e != 0) return e >= 2;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  return tiles >= sms / 2;
}

// Codes as a byte matrix [rows][K/2]: boxes of 128 rows x row_bytes (64 or 128) with
// the swizzle of the same width.
kq_status encode_codes_map(EncodeTiledFn enc, CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K,
                           int row_bytes) {
  const cuuint64_t gdim[2] = {cuuint64_t(K / 2), cuuint64_t(rows)};
  const cuuint64_t gstride[1] = {cuuint64_t(K / 2)};
  const cuuint32_t box[2] = {cuuint32_t(row_bytes), cuuint32_t(kq::kGmTile)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cuda_fail("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
  return KQ_OK;
}

// Tiled scales as a byte matrix of 256-byte half tiles: a box of 2 * n_tiles rows is
// n_tiles consecutive 512-byte 128 x 4 tiles; tiles past the buffer read as zeros.
kq_status encode_scales_map(EncodeTiledFn enc, CUtensorMap* map, const uint8_t* scales, int64_t rows, int64_t K,
                            int n_tiles) {
  const int64_t tiles = ((rows + 127) / 128) * (K / 128);
  const cuuint64_t gdim[2] = {256, cuuint64_t(2 * tiles)};
  const cuuint64_t gstride[1] = {256};
  const cuuint32_t box[2] = {256, cuuint32_t(2 * n_tiles)};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(scales), gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cuda_fail("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
  return KQ_OK;
}

// C as a [M][ldc] matrix of bf16 or fp32 for TMA tensor stores of 32 x 32 boxes with
// the swizzle of the box's row width (64 or 128 bytes).  False when C's base or row
// stride is not 16-byte aligned or the encoder refuses; the kernels then store
// directly.
bool encode_c_map(EncodeTiledFn enc, CUtensorMap* map, void* c, int64_t M, int64_t N, int64_t ldc, bool bf16) {
  const int64_t esz = bf16 ? 2 : 4;
  if (!aligned(c, 16) || (ldc * esz) % 16 != 0) return false;
  const cuuint64_t gdim[2] = {cuuint64_t(N), cuuint64_t(M)};
  const cuuint64_t gstride[1] = {cuuint64_t(ldc * esz)};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estride[2] = {1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, c, gdim, gstride, box,
             estride, CU_TENSOR_MAP_INTERLEAVE_NONE, bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Two-SM persistent W4A4 GEMM: one cluster of two CTAs per SM pair, 256 x 256 tiles,
// KS K-elements per stage.
template <int KS>
kq_status launch_gemm_pair(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                           const uint8_t* b_scales, int64_t N, int64_t K, void* c, int64_t ldc, bool c_bf16,
                           cudaStream_t stream) {
  using C = kq::G2Cfg<KS>;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
  if (C::kSmemBytes > dev->smem_optin) return KQ_ERR_UNSUPPORTED;
  CUtensorMap ma, mb, msa, msb;
  kq_status st;
  if ((st = encode_codes_map(enc, &ma, a_q, M, K, C::kRowBytes)) != KQ_OK ||
      (st = encode_codes_map(enc, &mb, b_q, N, K, C::kRowBytes)) != KQ_OK ||
      (st = encode_scales_map(enc, &msa, a_scales, M, K, C::kTiles)) != KQ_OK ||
      (st = encode_scales_map(enc, &msb, b_scales, N, K, C::kTiles)) != KQ_OK)
    return st;
  static std::atomic<int> attr_set[kMaxDevices];
  int devid = 0;
  cudaGetDevice(&devid);
  if (!attr_set[devid].load()) {
    const cudaError_t e = cudaFuncSetAttribute(kq::mxf4_gemm2_kernel<KS>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
    attr_set[devid].store(1);
  }
  CUtensorMap mc;
  std::memset(&mc, 0, sizeof(mc));
  kq::Gemm2Params p;
  p.c = c;
  p.M = M;
  p.N = N;
  p.ldc = ldc;
  p.c_bf16 = c_bf16 ? 1 : 0;
  p.c_tma = encode_c_map(enc, &mc, c, M, N, ldc, c_bf16) ? 1 : 0;
  p.n_ktiles = int(K / KS);
  p.n_ctiles = int(K / 128);
  p.tiles_m = int((M + 255) / 256);
  p.tiles_n = int((N + 255) / 256);
  const int64_t tiles = int64_t(p.tiles_m) * p.tiles_n;
  const int64_t clusters = std::min<int64_t>(tiles, dev->sms / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(2 * clusters));
  cfg.blockDim = dim3(unsigned(kq::kG2Threads));
  cfg.dynamicSmemBytes = size_t(C::kSmemBytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kq::mxf4_gemm2_kernel<KS>, ma, mb, msa, msb, mc, p);
  if (e != cudaSuccess) return cuda_fail("mxf4_gemm2_kernel launch", e);
  return KQ_OK;
}

// W4A4 GEMM: one 128 x 128 tile of C per CTA, N tiles across x, M tiles across y.
kq_status launch_gemm(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                      const uint8_t* b_scales, int64_t N, int64_t K, void* c, int64_t ldc, bool c_bf16,
                      cudaStream_t stream) {
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
  if (kq::kGmSmemBytes > dev->smem_optin) return KQ_ERR_UNSUPPORTED;
  // codes as a 2-D byte tensor [rows][K/2], 128-row x 64-byte boxes, 64-byte swizzle
  CUtensorMap maps[2];
  const uint8_t* codes[2] = {a_q, b_q};
  const int64_t rows[2] = {M, N};
  for (int i = 0; i < 2; i++) {
    const cuuint64_t gdim[2] = {cuuint64_t(K / 2), cuuint64_t(rows[i])};
    const cuuint64_t gstride[1] = {cuuint64_t(K / 2)};
    const cuuint32_t box[2] = {64, cuuint32_t(kq::kGmTile)};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes[i]), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cuda_fail("cuTensorMapEncodeTiled", cudaErrorInvalidValue);
  }
  static std::atomic<int> attr_set[kMaxDevices];
  int devid = 0;
  cudaGetDevice(&devid);
  if (!attr_set[devid].load()) {
    const cudaError_t e =
        cudaFuncSetAttribute(kq::mxf4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kq::kGmSmemBytes);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", e);
    attr_set[devid].store(1);
  }
  CUtensorMap mc;
  std::memset(&mc, 0, sizeof(mc));
  kq::GemmParams p;
  p.sa = a_scales;
  p.sb = b_scales;
  p.c = c;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ldc = ldc;
  p.c_bf16 = c_bf16 ? 1 : 0;
  p.c_tma = encode_c_map(enc, &mc, c, M, N, ldc, c_bf16) ? 1 : 0;
  p.n_ktiles = int((K + kq::kGmKStage - 1) / kq::kGmKStage);
  p.k_tail_blocks = int((K / 32 - 1) % 4) + 1;
  const int64_t gx = (N + kq::kGmTile - 1) / kq::kGmTile, gy = (M + kq::kGmTile - 1) / kq::kGmTile;
  return launch_pdl(kq::mxf4_gemm_kernel, dim3(unsigned(gx), unsigned(gy)), kq::kGmThreads, kq::kGmSmemBytes, stream,
                    "mxf4_gemm_kernel launch", maps[0], maps[1], mc, p);
}

kq_status check_x(const void* x, int64_t M, int64_t d, int64_t ldx) {
  if (M < 0 || d < 0) return KQ_ERR_INVALID_ARG;
  if (d % 32 != 0 || ldx < d) return KQ_ERR_SHAPE;
  if (d / 32 > int64_t(INT32_MAX) / 2 || M > (int64_t(1) << 40)) return KQ_ERR_SHAPE;
  if (x == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || ldx % 8 != 0) return KQ_ERR_ALIGN;
  return KQ_OK;
}

kq_status check_out(const uint8_t* q, const uint8_t* scales) {
  if (q == nullptr || scales == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(q, 16)) return KQ_ERR_ALIGN;
  return KQ_OK;
}

int grid_for(int64_t work, int threads) {
  const DeviceInfo* dev = device_info();
  const int64_t cap = dev ? int64_t(dev->sms) * 8 : 1184;
  int64_t g = (work + threads - 1) / threads;
  if (g > cap) g = cap;
  return g < 1 ? 1 : int(g);
}

// ---- variant selection for KQ_VAR_AUTO
//
// The faster variant for fp32 matrices with the factored form given, as measured
// at the shapes of the quantizer sweep (rows M x channels d, 32-element blocks;
// the sweep table of every kernel kind at every shape is the source).  A shape
// takes the entry of the nearest swept shape, distance measured in log2 M and
// log2 d.  bf16 matrices, and fp32 matrices without the factored form, have only
// the tensor-core variant.
struct AutoRule {
  int64_t M, d;
  kq_variant v;
};
constexpr AutoRule kAutoTable[] = {
    {1, 1152, KQ_VAR_MMA},            {1, 3072, KQ_VAR_MMA},            {1, 12288, KQ_VAR_BUTTERFLY},
    {16, 1152, KQ_VAR_BUTTERFLY},     {16, 3072, KQ_VAR_BUTTERFLY},     {16, 12288, KQ_VAR_BUTTERFLY},
    {256, 1152, KQ_VAR_BUTTERFLY},    {256, 3072, KQ_VAR_BUTTERFLY},    {256, 12288, KQ_VAR_BUTTERFLY},
    {4096, 1152, KQ_VAR_BUTTERFLY},   {4096, 3072, KQ_VAR_BUTTERFLY},   {4096, 12288, KQ_VAR_BUTTERFLY},
    {16384, 1152, KQ_VAR_BUTTERFLY},  {16384, 3072, KQ_VAR_BUTTERFLY},  {16384, 12288, KQ_VAR_BUTTERFLY},
    {65536, 1152, KQ_VAR_BUTTERFLY},  {65536, 3072, KQ_VAR_BUTTERFLY},  {65536, 12288, KQ_VAR_BUTTERFLY},
};

kq_variant table_variant(int64_t M, int64_t d) {
  const double lm = std::log2(double(M > 0 ? M : 1)), ld = std::log2(double(d > 0 ? d : 1));
  double best = 1e300;
  kq_variant v = KQ_VAR_BUTTERFLY;
  for (const AutoRule& r : kAutoTable) {
    const double dm = std::log2(double(r.M)) - lm, dd = std::log2(double(r.d)) - ld;
    const double dist = dm * dm + dd * dd;
    if (dist < best) {
      best = dist;
      v = r.v;
    }
  }
  return v;
}

// KQ_VARIANT=mma|butterfly in the environment replaces the table's choice for
// KQ_VAR_AUTO where that variant can serve the call (read once per process).
kq_variant env_variant() {
  static const kq_variant v = []() {
    const char* e = std::getenv("KQ_VARIANT");
    if (e == nullptr) return KQ_VAR_AUTO;
    if (std::strcmp(e, "mma") == 0) return KQ_VAR_MMA;
    if (std::strcmp(e, "butterfly") == 0) return KQ_VAR_BUTTERFLY;
    return KQ_VAR_AUTO;
  }();
  return v;
}

// The variant kq_quantize runs: an explicit request as given; KQ_VAR_AUTO through
// the override, then the table, within what the matrices allow.
kq_variant resolve_variant(int64_t M, int64_t d, kq_dtype mat_dtype, bool has_factored, kq_variant requested) {
  if (requested != KQ_VAR_AUTO) return requested;
  if (mat_dtype == KQ_BF16 || !has_factored) return KQ_VAR_MMA;
  const kq_variant e = env_variant();
  if (e != KQ_VAR_AUTO) return e;
  return table_variant(M, d);
}

}  // namespace

extern "C" {

int kq_abi_version(void) { return 204; }

const char* kq_status_string(kq_status s) {
  switch (s) {
    case KQ_OK: return "KQ_OK";
    case KQ_ERR_INVALID_ARG: return "KQ_ERR_INVALID_ARG: null pointer, bad enum or negative size";
    case KQ_ERR_SHAPE: return "KQ_ERR_SHAPE: d must be a multiple of 32 and ldx >= d";
    case KQ_ERR_ALIGN: return "KQ_ERR_ALIGN: pointer or row stride not aligned as required";
    case KQ_ERR_SINGULAR: return "KQ_ERR_SINGULAR: an LU factor has u == 0";
    case KQ_ERR_UNSUPPORTED: return "KQ_ERR_UNSUPPORTED: variant/dtype combination not provided";
    case KQ_ERR_CUDA: return "KQ_ERR_CUDA: a CUDA call failed";
    case KQ_ERR_DEVICE_TIMEOUT: return "KQ_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
  }
  return "unknown kq_status";
}

kq_status kq_expand_blocks_n(const float* params, int64_t nt, int log2n, int inverse, kq_dtype out_dtype,
                             void* mats, kq_stream_t stream) {
  if (nt < 0 || (out_dtype != KQ_F32 && out_dtype != KQ_BF16)) return KQ_ERR_INVALID_ARG;
  if (inverse < 0 || inverse > 2 || log2n < 1 || log2n > kq::kMaxFactors) return KQ_ERR_INVALID_ARG;
  if (nt == 0) return KQ_OK;
  if (params == nullptr || mats == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(params, 4) || !aligned(mats, 4)) return KQ_ERR_ALIGN;
  if (nt > (int64_t(INT32_MAX) * 256) >> (2 * log2n)) return KQ_ERR_SHAPE;  // grid of 256-thread blocks
  const int64_t n = nt << (2 * log2n);
  kq::expand_kernel<<<unsigned((n + 255) / 256), 256, 0, as_cuda(stream)>>>(params, nt, log2n, inverse,
                                                                           out_dtype == KQ_BF16 ? 1 : 0, mats);
  return launch_status("expand_kernel launch");
}

kq_status kq_expand_blocks(const float* params, int64_t nb, int inverse, kq_dtype out_dtype, void* mats,
                           kq_stream_t stream) {
  return kq_expand_blocks_n(params, nb, 5, inverse, out_dtype, mats, stream);
}

kq_status kq_expand_factored_n(const float* params, int64_t nt, int log2n, float* factored, kq_stream_t stream) {
  if (nt < 0 || log2n < 4 || log2n > 7) return KQ_ERR_INVALID_ARG;
  if (log2n == 4 && nt % 2 != 0) return KQ_ERR_SHAPE;  // two 16-element blocks per record
  if (nt == 0) return KQ_OK;
  if (params == nullptr || factored == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(params, 4) || !aligned(factored, 16)) return KQ_ERR_ALIGN;
  if (nt > (int64_t(1) << 29)) return KQ_ERR_SHAPE;
  const int64_t nb32 = log2n == 4 ? nt / 2 : nt << (log2n - 5);
  kq::expand_factored_kernel<<<unsigned((nb32 + 127) / 128), 128, 0, as_cuda(stream)>>>(params, nb32, log2n,
                                                                                        factored);
  return launch_status("expand_factored_kernel launch");
}

kq_status kq_expand_factored(const float* params, int64_t nb, float* factored, kq_stream_t stream) {
  return kq_expand_factored_n(params, nb, 5, factored, stream);
}

kq_status kq_quantize_n(const void* x, int64_t M, int64_t d, int64_t ldx, int log2n, const void* mats,
                        kq_dtype mat_dtype, const float* factored, uint8_t* q, uint8_t* scales, kq_variant variant,
                        kq_scale_layout scale_layout, kq_stream_t stream) {
  if (variant != KQ_VAR_AUTO && variant != KQ_VAR_MMA && variant != KQ_VAR_BUTTERFLY) return KQ_ERR_INVALID_ARG;
  if (scale_layout != KQ_SCALES_ROW_MAJOR && scale_layout != KQ_SCALES_MMA_TILED) return KQ_ERR_INVALID_ARG;
  if (log2n < 4 || log2n > 7) return KQ_ERR_INVALID_ARG;
  const int sf_tiled = scale_layout == KQ_SCALES_MMA_TILED ? 1 : 0;
  if (mat_dtype != KQ_F32 && mat_dtype != KQ_BF16) return KQ_ERR_INVALID_ARG;
  kq_status st = check_x(x, M, d, ldx);
  if (st != KQ_OK) return st;
  if (log2n > 5 && d % (int64_t(1) << log2n) != 0) return KQ_ERR_SHAPE;
  if (M == 0 || d == 0) return KQ_OK;
  st = check_out(q, scales);
  if (st != KQ_OK) return st;
  if (mats == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(mats, 16)) return KQ_ERR_ALIGN;
  const float* m32 = static_cast<const float*>(mats);
  if (log2n != 5) {
    // 16-, 64- and 128-element blocks: the butterfly only (fp32 matrices and the factored form)
    if (variant == KQ_VAR_MMA || mat_dtype == KQ_BF16) return KQ_ERR_UNSUPPORTED;
    if (factored == nullptr) return KQ_ERR_INVALID_ARG;
    if (!aligned(factored, 16)) return KQ_ERR_ALIGN;
    const cudaStream_t cs = as_cuda(stream);
    switch (log2n * 2 + sf_tiled) {
      case 8: return launch_quant<kq::MODE_KRON, 0, 16>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
      case 9: return launch_quant<kq::MODE_KRON, 1, 16>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
      case 12: return launch_quant<kq::MODE_KRON, 0, 64>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
      case 13: return launch_quant<kq::MODE_KRON, 1, 64>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
      case 14: return launch_quant<kq::MODE_KRON, 0, 128>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
      default: return launch_quant<kq::MODE_KRON, 1, 128>(x, M, d, ldx, m32, factored, nullptr, q, scales, cs);
    }
  }
  // bf16 matrices are only served by the tensor-core variant; AUTO resolves per shape
  if (variant == KQ_VAR_BUTTERFLY && mat_dtype == KQ_BF16) return KQ_ERR_UNSUPPORTED;
  const bool use_mma = resolve_variant(M, d, mat_dtype, factored != nullptr, variant) == KQ_VAR_MMA;
  if (use_mma)
    return launch_quant_mma(x, M, d, ldx, mats, mat_dtype == KQ_BF16, q, scales, sf_tiled, as_cuda(stream));
  if (factored == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(factored, 16)) return KQ_ERR_ALIGN;
  return sf_tiled ? launch_quant<kq::MODE_KRON, 1, 32>(x, M, d, ldx, m32, factored, nullptr, q, scales, as_cuda(stream))
                  : launch_quant<kq::MODE_KRON, 0, 32>(x, M, d, ldx, m32, factored, nullptr, q, scales, as_cuda(stream));
}

kq_status kq_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const void* mats, kq_dtype mat_dtype,
                      const float* factored, uint8_t* q, uint8_t* scales, kq_variant variant,
                      kq_scale_layout scale_layout, kq_stream_t stream) {
  return kq_quantize_n(x, M, d, ldx, 5, mats, mat_dtype, factored, q, scales, variant, scale_layout, stream);
}

kq_status kq_ref_smooth_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const float* inv_s,
                                 uint8_t* q, uint8_t* scales, kq_stream_t stream) {
  kq_status st = check_x(x, M, d, ldx);
  if (st != KQ_OK) return st;
  if (M == 0 || d == 0) return KQ_OK;
  st = check_out(q, scales);
  if (st != KQ_OK) return st;
  if (inv_s == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(inv_s, 16)) return KQ_ERR_ALIGN;
  return launch_quant<kq::MODE_SMOOTH, 0>(x, M, d, ldx, nullptr, nullptr, inv_s, q, scales, as_cuda(stream));
}

kq_status kq_ref_fwht_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, uint8_t* q, uint8_t* scales,
                               kq_stream_t stream) {
  kq_status st = check_x(x, M, d, ldx);
  if (st != KQ_OK) return st;
  if (M == 0 || d == 0) return KQ_OK;
  st = check_out(q, scales);
  if (st != KQ_OK) return st;
  return launch_quant<kq::MODE_FWHT, 0>(x, M, d, ldx, nullptr, nullptr, nullptr, q, scales, as_cuda(stream));
}

kq_status kq_dequantize(const uint8_t* q, const uint8_t* scales, int64_t M, int64_t d, const void* inv_mats,
                        kq_dtype mat_dtype, void* out, kq_dtype out_dtype, kq_stream_t stream) {
  if (M < 0 || d < 0) return KQ_ERR_INVALID_ARG;
  if ((mat_dtype != KQ_F32 && mat_dtype != KQ_BF16) || (out_dtype != KQ_F32 && out_dtype != KQ_BF16))
    return KQ_ERR_INVALID_ARG;
  if (d % 32 != 0) return KQ_ERR_SHAPE;
  if (M == 0 || d == 0) return KQ_OK;
  if (q == nullptr || scales == nullptr || out == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || (inv_mats != nullptr && !aligned(inv_mats, 4))) return KQ_ERR_ALIGN;
  const int64_t nb = d / 32;
  if (nb > int64_t(INT32_MAX)) return KQ_ERR_SHAPE;
  // block columns across x; groups of 8 warps x 8 rows across y, about four waves
  // of resident CTAs
  const DeviceInfo* dev = device_info();
  const int64_t want = (dev ? int64_t(dev->sms) : 148) * 8 * 4;
  int64_t gy = (want + nb - 1) / nb;
  const int64_t row_groups = (M + kq::kDqWarps * kq::kDqRows - 1) / (kq::kDqWarps * kq::kDqRows);
  if (gy > row_groups) gy = row_groups;
  if (gy > 65535) gy = 65535;
  auto kern = inv_mats != nullptr ? kq::dequant_kernel<1> : kq::dequant_kernel<0>;
  kern<<<dim3(unsigned(nb), unsigned(gy)), kq::kDqWarps * 32, 0, as_cuda(stream)>>>(
      q, scales, M, int(nb), inv_mats, mat_dtype == KQ_BF16 ? 1 : 0, out, out_dtype == KQ_BF16 ? 1 : 0);
  return launch_status("dequant_kernel launch");
}

kq_status kq_gemm_mxf4(const uint8_t* a_q, const uint8_t* a_scales, int64_t M, const uint8_t* b_q,
                       const uint8_t* b_scales, int64_t N, int64_t K, void* c, int64_t ldc, kq_dtype c_dtype,
                       kq_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return KQ_ERR_INVALID_ARG;
  if (c_dtype != KQ_F32 && c_dtype != KQ_BF16) return KQ_ERR_INVALID_ARG;
  if (K % 32 != 0 || ldc < N) return KQ_ERR_SHAPE;
  if (M == 0 || N == 0) return KQ_OK;
  if (K == 0) return KQ_ERR_SHAPE;
  if (a_q == nullptr || a_scales == nullptr || b_q == nullptr || b_scales == nullptr || c == nullptr)
    return KQ_ERR_INVALID_ARG;
  if (!aligned(a_q, 16) || !aligned(b_q, 16) || !aligned(a_scales, 16) || !aligned(b_scales, 16) ||
      !aligned(c, c_dtype == KQ_BF16 ? 2 : 4))
    return KQ_ERR_ALIGN;
  if (K / 2 > int64_t(INT32_MAX) - 128 || M > int64_t(65535) * kq::kGmTile || N > int64_t(INT32_MAX) - kq::kGmTile)
    return KQ_ERR_SHAPE;
  const DeviceInfo* dev = device_info();
  if (dev != nullptr && gemm_uses_pair(M, N, K, dev->sms)) {
    if (K % 256 == 0 && gemm_env() != 3)
      return launch_gemm_pair<256>(a_q, a_scales, M, b_q, b_scales, N, K, c, ldc, c_dtype == KQ_BF16,
                                   as_cuda(stream));
    return launch_gemm_pair<128>(a_q, a_scales, M, b_q, b_scales, N, K, c, ldc, c_dtype == KQ_BF16,
                                 as_cuda(stream));
  }
  return launch_gemm(a_q, a_scales, M, b_q, b_scales, N, K, c, ldc, c_dtype == KQ_BF16, as_cuda(stream));
}

kq_status kq_adaln_quantize(const void* x, int64_t M, int64_t d, int64_t ldx, const void* shift, const void* scale,
                            int64_t rows_per_group, float eps, const float* mats, const float* factored, uint8_t* q,
                            uint8_t* scales, kq_scale_layout scale_layout, float* stats, kq_stream_t stream) {
  if (scale_layout != KQ_SCALES_ROW_MAJOR && scale_layout != KQ_SCALES_MMA_TILED) return KQ_ERR_INVALID_ARG;
  if (rows_per_group < 1) return KQ_ERR_INVALID_ARG;
  kq_status st = check_x(x, M, d, ldx);
  if (st != KQ_OK) return st;
  if (M == 0 || d == 0) return KQ_OK;
  const int64_t nb = d / 32;
  if (nb > kq::kAlMaxThreads) return KQ_ERR_UNSUPPORTED;
  st = check_out(q, scales);
  if (st != KQ_OK) return st;
  if (shift == nullptr || scale == nullptr || mats == nullptr || factored == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(shift, 16) || !aligned(scale, 16) || !aligned(mats, 16) || !aligned(factored, 16) ||
      (stats != nullptr && !aligned(stats, 8)))
    return KQ_ERR_ALIGN;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  kq::AdaLnParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.M = M;
  p.nb = int(nb);
  p.nbw = (p.nb + 31) / 32 * 32;
  p.tree_pad = 1;
  while (p.tree_pad < p.nb) p.tree_pad *= 2;
  p.rows = kq::kAlMaxThreads / p.nbw;
  p.shift = static_cast<const uint16_t*>(shift);
  p.scale = static_cast<const uint16_t*>(scale);
  p.rows_per_group = rows_per_group;
  p.eps = eps;
  p.mats = mats;
  p.factored = factored;
  p.q = q;
  p.scales = scales;
  p.stats = stats;
  const int threads = p.rows * p.nbw;
  const int nws = p.tree_pad > 32 ? p.tree_pad / 32 : 1;
  int devid = 0;
  cudaGetDevice(&devid);
  if (stats != nullptr) {
    // two kernels: the statistics into stats, then the butterfly quantizer's ADALN form
    // reading them (h is formed inside it and never reaches memory)
    const int ssmem = 2 * p.rows * nws * 4;
    int per_sm = 0;
    const cudaError_t eo = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kq::adaln_stats_kernel, threads, ssmem);
    if (eo != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveBlocksPerMultiprocessor", eo);
    if (per_sm < 1) return cuda_fail("occupancy: no resident CTA", cudaErrorInvalidConfiguration);
    // one wave: every statistics CTA is resident before the quantizer's CTAs may launch
    const int64_t sgrid = std::min<int64_t>((M + p.rows - 1) / p.rows, int64_t(dev->sms) * per_sm);
    const kq_status sst = launch_pdl(kq::adaln_stats_kernel, dim3(unsigned(sgrid)), threads, ssmem,
                                     as_cuda(stream), "adaln_stats_kernel launch", p);
    if (sst != KQ_OK) return sst;
    AdaLnInput ada;
    ada.stats = stats;
    ada.shift = p.shift;
    ada.scale = p.scale;
    ada.rows_per_group = rows_per_group;
    return scale_layout == KQ_SCALES_MMA_TILED
               ? launch_quant<kq::MODE_KRON, 1, 32, true>(x, M, d, ldx, mats, factored, nullptr, q, scales,
                                                          as_cuda(stream), ada)
               : launch_quant<kq::MODE_KRON, 0, 32, true>(x, M, d, ldx, mats, factored, nullptr, q, scales,
                                                          as_cuda(stream), ada);
  }
  const int smem = (kq::kAlStages + 1) * threads * 64 + 2 * p.rows * nws * 4;
  const int which = scale_layout == KQ_SCALES_MMA_TILED ? 1 : 0;
  auto kern = which ? kq::adaln_quant_kernel<1> : kq::adaln_quant_kernel<0>;
  // the largest configuration: 512 threads, and at most 32 warp sums per buffer
  constexpr int kMaxSmem = (kq::kAlStages + 1) * kq::kAlMaxThreads * 64 + 2 * 32 * 4;
  if (smem > kMaxSmem || kMaxSmem > dev->smem_optin) return KQ_ERR_UNSUPPORTED;
  static std::atomic<int> attr_set[2][kMaxDevices];
  if (!attr_set[which][devid].load()) {
    const cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (ea != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(MaxDynamicSharedMemorySize)", ea);
    attr_set[which][devid].store(1);
  }
  int per_sm = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
  if (per_sm < 1) return cuda_fail("occupancy: no resident CTA", cudaErrorInvalidConfiguration);
  const int64_t groups = (M + p.rows - 1) / p.rows;
  const int64_t grid = std::min<int64_t>(groups, int64_t(dev->sms) * per_sm);
  return launch_pdl(kern, dim3(unsigned(grid)), threads, smem, as_cuda(stream), "adaln_quant_kernel launch", p);
}

kq_status kq_select_gemm_kernel(int64_t M, int64_t N, int64_t K, int* two_sm) {
  if (two_sm == nullptr || M < 0 || N < 0 || K < 0) return KQ_ERR_INVALID_ARG;
  if (K % 32 != 0) return KQ_ERR_SHAPE;
  const DeviceInfo* dev = device_info();
  if (dev == nullptr) return cuda_fail("device query", cudaErrorInvalidDevice);
  *two_sm = gemm_uses_pair(M, N, K, dev->sms) ? 1 : 0;
  return KQ_OK;
}

kq_status kq_e2m1_pack(const float* v, int64_t n, uint8_t* out, kq_stream_t stream) {
  if (n < 0) return KQ_ERR_INVALID_ARG;
  if (n % 2 != 0) return KQ_ERR_SHAPE;
  if (n == 0) return KQ_OK;
  if (v == nullptr || out == nullptr) return KQ_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(out, 4)) return KQ_ERR_ALIGN;
  kq::e2m1_pack_kernel<<<grid_for(n / 8 + 1, 256), 256, 0, as_cuda(stream)>>>(v, n, out);
  return launch_status("e2m1_pack_kernel launch");
}

kq_status kq_select_variant(int64_t M, int64_t d, int log2n, kq_dtype mat_dtype, int has_factored,
                            kq_variant* chosen) {
  if (chosen == nullptr || M < 0 || d < 0 || (mat_dtype != KQ_F32 && mat_dtype != KQ_BF16)) return KQ_ERR_INVALID_ARG;
  if (log2n < 4 || log2n > 7) return KQ_ERR_INVALID_ARG;
  if (log2n != 5) {  // 16-, 64- and 128-element blocks: the butterfly only
    if (mat_dtype == KQ_BF16 || !has_factored) return KQ_ERR_UNSUPPORTED;
    *chosen = KQ_VAR_BUTTERFLY;
    return KQ_OK;
  }
  *chosen = resolve_variant(M, d, mat_dtype, has_factored != 0, KQ_VAR_AUTO);
  return KQ_OK;
}

const char* kq_last_error(void) { return g_last_error; }

kq_status kq_get_device_error(int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail("cudaDeviceSynchronize", e);
  unsigned int flags = 0;
  e = cudaMemcpyFromSymbol(&flags, kq::g_dev_error, sizeof(flags));
  if (e != cudaSuccess) return cuda_fail("cudaMemcpyFromSymbol", e);
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(kq::g_dev_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyToSymbol", e);
  }
  if (flags & kq::kDevErrTimeout) return KQ_ERR_DEVICE_TIMEOUT;
  if (flags & kq::kDevErrSingular) return KQ_ERR_SINGULAR;
  return KQ_OK;
}

}  // extern "C"
