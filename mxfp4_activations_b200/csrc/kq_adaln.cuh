// kq_adaln.cuh -- the KroQuant quantizer fused with the AdaLN-modulated LayerNorm that
// produces its input in a DiT block ("KroQuant: Kronecker-Structured Block Transforms
// ...", Problem: AdaLN blocks keep the transform from being absorbed offline; the
// KroQuant abstract: normalisation layers between blocks force it to run online).
//
// Per row of x (bf16, d = 32 nb), in fp32 as DiT models compute their LayerNorm:
//   S1 = pairwise sum of the d inputs (padded with +0 to a power of two, neighbours
//        added level by level), mu = S1 / d
//   S2 = pairwise sum of (x_i - mu)^2, var = S2 / d, rstd = 1 / sqrt(var + eps)
//   h_i = bf16( ((x_i - mu) * rstd) * (1 + scale[g][i]) + shift[g][i] ),  g = row / rows_per_group
// every step one IEEE binary32 operation rounded to nearest even (no contraction; sqrt and
// division correctly rounded), so the statistics and h are the definition's bit for bit;
// then y = h K_b and the certified MXFP4 step of the butterfly quantizer (kq_quant.cuh)
// on h, which never leaves the chip.  Steps run on packed fp32 pairs where no multiply
// feeds a packed add; every add that follows a multiply is the scalar round-to-nearest
// intrinsic, which the compiler never contracts (a packed multiply followed by a packed add
// was measured to be fused into one FMA).
//
// Work mapping.  A CTA takes R rows per step, each on a slot of nbw = nb rounded up to a
// multiple of 32 threads: thread t takes block column c = t % nbw of slot t / nbw (columns
// >= nb are padding and contribute +0), so a thread keeps one block column for its life,
// with the column's butterfly coefficients in registers, and every warp lies in one row.
// Each thread streams its blocks of the coming steps through a private ring of
// kAlStages 64-byte shared-memory slots (cp.async), as the butterfly kernel does.
//
// The pairwise tree of a row is aligned to its blocks: the first five levels sum each
// block in registers, the next five pair the block sums of a warp by shfl_xor (fp64
// addition is commutative, so both partners form the same sum), and the rest pair the
// warp sums, which every warp of the slot reads from shared memory after one barrier.
// h of each block is staged in shared memory for the warp-cooperative exact path.
//
// Two forms.  adaln_quant_kernel does everything in one kernel (kq_adaln_quantize without
// a statistics buffer).  With one, adaln_stats_kernel writes each row's (mu, rstd) with
// the same tree and operations, and the butterfly quantizer's ADALN form (kq_quant.cuh)
// forms h from x, those statistics and the modulation vectors inside its own row loop:
// the quantizer keeps its two CTAs per SM and no CTA-wide barrier, and the statistics
// pass, free of the quantizer's registers, runs at two CTAs of up to 512 threads per SM.
#pragma once

#include "kq_quant.cuh"

namespace kq {

constexpr int kAlMaxThreads = 512;
constexpr int kAlStages = 3;  // ring slots per thread (blocks of two coming steps in flight)

struct AdaLnParams {
  const uint16_t* x;      // bf16 bits [M][ldx]
  int64_t ldx;
  int64_t M;
  int nb;                 // d / 32
  int nbw;                // nb rounded up to a multiple of 32: threads per row slot
  int tree_pad;           // smallest power of two >= nb (the row tree's width in blocks)
  int rows;               // R: row slots per CTA
  const uint16_t* shift;  // bf16 bits [G][nb * 32]
  const uint16_t* scale;  // bf16 bits [G][nb * 32]
  int64_t rows_per_group;
  float eps;
  const float* mats;      // fp32 [nb][32][32] (exact path)
  const float* factored;  // [nb][48]
  uint8_t* q;             // [M][nb * 16]
  uint8_t* scales;        // row-major [M][nb], or tiled (scale_index)
  float* stats;           // [M][2] (mu, rstd) or null
};

// Pairwise fp32 sum of the 32 values of one block (v_0 .. v_31): neighbours added level
// by level.
__device__ __forceinline__ float block_pairwise(const float (&v)[32]) {
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; j++) a[j] = __fadd_rn(v[2 * j], v[2 * j + 1]);
#pragma unroll
  for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
    for (int j = 0; j < n; j++) a[j] = __fadd_rn(a[2 * j], a[2 * j + 1]);
  return a[0];
}

// The rest of a row's pairwise tree above the block sums v (+0 for padding columns):
// pairs within the warp by shfl_xor (levels 6..10 of the row tree, at most log2 of the
// tree's width), then, for rows wider than a warp, pairs of the warp sums that the slot's
// warps leave in ws (padded with +0 to the tree's width / 32).  One barrier; every thread
// of the slot returns the row sum.  ws must not be written again before every thread of
// the CTA has passed the next barrier.
__device__ __forceinline__ float row_sum(float v, int c, int nbw, int tree_pad, float* ws) {
  const int wl = tree_pad >= 32 ? 5 : __ffs(tree_pad) - 1;
#pragma unroll 1
  for (int l = 0; l < wl; l++) v = __fadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, 1 << l));
  if (tree_pad <= 32) {
    __syncthreads();  // keeps the barrier count of every row the same
    return __shfl_sync(0xFFFFFFFFu, v, 0);
  }
  const int nw = tree_pad >> 5, lane = c & 31;
  if (lane == 0) ws[c >> 5] = v;
  if (lane == 0 && c == 0)
    for (int j = nbw >> 5; j < nw; j++) ws[j] = 0.0f;
  __syncthreads();
  float u = lane < nw ? ws[lane] : 0.0f;
#pragma unroll 1
  for (int o = 1; o < nw; o <<= 1) u = __fadd_rn(u, __shfl_xor_sync(0xFFFFFFFFu, u, o));
  return __shfl_sync(0xFFFFFFFFu, u, 0);
}

// The statistics of one row as its slot's threads hold it: thread c has block column c
// as 16 bf16 words w (zero for padding columns and rows past M, act false).  Returns the
// block's inputs as packed pairs in X and the row's mu and rstd in every thread.  Two
// barriers (row_sum); ws1, ws2: the slot's two warp-sum buffers.
__device__ __forceinline__ void row_stats(const uint32_t (&w)[16], bool act, int c, const AdaLnParams& p,
                                          float* ws1, float* ws2, uint64_t (&X)[16], float& mu, float& rstd) {
  const float d = float(p.nb * kBlock);
#pragma unroll
  for (int j = 0; j < 16; j++) X[j] = pk2(bf16lo(w[j]), bf16hi(w[j]));
  float b1 = 0.0f;
  if (act) {
    float xv[32];
#pragma unroll
    for (int j = 0; j < 16; j++) upk2(X[j], xv[2 * j], xv[2 * j + 1]);
    b1 = block_pairwise(xv);
  }
  const float s1 = row_sum(b1, c, p.nbw, p.tree_pad, ws1);
  mu = __fdiv_rn(s1, d);
  const uint64_t MU = pk2(mu, mu);
  float b2 = 0.0f;
  if (act) {
    float sq[32];
#pragma unroll
    for (int j = 0; j < 16; j++) {
      const uint64_t t = sub2_rn(X[j], MU);
      upk2(mul2_rn(t, t), sq[2 * j], sq[2 * j + 1]);
    }
    b2 = block_pairwise(sq);
  }
  const float s2 = row_sum(b2, c, p.nbw, p.tree_pad, ws2);
  const float var = __fdiv_rn(s2, d);
  rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, p.eps)));
}

// The statistics pass of the two-kernel form (kq_adaln_quantize given stats): each
// row's (mu, rstd), formed exactly as adaln_quant_kernel forms them, into p.stats; the
// butterfly quantizer's ADALN form then modulates and quantizes.  Same mapping of rows
// and block columns to threads as adaln_quant_kernel, without the quantizer, so two CTAs
// fit on an SM; each thread loads its next step's block while this step's sums run.
__global__ void __launch_bounds__(kAlMaxThreads, 2) adaln_stats_kernel(const __grid_constant__ AdaLnParams p) {
  extern __shared__ __align__(16) float st_ws[];  // [2][R][nws]
  const int R = p.rows;
  const int nws = p.tree_pad > 32 ? (p.tree_pad >> 5) : 1;
  const int t = threadIdx.x;
  const int rho = t / p.nbw, c = t % p.nbw;
  const bool col = c < p.nb;
  float* ws1 = st_ws + size_t(rho) * nws;
  float* ws2 = st_ws + size_t(R + rho) * nws;
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  const int64_t step_rows = int64_t(gridDim.x) * R;
  const int64_t r_first = int64_t(blockIdx.x) * R + rho;
  const int64_t n_steps = (p.M - int64_t(blockIdx.x) * R + step_rows - 1) / step_rows;  // CTA-uniform
  uint4 nx[4];
#pragma unroll
  for (int k = 0; k < 4; k++) nx[k] = make_uint4(0u, 0u, 0u, 0u);
  if (col && r_first < p.M) {
    const uint4* px = reinterpret_cast<const uint4*>(p.x + r_first * p.ldx + int64_t(c) * kBlock);
#pragma unroll
    for (int k = 0; k < 4; k++) nx[k] = __ldg(px + k);
  }
  grid_launch_dependents();
#pragma unroll 1
  for (int64_t i = 0; i < n_steps; i++) {
    const int64_t r = r_first + i * step_rows;
    const bool act = col && r < p.M;
    uint32_t w[16];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      w[4 * k] = nx[k].x;
      w[4 * k + 1] = nx[k].y;
      w[4 * k + 2] = nx[k].z;
      w[4 * k + 3] = nx[k].w;
    }
    const int64_t rn = r + step_rows;
    if (col && rn < p.M) {
      const uint4* px = reinterpret_cast<const uint4*>(p.x + rn * p.ldx + int64_t(c) * kBlock);
#pragma unroll
      for (int k = 0; k < 4; k++) nx[k] = __ldg(px + k);
    }
    uint64_t X[16];
    float mu, rstd;
    row_stats(w, act, c, p, ws1, ws2, X, mu, rstd);
    if (act && c == 0) *reinterpret_cast<float2*>(p.stats + 2 * r) = make_float2(mu, rstd);
  }
}

template <int TILED>
__global__ void __launch_bounds__(kAlMaxThreads, 1) adaln_quant_kernel(const __grid_constant__ AdaLnParams p) {
  extern __shared__ __align__(128) uint8_t al_smem[];
  const int R = p.rows;
  const int nws = p.tree_pad > 32 ? (p.tree_pad >> 5) : 1;  // warp sums per row tree
  uint8_t* ring = al_smem;                                      // [kAlStages][blockDim][64]
  uint16_t* hx = reinterpret_cast<uint16_t*>(al_smem + size_t(kAlStages) * blockDim.x * 64);  // [blockDim][32]
  float* ws = reinterpret_cast<float*>(al_smem + size_t(kAlStages + 1) * blockDim.x * 64);     // [2][R][nws]
  const int t = threadIdx.x;
  const int rho = t / p.nbw, c = t % p.nbw;
  const bool col = c < p.nb;
  const int cc = col ? c : 0;
  float* ws1 = ws + size_t(rho) * nws;
  float* ws2 = ws + size_t(R + rho) * nws;
  uint16_t* hmine = hx + size_t(t) * kBlock;
  const int sw = (t >> 1) & 3;
  const uint32_t cbase = smem_addr(ring) + uint32_t(t) * 64u;
  const uint32_t kStage = blockDim.x * 64u;

  QuantParams qp = {};
  qp.nb = p.nb;
  qp.factored = p.factored;
  qp.mats = p.mats;
  grid_dependency_wait();  // inputs may come from the previous kernel in the stream

  const int64_t step_rows = int64_t(gridDim.x) * R;
  const int64_t r_first = int64_t(blockIdx.x) * R + rho;
  const int64_t n_steps = (p.M - int64_t(blockIdx.x) * R + step_rows - 1) / step_rows;  // CTA-uniform
  // the first kAlStages - 1 steps' blocks go in flight before anything else
#pragma unroll
  for (int s = 0; s < kAlStages - 1; s++) {
    const int64_t r = r_first + s * step_rows;
    if (col && r < p.M) copy_block_async(cbase + s * kStage, sw, p.x + r * p.ldx + int64_t(c) * kBlock);
    copy_commit();
  }
  grid_launch_dependents();
  ColCoef cf;
  load_coef<MODE_KRON, 32>(qp, cc, cf);

#pragma unroll 1
  for (int64_t i = 0; i < n_steps; i++) {
    const int64_t r = r_first + i * step_rows;
    const bool act = col && r < p.M;
    // refill the slot read one step ago with the block kAlStages - 1 steps ahead
    {
      const int64_t ra = r + (kAlStages - 1) * step_rows;
      const uint32_t slot = uint32_t((i + kAlStages - 1) % kAlStages) * kStage;
      if (col && ra < p.M) copy_block_async(cbase + slot, sw, p.x + ra * p.ldx + int64_t(c) * kBlock);
      copy_commit();
    }
    copy_wait<kAlStages - 1>();  // this step's block has landed
    uint32_t w[16];
    read_slot(cbase + uint32_t(i % kAlStages) * kStage, sw, w);
    if (!act) {
#pragma unroll
      for (int k = 0; k < 16; k++) w[k] = 0u;
    }
    // the modulation vectors of this row's group, in flight while the statistics run
    const int64_t g = act ? r / p.rows_per_group : 0;
    uint4 sv[4], hv[4];
    {
      const uint4* ps = reinterpret_cast<const uint4*>(p.scale + g * (int64_t(p.nb) * kBlock) + int64_t(cc) * kBlock);
      const uint4* ph = reinterpret_cast<const uint4*>(p.shift + g * (int64_t(p.nb) * kBlock) + int64_t(cc) * kBlock);
#pragma unroll
      for (int k = 0; k < 4; k++) {
        sv[k] = act ? __ldg(ps + k) : make_uint4(0u, 0u, 0u, 0u);
        hv[k] = act ? __ldg(ph + k) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // statistics (padding columns and rows past M contribute +0)
    uint64_t X[16];
    float mu, rstd;
    row_stats(w, act, c, p, ws1, ws2, X, mu, rstd);
    if (act && c == 0 && p.stats != nullptr) {
      p.stats[2 * r] = mu;
      p.stats[2 * r + 1] = rstd;
    }
    // modulation, one bf16 rounding per element
    uint32_t hw[16];
    modulate(X, mu, rstd, sv, hv, hw);
    reinterpret_cast<uint4*>(hmine)[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    reinterpret_cast<uint4*>(hmine)[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    reinterpret_cast<uint4*>(hmine)[2] = make_uint4(hw[8], hw[9], hw[10], hw[11]);
    reinterpret_cast<uint4*>(hmine)[3] = make_uint4(hw[12], hw[13], hw[14], hw[15]);
    // transform and certified MXFP4 on h
    const int64_t rr = act ? r : 0;
    uint8_t* qb = p.q + (rr * p.nb + cc) * 16;
    uint8_t* sb = p.scales + scale_index(rr, cc, p.nb, TILED);
    const bool need = quant_block<MODE_KRON, 32>(cf, hw, act, qb, sb);
    if (__any_sync(0xFFFFFFFFu, need)) {
      __syncwarp();  // every lane's staged h is visible to the warp
      warp_exact_pass<KSRC_F32, 32, false>(need, hmine, p.mats + kmat_offset<32>(cc), qb, sb);
    }
  }
  copy_wait<0>();  // no copy still writes the ring
}

}  // namespace kq
