// Whole-layer statistics for VMC [IntLoRA paper notes (ICML2025), method
// section 3: R* = r^alpha R with r = sigma_W / sigma_R]. sigma is the
// population standard deviation over the d x n layer.
//
// One pass reads W (16-byte vector loads) and regenerates R (Philox + Laplace)
// for the same elements; each CTA accumulates shifted sums in fp64 (shift K =
// W[0] for W, 0 for R, whose mean is 0 by symmetry; R's sums are taken of
// R / ln 2 and scaled back when sigma is formed), writes one partial, and
// a finalize kernel adds the partials in a fixed order, so sigma does not
// depend on scheduling. var = (S2 - S1^2 / N) / N.
#include <cuda_runtime.h>

#include <cstdint>

#include "intlora_device.cuh"
#include "intlora_kernels.h"

namespace intlora {

namespace {

constexpr int kStatsThreads = 256;
constexpr double kLn2d = 0.693147180559945309417232121458;

__device__ __forceinline__ void block_sum4(double v[4], double* red /* [4][32] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  warp_sum2(v[0], v[1]);
  warp_sum2(v[2], v[3]);
  if (lane == 0)
    for (int q = 0; q < 4; ++q) red[q * 32 + warp] = v[q];
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    for (int q = 0; q < 4; ++q) v[q] = lane < nw ? red[q * 32 + lane] : 0.0;
    warp_sum2(v[0], v[1]);
    warp_sum2(v[2], v[3]);
  }
}

// Sums of one group of 4 consecutive elements (one Philox block). fp32 partial
// sums of a few groups are flushed into the fp64 accumulators. Each sum is a
// pair of fp32 lanes (f32x2 instructions): words 0 and 2 feed the low half,
// words 1 and 3 the high half.
struct GroupSums {
  uint64_t w1 = 0, w2 = 0, r1 = 0, r2 = 0;
};

template <bool HAS_W, bool SMALL, bool GENERIC>
__device__ __forceinline__ void add_group(GroupSums& g, const StatsJob& J, const float* wgroup,
                                          uint64_t group, float K, int valid, uint32_t k0, uint32_t k1,
                                          const PhiloxSmall& ph, int dist) {
  // SMALL: fewer than 2^34 elements, so the block index's high word is 0
  const uint4 w = SMALL ? philox10_small(static_cast<uint32_t>(group), ph)
                        : aux_block(static_cast<uint64_t>(group), J.stream_id, k0, k1);
  if (GENERIC) {
    // another auxiliary law: R itself is summed
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    float rv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      rv[c] = c < valid ? aux_value_generic(dist, words[c & 2], words[c | 1], (c & 1) != 0) : 0.0f;
    const uint64_t r01 = f2_pack(rv[0], rv[1]), r23 = f2_pack(rv[2], rv[3]);
    g.r1 = f2_add(f2_add(g.r1, r01), r23);
    g.r2 = f2_fma(r23, r23, f2_fma(r01, r01, g.r2));
  } else if (valid == 4) {
    // R / ln 2 = +-log2(w): the sums run in the log2 domain (the sign is a
    // factor of +-1, R^2 needs none) and the finalize kernel scales by ln 2
    const uint64_t l01 = laplace_log2_x2(w.x, w.y), l23 = laplace_log2_x2(w.z, w.w);
    const uint64_t s01 = f2_pack(laplace_sign(w.x, 1.0f), laplace_sign(w.y, 1.0f));
    const uint64_t s23 = f2_pack(laplace_sign(w.z, 1.0f), laplace_sign(w.w, 1.0f));
    g.r1 = f2_fma(l23, s23, f2_fma(l01, s01, g.r1));
    g.r2 = f2_fma(l23, l23, f2_fma(l01, l01, g.r2));
  } else {
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    float rv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) rv[c] = c < valid ? laplace_scaled(words[c], 1.0f) : 0.0f;
    const uint64_t r01 = f2_pack(rv[0], rv[1]), r23 = f2_pack(rv[2], rv[3]);
    g.r1 = f2_add(f2_add(g.r1, r01), r23);
    g.r2 = f2_fma(r23, r23, f2_fma(r01, r01, g.r2));
  }
  if (HAS_W) {
    uint64_t x01, x23;                   // W - K, elements past the tail left at 0
    if (valid == 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(wgroup));
      const uint64_t nk = f2_pack(-K, -K);
      x01 = f2_add(f2_pack(v.x, v.y), nk);
      x23 = f2_add(f2_pack(v.z, v.w), nk);
    } else {
      float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < valid) x[c] = __ldg(wgroup + c) - K;
      x01 = f2_pack(x[0], x[1]);
      x23 = f2_pack(x[2], x[3]);
    }
    g.w1 = f2_add(f2_add(g.w1, x01), x23);
    g.w2 = f2_fma(x23, x23, f2_fma(x01, x01, g.w2));
  }
}

__device__ __forceinline__ double f2_sum(uint64_t v) {
  return static_cast<double>(f2_lo(v)) + static_cast<double>(f2_hi(v));
}

template <bool HAS_W, bool SMALL, bool GENERIC>
__device__ __forceinline__ void stats_body(const StatsJob& J, int64_t local, double acc[4],
                                           uint32_t k0, uint32_t k1, int dist) {
  constexpr int kFlush = 16;  // groups per fp32 partial
  const int64_t full = J.numel >> 2;                 // complete groups
  const int64_t stride = static_cast<int64_t>(J.nblocks) * kStatsThreads;
  const float K = HAS_W ? __ldg(J.W) : 0.0f;
  const int64_t g0 = local * kStatsThreads + threadIdx.x;
  // this thread's groups g0, g0 + stride, ...: a 32-bit trip count, the group
  // index (Philox counter) and the W pointer advance by the stride
  const int32_t count = g0 < full ? static_cast<int32_t>((full - 1 - g0) / stride + 1) : 0;
  uint64_t g = static_cast<uint64_t>(g0);
  const float* wp = HAS_W ? J.W + 4 * g0 : nullptr;
  const PhiloxSmall ph = philox_small_setup(J.stream_id, k0, k1);
  for (int32_t k = 0; k < count;) {
    GroupSums s;
    const int32_t kend = min(count, k + kFlush);
#pragma unroll 4
    for (; k < kend; ++k, g += stride) {
      add_group<HAS_W, SMALL, GENERIC>(s, J, wp, g, K, 4, k0, k1, ph, dist);
      if (HAS_W) wp += 4 * stride;
    }
    acc[0] += f2_sum(s.w1);
    acc[1] += f2_sum(s.w2);
    acc[2] += f2_sum(s.r1);
    acc[3] += f2_sum(s.r2);
  }
  const int tail = static_cast<int>(J.numel & 3);
  if (tail != 0 && local == 0 && threadIdx.x == 0) {
    GroupSums s;
    add_group<HAS_W, SMALL, GENERIC>(s, J, HAS_W ? J.W + 4 * full : nullptr, full, K, tail, k0, k1, ph,
                                     dist);
    acc[0] += f2_sum(s.w1);
    acc[1] += f2_sum(s.w2);
    acc[2] += f2_sum(s.r1);
    acc[3] += f2_sum(s.r2);
  }
}

// GENERIC: an auxiliary law other than Laplace (b.dist)
template <bool GENERIC>
__global__ void __launch_bounds__(kStatsThreads) stats_kernel(const __grid_constant__ StatsBatch b) {
  __shared__ double red[4 * 32];
  const int64_t bid = blockIdx.x;
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].block_begin <= bid) ++j;
  const StatsJob& J = b.job[j];
  const int64_t local = bid - J.block_begin;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  const bool small = J.numel < (int64_t{1} << 34);
  if (J.W != nullptr) {
    if (small) stats_body<true, true, GENERIC>(J, local, acc, b.key0, b.key1, b.dist);
    else stats_body<true, false, GENERIC>(J, local, acc, b.key0, b.key1, b.dist);
  } else {
    if (small) stats_body<false, true, GENERIC>(J, local, acc, b.key0, b.key1, b.dist);
    else stats_body<false, false, GENERIC>(J, local, acc, b.key0, b.key1, b.dist);
  }
  block_sum4(acc, red);
  if (threadIdx.x == 0)
    for (int q = 0; q < 4; ++q) J.partial[local * 4 + q] = acc[q];
}

__global__ void __launch_bounds__(kStatsThreads) stats_finalize_kernel(const __grid_constant__ StatsBatch b) {
  __shared__ double red[4 * 32];
  const StatsJob& J = b.job[blockIdx.x];
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int64_t k = threadIdx.x; k < J.nblocks; k += kStatsThreads)
    for (int q = 0; q < 4; ++q) acc[q] += J.partial[k * 4 + q];
  block_sum4(acc, red);
  if (threadIdx.x == 0) {
    const double N = static_cast<double>(J.numel);
    if (J.W != nullptr && J.sigma_w_out != nullptr) {
      const double var = (acc[1] - acc[0] * acc[0] / N) / N;
      *J.sigma_w_out = sqrt(fmax(var, 0.0));
    }
    if (J.sigma_r_out != nullptr) {
      const double var = (acc[3] - acc[2] * acc[2] / N) / N;   // Laplace: of R / ln 2
      *J.sigma_r_out = (b.dist == kDistLaplace ? kLn2d : 1.0) * sqrt(fmax(var, 0.0));
    }
  }
}

__global__ void zero_kernel(float* p, int64_t count) {
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < count;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[k] = 0.0f;
}

}  // namespace

cudaError_t launch_stats(const StatsBatch& b, int64_t total_blocks, cudaStream_t s) {
  if (b.dist == kDistLaplace)
    stats_kernel<false><<<static_cast<unsigned>(total_blocks), kStatsThreads, 0, s>>>(b);
  else
    stats_kernel<true><<<static_cast<unsigned>(total_blocks), kStatsThreads, 0, s>>>(b);
  return counted(cudaGetLastError());
}

cudaError_t launch_stats_finalize(const StatsBatch& b, cudaStream_t s) {
  stats_finalize_kernel<<<static_cast<unsigned>(b.count), kStatsThreads, 0, s>>>(b);
  return counted(cudaGetLastError());
}

cudaError_t launch_zero(float* p, int64_t count, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  const int64_t blocks = min64((count + 255) / 256, 148 * 8);
  zero_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(p, count);
  return counted(cudaGetLastError());
}

}  // namespace intlora
