// STE backward of IntLoRA [IntLoRA paper notes (ICML2025), "两种实现版本":
// training passes gradients through the quantizers with the straight-through
// estimator], so with G the upstream gradient on W' (d x n):
//     dA = G B^T   (d x r),       dB = A^T G   (r x n).
// Both are contractions over a long axis of G (n for dA, d for dB).
//
// CUDA-core path: one tiled kernel computes OUT[M][r] = X[M][K] Y[K][r] with
// X = G, Y = B^T for dA and X = G^T, Y = A for dB^T (stored transposed into
// dB). 64 x 64 tiles of G are staged in shared memory as fp32 (transposed so
// one 16-byte load gives a thread its 4 rows), each thread keeps a 4 x 2 block
// of the output in registers, and K is split over CTAs whose partial sums are
// added with fp32 atomics into the zero-initialized output.
#include <cuda_runtime.h>

#include <cstdint>

#include "intlora_device.cuh"
#include "intlora_kernels.h"

namespace intlora {

namespace {

constexpr int kSteThreads = 256;
constexpr int kBM = 64;   // output rows per CTA
constexpr int kBK = 64;   // reduction slice per stage
constexpr int kRB = 32;   // output columns (rank) per CTA

__device__ __forceinline__ float bf16f(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

template <bool TRANS>
__global__ void __launch_bounds__(kSteThreads) ste_gemm_kernel(const __grid_constant__ SteBatch b) {
  __shared__ __align__(16) float Xs[kBK][kBM + 4];
  __shared__ __align__(16) float Ys[kBK][kRB + 2];

  int64_t t = blockIdx.x;
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].tile_begin <= t) ++j;
  const SteJob& J = b.job[j];
  t -= J.tile_begin;
  const int64_t M = TRANS ? J.n : J.d;
  const int64_t K = TRANS ? J.d : J.n;
  const int r = J.r;
  const int mtiles = static_cast<int>((M + kBM - 1) / kBM);
  const int rtiles = (r + kRB - 1) / kRB;
  const int ksplit = J.ksplit;
  const int mt = static_cast<int>(t % mtiles);
  const int rt = static_cast<int>((t / mtiles) % rtiles);
  const int ks = static_cast<int>(t / (static_cast<int64_t>(mtiles) * rtiles));
  const int64_t m0 = static_cast<int64_t>(mt) * kBM;
  const int k0r = rt * kRB;
  const int64_t kper = ((K + ksplit - 1) / ksplit + kBK - 1) / kBK * kBK;
  const int64_t kbeg = ks * kper;
  const int64_t kend = min64(K, kbeg + kper);

  const int tid = threadIdx.x;
  const int tr = tid & 15;          // row group: rows 4 tr .. 4 tr + 3
  const int tc = tid >> 4;          // column pair: 2 tc, 2 tc + 1
  float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};

  for (int64_t kb = kbeg; kb < kend; kb += kBK) {
    // stage X^T tile: Xs[kk][mm] = X[m0 + mm][kb + kk]
    for (int idx = tid; idx < kBK * kBM; idx += kSteThreads) {
      int kk, mm;
      if (TRANS) { kk = idx / kBM; mm = idx % kBM; }   // coalesced along m (= G column)
      else { mm = idx / kBK; kk = idx % kBK; }         // coalesced along k (= G column)
      const int64_t m = m0 + mm, k = kb + kk;
      float v = 0.0f;
      if (m < M && k < kend) v = TRANS ? bf16f(J.G[k * J.n + m]) : bf16f(J.G[m * J.n + k]);
      Xs[kk][mm] = v;
    }
    // stage Y tile: Ys[kk][c] = Y[kb + kk][k0r + c]
    for (int idx = tid; idx < kBK * kRB; idx += kSteThreads) {
      int kk, c;
      if (TRANS) { kk = idx / kRB; c = idx % kRB; }    // A row-major: rank contiguous
      else { c = idx / kBK; kk = idx % kBK; }          // B row-major: k contiguous
      const int64_t k = kb + kk;
      const int rc = k0r + c;
      float v = 0.0f;
      if (rc < r && k < kend) v = TRANS ? bf16f(J.A[k * r + rc]) : bf16f(J.B[rc * J.n + k]);
      Ys[kk][c] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kBK; ++kk) {
      const float4 x = *reinterpret_cast<const float4*>(&Xs[kk][4 * tr]);
      const float2 y = *reinterpret_cast<const float2*>(&Ys[kk][2 * tc]);
      const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        acc[a][0] = fmaf(xv[a], y.x, acc[a][0]);
        acc[a][1] = fmaf(xv[a], y.y, acc[a][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t m = m0 + 4 * tr + a;
    if (m >= M) continue;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int rc = k0r + 2 * tc + c;
      if (rc >= r) continue;
      float* dst = TRANS ? &J.dB[static_cast<int64_t>(rc) * J.n + m] : &J.dA[m * r + rc];
      if (ksplit > 1) atomicAdd(dst, acc[a][c]);
      else *dst = acc[a][c];
    }
  }
}

// Zero the outputs that split-K CTAs accumulate into (one launch per batch).
__global__ void ste_zero_kernel(const __grid_constant__ SteBatch b) {
  for (int j = 0; j < b.count; ++j) {
    const SteJob& J = b.job[j];
    if (J.ksplit <= 1) continue;
    float* p = b.transposed ? J.dB : J.dA;
    const int64_t count = b.transposed ? static_cast<int64_t>(J.r) * J.n : J.d * J.r;
    for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < count;
         k += static_cast<int64_t>(gridDim.x) * blockDim.x)
      p[k] = 0.0f;
  }
}

}  // namespace

cudaError_t launch_ste(const SteBatch& b, cudaStream_t s) {
  if (b.count <= 0) return cudaSuccess;
  bool any_split = false;
  for (int j = 0; j < b.count; ++j) any_split = any_split || b.job[j].ksplit > 1;
  if (any_split) ste_zero_kernel<<<148 * 4, 256, 0, s>>>(b);
  if (!b.transposed)
    ste_gemm_kernel<false><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
  else
    ste_gemm_kernel<true><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
  return cudaGetLastError();
}

}  // namespace intlora
