// Small kernels of the IntLoRA training backward (the linear Y = X W'^T with
// W' the quantized merged weight; the gradient reaches A and B through the
// straight-through estimator [IntLoRA paper notes (ICML2025), method section,
// the two variants: training passes the quantizers with the STE]).
//
// The backward is composed on the host (intlora_train_backward_batched) from
// the library's tensor-core kernels without ever forming the weight gradient
// G = dY^T X (d x n): with Z1 = X B^T and Z2 = dY A (tokens x r),
//   dA = G B^T = dY^T Z1,   dB = A^T G = Z2^T X,   dX = dY W'.
// The kernels here do the glue: a tiled bf16 transpose (W'^T and A^T, so
// every GEMM operand is K-major), the exact split of Z into two bf16 halves
// (Z = hi + lo to ~2^-17, so the bf16 tensor-core products stay
// fp32-faithful), and the final sum of the two halves' products.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "intlora_device.cuh"
#include "intlora_kernels.h"

namespace intlora {

namespace {

constexpr int kTrTile = 32;

struct TrBatch {
  TransposeJob job[kMaxBatch];
  int32_t count;
};

// out[c][r] = in[r][c] for one rows x cols bf16 matrix per job; a CTA moves a
// 32 x 32 tile through shared memory (coalesced reads and writes). Jobs are
// laid end to end over blockIdx.x by their tile counts.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __grid_constant__ TrBatch b) {
  __shared__ uint16_t tile[kTrTile][kTrTile + 1];
  int64_t bid = blockIdx.x;
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].block_begin <= bid) ++j;
  const TransposeJob& J = b.job[j];
  bid -= J.block_begin;
  const int64_t tiles_c = (J.cols + kTrTile - 1) / kTrTile;
  const int64_t r0 = (bid / tiles_c) * kTrTile, c0 = (bid % tiles_c) * kTrTile;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;    // 32 x 8 threads
  for (int y = ty; y < kTrTile; y += 8) {
    const int64_t r = r0 + y, c = c0 + tx;
    tile[y][tx] = (r < J.rows && c < J.cols) ? J.in[r * J.cols + c] : uint16_t{0};
  }
  __syncthreads();
  for (int y = ty; y < kTrTile; y += 8) {
    const int64_t c = c0 + y, r = r0 + tx;                    // output row c, column r
    if (c < J.cols && r < J.rows) J.out[c * J.rows + r] = tile[tx][y];
  }
}

struct SplitZBatch {
  SplitZJob job[kMaxBatch];
  int32_t count;
};

// Zs[t][k] = bf16(Z[t][k]) and Zs[t][r + k] = bf16(Z[t][k] - Zs[t][k]): the
// head rounded to nearest even, the tail (exact in fp32) rounded likewise.
__global__ void __launch_bounds__(256) split_hilo_kernel(const __grid_constant__ SplitZBatch b) {
  for (int j = 0; j < b.count; ++j) {
    const SplitZJob& J = b.job[j];
    const int64_t total = J.rows * J.r;
    for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < total; e += static_cast<int64_t>(gridDim.x) * 256) {
      const int64_t t = e / J.r;
      const int k = static_cast<int>(e - t * J.r);
      const float z = J.z[e];
      const __nv_bfloat16 hi = __float2bfloat16_rn(z);
      const __nv_bfloat16 lo = __float2bfloat16_rn(z - __bfloat162float(hi));
      __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(J.zs) + t * 2 * J.r;
      row[k] = hi;
      row[J.r + k] = lo;
    }
  }
}

struct CombineBatch {
  CombineJob job[kMaxBatch];
  int32_t count;
};

// out = top + bottom of a 2r x cols product (the head and tail halves of Z),
// written transposed (cols x r) when `transposed` is set.
__global__ void __launch_bounds__(256) combine_halves_kernel(const __grid_constant__ CombineBatch b) {
  for (int j = 0; j < b.count; ++j) {
    const CombineJob& J = b.job[j];
    const int64_t total = static_cast<int64_t>(J.r) * J.cols;
    for (int64_t e = blockIdx.x * 256 + threadIdx.x; e < total; e += static_cast<int64_t>(gridDim.x) * 256) {
      const int64_t k = e / J.cols;
      const int64_t c = e - k * J.cols;
      const float v = J.in[k * J.cols + c] + J.in[(k + J.r) * J.cols + c];
      if (J.transposed) J.out[c * J.r + k] = v;
      else J.out[e] = v;
    }
  }
}

}  // namespace

cudaError_t launch_transpose_bf16(const TransposeJob* jobs, int count, cudaStream_t s) {
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    static thread_local TrBatch b;
    std::memset(&b, 0, sizeof b);
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    int64_t blocks = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.job[k].block_begin = blocks;
      blocks += ((jobs[k0 + k].rows + kTrTile - 1) / kTrTile) * ((jobs[k0 + k].cols + kTrTile - 1) / kTrTile);
    }
    b.count = m;
    if (blocks == 0) continue;
    transpose_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_split_hilo(const SplitZJob* jobs, int count, cudaStream_t s) {
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    static thread_local SplitZBatch b;
    std::memset(&b, 0, sizeof b);
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    int64_t most = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      most = jobs[k0 + k].rows * jobs[k0 + k].r > most ? jobs[k0 + k].rows * jobs[k0 + k].r : most;
    }
    b.count = m;
    if (most == 0) continue;
    const int64_t blocks = min64((most + 255) / 256, 148 * 8);
    split_hilo_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_combine_halves(const CombineJob* jobs, int count, cudaStream_t s) {
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    static thread_local CombineBatch b;
    std::memset(&b, 0, sizeof b);
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    int64_t most = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      const int64_t t = static_cast<int64_t>(jobs[k0 + k].r) * jobs[k0 + k].cols;
      most = t > most ? t : most;
    }
    b.count = m;
    if (most == 0) continue;
    const int64_t blocks = min64((most + 255) / 256, 148 * 8);
    combine_halves_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace intlora
