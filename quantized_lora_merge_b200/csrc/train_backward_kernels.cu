// Small kernels of the IntLoRA training backward (the linear Y = X W'^T with
// W' the quantized merged weight; the gradient reaches A and B through the
// straight-through estimator [IntLoRA paper notes (ICML2025), method section,
// the two variants: training passes the quantizers with the STE]).
//
// The backward is composed on the host (intlora_train_backward_batched) from
// the library's tensor-core kernels without ever forming the weight gradient
// G = dY^T X (d x n): with Z1 = X B^T and Z2 = dY A (tokens x r),
//   dA = G B^T = dY^T Z1,   dB = A^T G = Z2^T X,   dX = dY W'.
// The low-rank products run as passes of the STE kernel, which reads a
// tokens x m activation once and forms both of its products (against an
// r-row operand and a tokens x r operand): X -> Z1; dY -> Z2 and dA; X -> dB.
// The kernels here do the glue: a tiled bf16 transpose (W'^T for the dX
// GEMM, A^T for the dY pass), the exact split of Z into two bf16 halves
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

constexpr int kTrTile = 64;
constexpr int kGlueCtas = 148 * 8;             // persistent grids: a few CTAs per SM walk the work

struct TrBatch {
  TransposeJob job[kMaxBatch];
  int32_t count;
  int64_t total;                               // tiles of all jobs
};

// Index of the job whose range [begin[j], begin[j + 1]) holds x (begin
// ascending, begin[0] = 0): a binary search over the batch.
template <typename J>
__device__ __forceinline__ int find_job(const J* job, int count, int64_t x) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (job[mid].block_begin <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// out[c][r] = in[r][c] for one rows x cols bf16 matrix per job. A CTA moves
// 64 x 64 tiles through shared memory with 16-byte global loads and stores
// (8 elements a thread per access; scalar at ragged edges or when a row
// length is not a multiple of 8), walking the tiles of all jobs with a grid
// stride. Shared memory holds a tile row as 8 chunks of 8 elements, chunk q
// of row y at position q ^ (y & 7) ^ ((y >> 3) & 7): row writes and the
// column gathers of the write phase are both free of bank conflicts.
__device__ __forceinline__ int tr_chunk(int y, int q) { return q ^ (y & 7) ^ ((y >> 3) & 7); }

__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __grid_constant__ TrBatch b) {
  __shared__ __align__(16) uint16_t tile[kTrTile * kTrTile];
  for (int64_t t = blockIdx.x; t < b.total; t += gridDim.x) {
    const TransposeJob& J = b.job[find_job(b.job, b.count, t)];
    const int64_t local = t - J.block_begin;
    const int64_t tiles_c = (J.cols + kTrTile - 1) / kTrTile;
    const int64_t r0 = (local / tiles_c) * kTrTile, c0 = (local % tiles_c) * kTrTile;
    const bool vec_in = (J.cols & 7) == 0, vec_out = (J.rows & 7) == 0;
    __syncthreads();                                          // the last tile's reads are done
    for (int c = threadIdx.x; c < kTrTile * 8; c += 256) {
      const int y = c >> 3, q = c & 7;
      const int64_t r = r0 + y, col = c0 + 8 * q;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < J.rows) {
        const uint16_t* src = J.in + r * J.cols + col;
        if (vec_in && col + 8 <= J.cols) {
          v = __ldg(reinterpret_cast<const uint4*>(src));
        } else {
          uint16_t e[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) e[k] = col + k < J.cols ? src[k] : uint16_t{0};
          v = make_uint4(e[0] | (static_cast<uint32_t>(e[1]) << 16), e[2] | (static_cast<uint32_t>(e[3]) << 16),
                         e[4] | (static_cast<uint32_t>(e[5]) << 16), e[6] | (static_cast<uint32_t>(e[7]) << 16));
        }
      }
      *reinterpret_cast<uint4*>(tile + y * kTrTile + 8 * tr_chunk(y, q)) = v;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < kTrTile * 8; c += 256) {
      const int oy = c >> 3, oq = c & 7;                      // output row c0 + oy, columns r0 + 8 oq ..
      const int64_t orow = c0 + oy, ocol = r0 + 8 * oq;
      if (orow >= J.cols || ocol >= J.rows) continue;
      uint16_t e[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int y = 8 * oq + k;
        e[k] = tile[y * kTrTile + 8 * tr_chunk(y, oy >> 3) + (oy & 7)];
      }
      uint16_t* dst = J.out + orow * J.rows + ocol;
      if (vec_out && ocol + 8 <= J.rows) {
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(e[0] | (static_cast<uint32_t>(e[1]) << 16), e[2] | (static_cast<uint32_t>(e[3]) << 16),
                       e[4] | (static_cast<uint32_t>(e[5]) << 16), e[6] | (static_cast<uint32_t>(e[7]) << 16));
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (ocol + k < J.rows) dst[k] = e[k];
      }
    }
  }
}

struct SplitZBatch {
  SplitZJob job[kMaxBatch];
  int64_t begin[kMaxBatch + 1];                // element offsets of the jobs
  int32_t count;
};
__device__ __forceinline__ int find_offset(const int64_t* begin, int count, int64_t x) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (begin[mid] <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Zs[t][k] = bf16(Z[t][k]) and Zs[t][r + k] = bf16(Z[t][k] - Zs[t][k]): the
// head rounded to nearest even, the tail (exact in fp32) rounded likewise.
// Z is read with a row stride (the first r columns of a wider product). One
// flat element index over all jobs.
__global__ void __launch_bounds__(256) split_hilo_kernel(const __grid_constant__ SplitZBatch b) {
  const int64_t total = b.begin[b.count];
  for (int64_t x = blockIdx.x * 256 + threadIdx.x; x < total; x += static_cast<int64_t>(gridDim.x) * 256) {
    const int j = find_offset(b.begin, b.count, x);
    const SplitZJob& J = b.job[j];
    const int64_t e = x - b.begin[j];
    const int64_t t = e / J.r;
    const int k = static_cast<int>(e - t * J.r);
    const float z = J.z[t * J.ld + k];
    const __nv_bfloat16 hi = __float2bfloat16_rn(z);
    const __nv_bfloat16 lo = __float2bfloat16_rn(z - __bfloat162float(hi));
    __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(J.zs) + t * 2 * J.r;
    row[k] = hi;
    row[J.r + k] = lo;
  }
}

struct CombineBatch {
  CombineJob job[kMaxBatch];
  int64_t begin[kMaxBatch + 1];
  int32_t count;
};

// out = top + bottom of a 2r x cols product (the head and tail halves of Z),
// written transposed (cols x r) when `transposed` is set. One flat element
// index over all jobs.
__global__ void __launch_bounds__(256) combine_halves_kernel(const __grid_constant__ CombineBatch b) {
  const int64_t total = b.begin[b.count];
  for (int64_t x = blockIdx.x * 256 + threadIdx.x; x < total; x += static_cast<int64_t>(gridDim.x) * 256) {
    const int j = find_offset(b.begin, b.count, x);
    const CombineJob& J = b.job[j];
    const int64_t e = x - b.begin[j];
    const int64_t k = e / J.cols;
    const int64_t c = e - k * J.cols;
    const float v = J.in[k * J.cols + c] + J.in[(k + J.r) * J.cols + c];
    if (J.transposed) J.out[c * J.r + k] = v;
    else J.out[e] = v;
  }
}

}  // namespace

cudaError_t launch_transpose_bf16(const TransposeJob* jobs, int count, cudaStream_t s) {
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    static thread_local TrBatch b;
    std::memset(&b, 0, sizeof b);
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    int64_t tiles = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.job[k].block_begin = tiles;
      tiles += ((jobs[k0 + k].rows + kTrTile - 1) / kTrTile) * ((jobs[k0 + k].cols + kTrTile - 1) / kTrTile);
    }
    b.count = m;
    b.total = tiles;
    if (tiles == 0) continue;
    transpose_bf16_kernel<<<static_cast<unsigned>(min64(tiles, kGlueCtas)), 256, 0, s>>>(b);
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
    int64_t total = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.begin[k] = total;
      total += jobs[k0 + k].rows * jobs[k0 + k].r;
    }
    b.begin[m] = total;
    b.count = m;
    if (total == 0) continue;
    split_hilo_kernel<<<static_cast<unsigned>(min64((total + 255) / 256, kGlueCtas)), 256, 0, s>>>(b);
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
    int64_t total = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.begin[k] = total;
      total += static_cast<int64_t>(jobs[k0 + k].r) * jobs[k0 + k].cols;
    }
    b.begin[m] = total;
    b.count = m;
    if (total == 0) continue;
    combine_halves_kernel<<<static_cast<unsigned>(min64((total + 255) / 256, kGlueCtas)), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace intlora
