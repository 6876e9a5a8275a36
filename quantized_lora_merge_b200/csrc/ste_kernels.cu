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
#include <cstring>

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

// Masked STE: the base code of element (row, col) and whether G is kept there
// (code != z: D != 0).
__device__ __forceinline__ bool mask_keep(const SteJob& J, int64_t row, int64_t col) {
  const uint8_t* rp = J.mcodes + row * J.mld;
  const int32_t code = J.mbits == 8 ? static_cast<int32_t>(__ldg(rp + col))
                                    : static_cast<int32_t>((__ldg(rp + (col >> 1)) >> (4 * (col & 1))) & 0xFu);
  return code != __ldg(J.mz + row);
}
// The same for the 4 consecutive columns c0..c0+3 (c0 % 4 == 0) of a row,
// applied to their bf16 values (2 per word).
__device__ __forceinline__ uint2 mask_bf16x4(const SteJob& J, int64_t row, int64_t c0, uint2 g) {
  const uint8_t* rp = J.mcodes + row * J.mld;
  uint32_t codes;
  if (J.mbits == 8) {
    codes = __ldg(reinterpret_cast<const uint32_t*>(rp + c0));
  } else {
    const uint32_t h = __ldg(reinterpret_cast<const uint16_t*>(rp + (c0 >> 1)));
    codes = (h & 0xFu) | ((h & 0xF0u) << 4) | ((h & 0xF00u) << 8) | ((h & 0xF000u) << 12);
  }
  const uint32_t z = static_cast<uint32_t>(__ldg(J.mz + row));
  const uint32_t k0 = ((codes & 0xFFu) != z) ? 0x0000FFFFu : 0u;
  const uint32_t k1 = (((codes >> 8) & 0xFFu) != z) ? 0xFFFF0000u : 0u;
  const uint32_t k2 = (((codes >> 16) & 0xFFu) != z) ? 0x0000FFFFu : 0u;
  const uint32_t k3 = ((codes >> 24) != z) ? 0xFFFF0000u : 0u;
  return make_uint2(g.x & (k0 | k1), g.y & (k2 | k3));
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
      if (m < M && k < kend) {
        const int64_t row = TRANS ? k : m, col = TRANS ? m : k;
        v = bf16f(J.G[row * J.n + col]);
        if (J.mcodes != nullptr && !mask_keep(J, row, col)) v = 0.0f;
      }
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

// Fused single pass over G for ranks up to 8 (CUDA cores). A CTA owns a strip
// of 128 columns and a range of rows; each lane owns 4 consecutive columns
// (one 8-byte load of G per row), keeps B[:, its columns] and its dB partial
// sums in registers, and forms the dA partial dot products of every row over
// its columns, which a warp shuffle tree sums over the strip. Partial sums of
// dA (per row and strip) and dB (per strip and row range) are added with fp32
// atomics into the zero-initialized outputs. G is read exactly once.
constexpr int kStripCols = 128;

__device__ __forceinline__ void unpack_bf16x4(uint2 raw, float out[4]) {
  out[0] = __uint_as_float(raw.x << 16);
  out[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  out[2] = __uint_as_float(raw.y << 16);
  out[3] = __uint_as_float(raw.y & 0xFFFF0000u);
}

// A[i, 0..RB) as floats (zero past r); one vector load when r == RB.
template <int RB>
__device__ __forceinline__ void load_a_row(const uint16_t* A, int64_t i, int r, float a[RB]) {
  if (r == RB && RB == 4) {
    unpack_bf16x4(__ldg(reinterpret_cast<const uint2*>(A + i * 4)), a);
  } else if (r == RB && RB == 8) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(A + i * 8));
    unpack_bf16x4(make_uint2(raw.x, raw.y), a);
    unpack_bf16x4(make_uint2(raw.z, raw.w), a + 4);
  } else {
#pragma unroll
    for (int k = 0; k < RB; ++k) a[k] = k < r ? bf16f(A[i * r + k]) : 0.0f;
  }
}

// Sum over the 32 lanes of each of the 32 values v[0..31] that every lane
// holds; lane L ends with the total of value index (L's bits in the order the
// halvings visit them). 31 shuffles for 32 sums instead of 5 per sum.
__device__ __forceinline__ float transpose_reduce32(float v[32], int lane) {
#pragma unroll
  for (int s = 16, half = 16; s >= 1; s >>= 1, half >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// Value index whose total lane L holds after transpose_reduce32: at the step
// with shuffle distance s the lanes with bit s set keep the upper half.
__device__ __forceinline__ int transpose_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int s = 16, half = 16; s >= 1; s >>= 1, half >>= 1)
    if (lane & s) idx += half;
  return idx;
}

template <int RB>
__global__ void __launch_bounds__(kSteThreads, 2) ste_fused_kernel(const __grid_constant__ SteBatch b) {
  int64_t t = blockIdx.x;
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].tile_begin <= t) ++j;
  const SteJob& J = b.job[j];
  t -= J.tile_begin;
  const int64_t n = J.n;
  const int r = J.r;
  const uint16_t* __restrict__ G = J.G;
  const uint16_t* __restrict__ A = J.A;
  const int strips = static_cast<int>((n + kStripCols - 1) / kStripCols);
  const int strip = static_cast<int>(t % strips);
  const int rchunk = static_cast<int>(t / strips);
  const int64_t rows_per = (J.d + J.ksplit - 1) / J.ksplit;
  const int64_t i_begin = rchunk * rows_per;
  const int64_t i_end = min64(J.d, i_begin + rows_per);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = static_cast<int64_t>(strip) * kStripCols + lane * 4;
  const bool col_ok = c0 < n;               // n % 8 == 0: a lane's 4 columns are all in or out

  float bv[RB][4];
#pragma unroll
  for (int k = 0; k < RB; ++k) {
    if (k < r && col_ok) unpack_bf16x4(__ldg(reinterpret_cast<const uint2*>(J.B + static_cast<int64_t>(k) * n + c0)), bv[k]);
    else bv[k][0] = bv[k][1] = bv[k][2] = bv[k][3] = 0.0f;
  }
  float dbacc[RB][4];
#pragma unroll
  for (int k = 0; k < RB; ++k) dbacc[k][0] = dbacc[k][1] = dbacc[k][2] = dbacc[k][3] = 0.0f;

  // Rows in groups of RG = 32 / RB per warp: the RG x RB partial dot products
  // of dA are summed over the lanes by one transpose-reduce.
  constexpr int RG = 32 / RB;
  constexpr int kWarps = kSteThreads / 32;
  const int my_idx = transpose_index(lane);
  const int my_row = my_idx / RB, my_k = my_idx % RB;
  for (int64_t i0 = i_begin + warp * RG; i0 < i_end; i0 += kWarps * RG) {
    float P[32];
    // all RG rows of G are requested before any is used (RG loads in flight)
    uint2 graw[RG];
#pragma unroll
    for (int u = 0; u < RG; ++u) {
      const int64_t i = i0 + u;
      graw[u] = (i < i_end && col_ok) ? __ldg(reinterpret_cast<const uint2*>(G + i * n + c0))
                                      : make_uint2(0u, 0u);
      if (J.mcodes != nullptr && i < i_end && col_ok) graw[u] = mask_bf16x4(J, i, c0, graw[u]);
    }
#pragma unroll
    for (int u = 0; u < RG; ++u) {
      const int64_t i = i0 + u;
      float a[RB];
      if (i < i_end) load_a_row<RB>(A, i, r, a);
      else
#pragma unroll
        for (int k = 0; k < RB; ++k) a[k] = 0.0f;
      float g[4];
      unpack_bf16x4(graw[u], g);
#pragma unroll
      for (int k = 0; k < RB; ++k) {
        float acc = g[0] * bv[k][0];
#pragma unroll
        for (int c = 1; c < 4; ++c) acc = fmaf(g[c], bv[k][c], acc);
        P[u * RB + k] = acc;
#pragma unroll
        for (int c = 0; c < 4; ++c) dbacc[k][c] = fmaf(a[k], g[c], dbacc[k][c]);
      }
    }
    const float total = transpose_reduce32(P, lane);
    const int64_t row = i0 + my_row;
    if (row < i_end && my_k < r) atomicAdd(&J.dA[row * r + my_k], total);
  }
  if (col_ok) {
#pragma unroll
    for (int k = 0; k < RB; ++k) {
      if (k >= r) break;
#pragma unroll
      for (int c = 0; c < 4; ++c) atomicAdd(&J.dB[static_cast<int64_t>(k) * n + c0 + c], dbacc[k][c]);
    }
  }
}

// Zero the outputs that split-K CTAs accumulate into (one launch per batch).
__global__ void ste_zero_kernel(const __grid_constant__ SteBatch b) {
  for (int j = 0; j < b.count; ++j) {
    const SteJob& J = b.job[j];
    const bool both = b.fused != 0;
    for (int which = 0; which < 2; ++which) {
      const bool is_db = which == 1;
      if (!both && (J.ksplit <= 1 || is_db != (b.transposed != 0))) continue;
      float* p = is_db ? J.dB : J.dA;
      const int64_t count = is_db ? static_cast<int64_t>(J.r) * J.n : J.d * J.r;
      for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < count;
           k += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[k] = 0.0f;
    }
  }
}

}  // namespace

namespace {

// Zeroing of many small buffers in one launch: every CTA clears one chunk of
// kZeroChunk floats of one segment.
constexpr int kZeroSegments = 2 * kMaxBatch;
constexpr int kZeroChunk = 4096;
struct ZeroBatch {
  float* ptr[kZeroSegments];
  int64_t count[kZeroSegments];
  int32_t block_begin[kZeroSegments + 1];
  int32_t segments;
};

__global__ void __launch_bounds__(256) zero_segments_kernel(const __grid_constant__ ZeroBatch z) {
  const int bid = blockIdx.x;
  int lo = 0, hi = z.segments - 1;         // last segment whose first block <= bid
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (z.block_begin[mid] <= bid) lo = mid;
    else hi = mid - 1;
  }
  const int64_t base = static_cast<int64_t>(bid - z.block_begin[lo]) * kZeroChunk;
  const int64_t end = min64(z.count[lo], base + kZeroChunk);
  float* p = z.ptr[lo];
  for (int64_t k = base + threadIdx.x; k < end; k += 256) p[k] = 0.0f;
}

}  // namespace

namespace {
constexpr int kMaskChunk = 256 * 8;      // octets per CTA step

struct MaskBatch {
  MaskJob job[kMaxBatch];
  int64_t chunk_begin[kMaxBatch + 1];     // CTA steps before job k
  int32_t count;
};

// Octets (8 consecutive elements of a row) in chunks of kMaskChunk, each
// chunk inside one job: a 16-byte load of G and of its codes' bytes when the
// row allows it, else element by element.
__global__ void __launch_bounds__(256) mask_g_kernel(const __grid_constant__ MaskBatch b) {
  const int64_t total = b.chunk_begin[b.count];
  int k = 0;
  for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
    while (k + 1 < b.count && b.chunk_begin[k + 1] <= c) ++k;       // chunks only increase
    const MaskJob& J = b.job[k];
    const int64_t per_row = (J.n + 7) / 8;
    const int64_t octets = J.d * per_row;
    const int64_t o_begin = (c - b.chunk_begin[k]) * kMaskChunk;
    const int64_t o_end = min64(octets, o_begin + kMaskChunk);
    for (int64_t o = o_begin + threadIdx.x; o < o_end; o += blockDim.x) {
      const int64_t i = o / per_row;
      const int64_t j0 = (o - i * per_row) * 8;
      const uint8_t* crow = J.codes + i * J.ld;
      const uint32_t z = static_cast<uint32_t>(__ldg(J.z + i));
      const uint16_t* src = J.G + i * J.n + j0;
      uint16_t* dst = J.out + i * J.n + j0;
      if (J.n % 8 == 0) {
        uint4 g = __ldg(reinterpret_cast<const uint4*>(src));
        uint32_t c[8];
        if (J.bits == 8) {
          const uint2 cb = __ldg(reinterpret_cast<const uint2*>(crow + j0));
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            c[q] = (cb.x >> (8 * q)) & 0xFFu;
            c[q + 4] = (cb.y >> (8 * q)) & 0xFFu;
          }
        } else {
          const uint32_t cw = __ldg(reinterpret_cast<const uint32_t*>(crow + (j0 >> 1)));
  #pragma unroll
          for (int q = 0; q < 8; ++q) c[q] = (cw >> (4 * q)) & 0xFu;
        }
        uint32_t* gw = reinterpret_cast<uint32_t*>(&g);
  #pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = c[2 * q] != z ? 0x0000FFFFu : 0u;
          const uint32_t hi = c[2 * q + 1] != z ? 0xFFFF0000u : 0u;
          gw[q] &= lo | hi;
        }
        *reinterpret_cast<uint4*>(dst) = g;
      } else {
        for (int q = 0; q < 8 && j0 + q < J.n; ++q) {
          const int64_t j = j0 + q;
          const uint32_t code = J.bits == 8 ? crow[j] : (crow[j >> 1] >> (4 * (j & 1))) & 0xFu;
          dst[q] = code != z ? src[q] : static_cast<uint16_t>(0);
        }
      }
    }
  }
}
}  // namespace

cudaError_t launch_mask_g(const MaskJob* jobs, int count, cudaStream_t s) {
  static thread_local MaskBatch b;
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    std::memset(&b, 0, sizeof b);
    int64_t chunks = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.chunk_begin[k] = chunks;
      chunks += (jobs[k0 + k].d * ((jobs[k0 + k].n + 7) / 8) + kMaskChunk - 1) / kMaskChunk;
    }
    b.chunk_begin[m] = chunks;
    b.count = m;
    if (chunks == 0) continue;
    const int64_t blocks = min64(chunks, 148 * 8);
    mask_g_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_ste_zero(const SteBatch& b, cudaStream_t s) {
  if (b.count <= 0) return cudaSuccess;
  ZeroBatch z;
  std::memset(&z, 0, sizeof z);
  int blocks = 0, seg = 0;
  for (int j = 0; j < b.count; ++j) {
    const SteJob& J = b.job[j];
    const int64_t counts[2] = {J.d * J.r, static_cast<int64_t>(J.r) * J.n};
    float* ptrs[2] = {J.dA, J.dB};
    for (int w = 0; w < 2; ++w) {
      if (counts[w] <= 0) continue;
      z.ptr[seg] = ptrs[w];
      z.count[seg] = counts[w];
      z.block_begin[seg] = blocks;
      blocks += static_cast<int>((counts[w] + kZeroChunk - 1) / kZeroChunk);
      ++seg;
    }
  }
  z.segments = seg;
  z.block_begin[seg] = blocks;
  if (blocks == 0) return cudaSuccess;
  zero_segments_kernel<<<blocks, 256, 0, s>>>(z);
  return counted(cudaGetLastError());
}

cudaError_t launch_ste(const SteBatch& b, cudaStream_t s) {
  if (b.count <= 0) return cudaSuccess;
  if (b.fused) {
    cudaError_t e = launch_ste_zero(b, s);
    if (e != cudaSuccess) return e;
    if (b.fused == 4)
      ste_fused_kernel<4><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
    else
      ste_fused_kernel<8><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
    return counted(cudaGetLastError());
  }
  bool any_split = false;
  for (int j = 0; j < b.count; ++j) any_split = any_split || b.job[j].ksplit > 1;
  if (any_split) {
    ste_zero_kernel<<<148 * 4, 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  if (!b.transposed)
    ste_gemm_kernel<false><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
  else
    ste_gemm_kernel<true><<<static_cast<unsigned>(b.total_tiles), kSteThreads, 0, s>>>(b);
  return counted(cudaGetLastError());
}

}  // namespace intlora
