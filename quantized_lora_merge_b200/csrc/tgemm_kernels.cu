// Low-rank product T = A B of the IntLoRA merge on the 5th-generation tensor
// cores, for the larger ranks [IntLoRA paper notes (ICML2025), method
// section 2, MLA: U = s + (R* + A B) / D]. At r >= 32 the product costs more
// CUDA-core FMAs per merged element than everything else the merge does, so
// it is computed once per layer into a workspace and the row kernels read T.
//
// Precision: a "3-term split" on tf32. Each fp32 operand x is split exactly
// into x_hi (x rounded to tf32, low 13 mantissa bits zero) and x_lo = x - x_hi
// (rounded to tf32 as well); A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi with fp32
// accumulation. The dropped A_lo B_lo and the rounding of the lo parts are
// ~2^-21 of |A||B| per term, below the fp32 rounding of a CUDA-core dot
// product of the same length.
//
// Layout: a split kernel writes A_hi, A_lo (d x kp) and B^T_hi, B^T_lo
// (n x kp), kp = r rounded up to 32 (one 128-byte row of fp32), zero padded,
// so both MMA operands are K-major. The GEMM kernel gives a CTA units of 128
// rows x a run of 128-column tiles: TMA loads the unit's A_hi / A_lo once and
// the B tiles through a pipeline; one thread issues
// tcgen05.mma.cta_group::1.kind::tf32 (M = N = 128, K = 8 per instruction,
// three per K step) into a double-buffered TMEM accumulator, and four warps
// drain it (tcgen05.ld) into T rows with 16-byte stores.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>

#include "intlora_device.cuh"
#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

using namespace tc;

constexpr int kTgThreads = 256;
constexpr int kTgRows = 128;                      // tile rows (M)
constexpr int kTgCols = 128;                      // tile columns (N)
constexpr uint32_t kAtomBytes = kTgRows * 128;    // 128 rows x 32 fp32 (one K atom)
constexpr int kMaxTgJobs = 48;
constexpr int kTgMaxStages = 6;                   // pipeline stages at most (host picks 2-6)

__device__ unsigned int g_tg_timeouts;

__device__ __forceinline__ bool wait_c(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait(bar, parity, abort_flag, &g_tg_timeouts);
}

// ---- split ---------------------------------------------------------------------
struct SplitJob {
  const float* A;
  const float* B;
  float* a_hi;
  float* a_lo;
  float* b_hi;
  float* b_lo;
  int64_t d, n;
  int32_t r, kp;
  int64_t block_begin;
};
struct SplitBatch {
  SplitJob job[kMaxBatch];
  int32_t count;
  int64_t total_blocks;
};
constexpr int kSplitPerBlock = 256 * 4;

__device__ __forceinline__ float tf32_round(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
}

__global__ void __launch_bounds__(256) t_split_kernel(const __grid_constant__ SplitBatch b) {
  const int64_t bid = blockIdx.x;
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].block_begin <= bid) ++j;
  const SplitJob& J = b.job[j];
  const int64_t na = J.d * J.kp, total = (J.d + J.n) * J.kp;
  const int64_t base = (bid - J.block_begin) * kSplitPerBlock;
  for (int64_t idx = base + threadIdx.x; idx < min64(total, base + kSplitPerBlock); idx += 256) {
    float v;
    if (idx < na) {
      const int64_t i = idx / J.kp;
      const int k = static_cast<int>(idx - i * J.kp);
      v = k < J.r ? __ldg(J.A + i * J.r + k) : 0.0f;
    } else {
      const int64_t jn = (idx - na) / J.kp;
      const int k = static_cast<int>(idx - na - jn * J.kp);
      v = k < J.r ? __ldg(J.B + static_cast<int64_t>(k) * J.n + jn) : 0.0f;
    }
    const float hi = tf32_round(v);
    const float lo = tf32_round(v - hi);
    if (idx < na) {
      J.a_hi[idx] = hi;
      J.a_lo[idx] = lo;
    } else {
      J.b_hi[idx - na] = hi;
      J.b_lo[idx - na] = lo;
    }
  }
}

// ---- GEMM ----------------------------------------------------------------------
struct alignas(64) TgJob {
  CUtensorMap a_hi, a_lo, b_hi, b_lo;   // {kp, rows}, box {32, 128}, 128B swizzle
  float* T;                              // d x n
  int64_t d, n;
  int32_t kp;
  int32_t col_tiles;
  int32_t chunks;
  int32_t pad;
  int64_t unit_begin;
};
struct TgBatch {
  TgJob job[kMaxTgJobs];
  int32_t count;
  int32_t kp_max;                        // shared memory is carved for this K
  int32_t stages;
  int32_t tiles_per_unit;
  int64_t total_units;
};

struct TgUnit {
  int job;
  int64_t i0;
  int ct0, ct1;
};
__device__ __forceinline__ TgUnit tg_unit(const TgBatch& b, int64_t u) {
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].unit_begin <= u) ++j;
  const TgJob& J = b.job[j];
  const int64_t local = u - J.unit_begin;
  const int64_t rb = local / J.chunks;
  const int cc = static_cast<int>(local - rb * J.chunks);
  TgUnit x;
  x.job = j;
  x.i0 = rb * kTgRows;
  x.ct0 = cc * b.tiles_per_unit;
  x.ct1 = min(J.col_tiles, x.ct0 + b.tiles_per_unit);
  return x;
}

// kind::tf32, fp32 D, both operands K-major, M = N = 128.
constexpr uint32_t kTgIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(kTgCols >> 3) << 17) |
                              (static_cast<uint32_t>(kTgRows >> 4) << 24);

__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kTgIdesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kTgThreads, 1) t_gemm_kernel(const __grid_constant__ TgBatch b) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ __align__(8) uint64_t drain_bar;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const int S = b.stages;
  const uint32_t op_bytes = static_cast<uint32_t>(b.kp_max / 32) * kAtomBytes;   // one operand tile
  uint8_t* sA = base;                                   // A_hi | A_lo of the unit
  uint8_t* sB = sA + 2 * op_bytes;                      // [S] x (B_hi | B_lo)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S * 2 * op_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* a_full = bars + 2 * S;
  uint64_t* a_empty = a_full + 1;
  uint64_t* d_full = a_full + 2;                        // [2]
  uint64_t* d_empty = a_full + 4;                       // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&d_full[q], 1);
      mbar_init(&d_empty[q], 128);
    }
    abort_flag = 0;
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(2 * kTgCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;                      // D[q] at column q * 128

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0, ucount = 0;
      uint32_t ph = 0;
      int armed[kTgMaxStages], armed_a = -1;     // parity last armed per barrier (-1: never)
      for (int q = 0; q < kTgMaxStages; ++q) armed[q] = -1;
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x, ++ucount) {
        const TgUnit x = tg_unit(b, u);
        const TgJob& J = b.job[x.job];
        const int atoms = J.kp / 32;
        const int32_t y0 = static_cast<int32_t>(x.i0);
        if (!wait_c(a_empty, (static_cast<uint32_t>(ucount) & 1u) ^ 1u, &abort_flag)) break;
        mbar_arrive_tx(a_full, 2u * atoms * kAtomBytes);
        armed_a = ucount & 1;
        for (int at = 0; at < atoms; ++at) {
          tma_load_2d(sA + at * kAtomBytes, &J.a_hi, at * 32, y0, a_full);
          tma_load_2d(sA + op_bytes + at * kAtomBytes, &J.a_lo, at * 32, y0, a_full);
        }
        bool ok = true;
        for (int ct = x.ct0; ct < x.ct1; ++ct) {
          if (!wait_c(&empty[stage], ph ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_tx(&full[stage], 2u * atoms * kAtomBytes);
          armed[stage] = static_cast<int>(ph);
          uint8_t* dst = sB + stage * 2 * op_bytes;
          for (int at = 0; at < atoms; ++at) {
            tma_load_2d(dst + at * kAtomBytes, &J.b_hi, at * 32, ct * kTgCols, &full[stage]);
            tma_load_2d(dst + op_bytes + at * kAtomBytes, &J.b_lo, at * 32, ct * kTgCols, &full[stage]);
          }
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (abort_flag) {      // copies in flight land before the CTA goes away
        for (int q = 0; q < S; ++q) drain_phase(&full[q], armed[q]);
        drain_phase(a_full, armed_a);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0, buf = 0, ucount = 0;
      uint32_t ph = 0, bph = 0;
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x, ++ucount) {
        const TgUnit x = tg_unit(b, u);
        const int ksteps = b.job[x.job].kp / 8;
        if (!wait_c(a_full, static_cast<uint32_t>(ucount) & 1u, &abort_flag)) break;
        tc_fence_after();
        const uint64_t ahi0 = kmajor_desc(smem_u32(sA));
        const uint64_t alo0 = kmajor_desc(smem_u32(sA + op_bytes));
        bool ok = true;
        for (int ct = x.ct0; ct < x.ct1; ++ct) {
          if (!wait_c(&full[stage], ph, &abort_flag) || !wait_c(&d_empty[buf], bph ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bhi0 = kmajor_desc(smem_u32(sB + stage * 2 * op_bytes));
          const uint64_t blo0 = kmajor_desc(smem_u32(sB + stage * 2 * op_bytes + op_bytes));
          const uint32_t dt = tmem + static_cast<uint32_t>(buf * kTgCols);
          for (int ks = 0; ks < ksteps; ++ks) {
            // 8 fp32 (32 bytes) per K step inside a 128-byte row; a new
            // 32-column atom every 4 steps (16-byte descriptor units)
            const uint64_t off = static_cast<uint64_t>((ks >> 2) * (kAtomBytes >> 4) + (ks & 3) * 2);
            tc_mma_tf32(dt, ahi0 + off, bhi0 + off, ks > 0 ? 1u : 0u);
            tc_mma_tf32(dt, ahi0 + off, blo0 + off, 1u);
            tc_mma_tf32(dt, alo0 + off, bhi0 + off, 1u);
          }
          tc_commit(&empty[stage]);
          tc_commit(&d_full[buf]);
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
          if (++buf == 2) {
            buf = 0;
            bph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(a_empty);
      }
      if (abort_flag) drain_mma(&drain_bar);   // products in flight complete first
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM lane = tile row
    const int e = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int buf = 0;
    uint32_t bph = 0;
    float v[16];
    for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x) {
      const TgUnit x = tg_unit(b, u);
      const TgJob& J = b.job[x.job];
      const int64_t i = x.i0 + e;
      const int64_t n = J.n;
      bool ok = true;
      for (int ct = x.ct0; ct < x.ct1; ++ct) {
        if (!wait_c(&d_full[buf], bph, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c0 = 0; c0 < kTgCols; c0 += 16) {
          tmem_ld16(tmem + lane_base + static_cast<uint32_t>(buf * kTgCols + c0), v);
          tmem_ld_wait();
          const int64_t j = static_cast<int64_t>(ct) * kTgCols + c0;
          if (i < J.d && j < n) {
            float* dst = J.T + i * n + j;
            if (j + 16 <= n && (n & 3) == 0) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            } else {
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (j + q < n) dst[q] = v[q];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&d_empty[buf]);
        if (++buf == 2) {
          buf = 0;
          bph ^= 1u;
        }
      }
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kTgCols)
                 : "memory");
  }
}

size_t tg_smem_bytes(int kp_max, int stages) {
  const size_t op = static_cast<size_t>(kp_max / 32) * kAtomBytes;
  return 1024 + 2 * op + static_cast<size_t>(stages) * 2 * op + (2 * stages + 6) * 8;
}

}  // namespace

// Ranks in (64, 128] run as two passes over the rank: T = A[:, :64] B[:64]
// written into T, A[:, 64:] B[64:] into a second buffer, then added. These
// copy a column block of A into a dense buffer and add the second product.
__global__ void copy_cols_kernel(const float* src, int64_t ld_src, int32_t col0, int32_t cols, int64_t d,
                                 float* dst) {
  const int64_t total = d * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / cols;
    dst[e] = __ldg(src + i * ld_src + col0 + (e - i * cols));
  }
}

__global__ void add_f32_kernel(float* t, const float* t2, int64_t count) {
  const int64_t quads = count >> 2;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < quads;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = reinterpret_cast<float4*>(t)[q];
    const float4 b = __ldg(reinterpret_cast<const float4*>(t2) + q);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    reinterpret_cast<float4*>(t)[q] = a;
  }
  if (blockIdx.x == 0 && threadIdx.x < (count & 3)) {
    const int64_t e = (quads << 2) + threadIdx.x;
    t[e] += t2[e];
  }
}

cudaError_t launch_copy_cols(const float* src, int64_t ld_src, int32_t col0, int32_t cols, int64_t d, float* dst,
                             cudaStream_t s) {
  const int64_t total = d * cols;
  if (total <= 0) return cudaSuccess;
  copy_cols_kernel<<<static_cast<unsigned>(min64((total + 255) / 256, 148 * 8)), 256, 0, s>>>(src, ld_src, col0,
                                                                                             cols, d, dst);
  return counted(cudaGetLastError());
}

// t and t2 16-byte aligned.
cudaError_t launch_add_f32(float* t, const float* t2, int64_t count, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  add_f32_kernel<<<static_cast<unsigned>(min64((count / 4 + 255) / 256 + 1, 148 * 16)), 256, 0, s>>>(t, t2, count);
  return counted(cudaGetLastError());
}

int64_t t_gemm_kp(int32_t r) { return r <= 32 ? 32 : 64; }

bool t_gemm_supported(int64_t d, int64_t n, int32_t r) {
  return r >= kTensorTMinRank && r <= kTensorTMaxRank && n % 4 == 0 && d <= (int64_t{1} << 31) &&
         n <= (int64_t{1} << 31) && tc::encode_fn() != nullptr;
}

cudaError_t launch_t_split(const TGemmJob* jobs, int count, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  {
    static thread_local SplitBatch sb;
    std::memset(&sb, 0, sizeof sb);
    int64_t blocks = 0;
    for (int k = 0; k < count; ++k) {
      const TGemmJob& j = jobs[k];
      SplitJob& t = sb.job[k];
      t.A = j.A;
      t.B = j.B;
      t.a_hi = j.a_hi;
      t.a_lo = j.a_lo;
      t.b_hi = j.b_hi;
      t.b_lo = j.b_lo;
      t.d = j.d;
      t.n = j.n;
      t.r = j.r;
      t.kp = j.kp;
      t.block_begin = blocks;
      blocks += ((j.d + j.n) * j.kp + kSplitPerBlock - 1) / kSplitPerBlock;
    }
    sb.count = count;
    sb.total_blocks = blocks;
    t_split_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(sb);
    cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_t_gemm(const TGemmJob* jobs, int count, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  // 1. split the operands (one launch for the whole batch)
  {
    cudaError_t e = launch_t_split(jobs, count, s);
    if (e != cudaSuccess) return e;
  }
  // 2. the products, up to kMaxTgJobs layers per launch
  static thread_local TgBatch b;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  for (int k0 = 0; k0 < count; k0 += kMaxTgJobs) {
    const int m = count - k0 < kMaxTgJobs ? count - k0 : kMaxTgJobs;
    std::memset(&b, 0, sizeof b);
    int kp_max = 32;
    for (int k = 0; k < m; ++k) kp_max = jobs[k0 + k].kp > kp_max ? jobs[k0 + k].kp : kp_max;
    b.tiles_per_unit = 32;
    int64_t units = 0;
    for (int k = 0; k < m; ++k) {
      const TGemmJob& j = jobs[k0 + k];
      TgJob& t = b.job[k];
      const bool ok = tc::encode_2d(&t.a_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.a_hi, j.d, j.kp, 32, kTgRows) &&
                      tc::encode_2d(&t.a_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.a_lo, j.d, j.kp, 32, kTgRows) &&
                      tc::encode_2d(&t.b_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.b_hi, j.n, j.kp, 32, kTgCols) &&
                      tc::encode_2d(&t.b_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.b_lo, j.n, j.kp, 32, kTgCols);
      if (!ok) return cudaErrorInvalidValue;
      t.T = j.T;
      t.d = j.d;
      t.n = j.n;
      t.kp = j.kp;
      t.col_tiles = static_cast<int32_t>((j.n + kTgCols - 1) / kTgCols);
      t.chunks = (t.col_tiles + b.tiles_per_unit - 1) / b.tiles_per_unit;
      t.unit_begin = units;
      units += ((j.d + kTgRows - 1) / kTgRows) * t.chunks;
    }
    b.count = m;
    b.kp_max = kp_max;
    int stages = 6;
    while (stages > 2 && tg_smem_bytes(kp_max, stages) > 232448) --stages;
    b.stages = stages;
    b.total_units = units;
    const size_t smem = tg_smem_bytes(kp_max, stages);
    cudaError_t e = cudaFuncSetAttribute(t_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t grid = units < sms ? units : sms;
    t_gemm_kernel<<<static_cast<unsigned>(grid), kTgThreads, smem, s>>>(b);
    e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

unsigned int t_gemm_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_tg_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
