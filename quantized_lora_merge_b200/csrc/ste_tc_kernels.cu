// STE backward of IntLoRA on the 5th-generation tensor cores (sm_100a):
// dA = G B^T and dB = A^T G [IntLoRA paper notes (ICML2025), method section 2:
// the straight-through estimator passes the gradient of W' to A B unchanged].
//
// One pass over G feeds both products. A CTA works on units of 128 rows of G
// times a run of 128-column tiles. Per tile, TMA brings the G tile (two
// 64-column boxes, 128-byte swizzle) and the matching 128 columns of B into a
// pipeline stage; one thread issues
//   GEMM1  D1[128 rows x RP]  += G_tile (K-major)  * B_tile^T   (K = columns)
//   GEMM2  D2[128 cols x RP]   = G_tile^T (MN-major, same bytes) * A_blk^T (K = rows)
// with tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in TMEM). D2 holds the
// unit's contribution to dB^T for that tile and is drained by four epilogue
// warps (tcgen05.ld, then fp32 reductions into dB); D1 accumulates over the
// unit's tiles and is drained into dA at the end of the unit. Two warps stage
// the unit's 128 rows of A, transposed into the K-major operand layout. Roles
// meet on mbarriers; every wait is bounded and a timeout is counted in a
// device word and makes the CTA stop, release its tensor memory and return.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

using namespace tc;

constexpr int kTcThreads = 256;
constexpr int kTileRows = 128;                 // rows of G per unit (GEMM1 M, GEMM2 K)
constexpr int kTileCols = 128;                 // columns of G per tile (GEMM1 K, GEMM2 M)
constexpr uint32_t kGBytes = kTileRows * kTileCols * 2;
constexpr uint32_t kBoxBytes = kTileRows * 64 * 2;    // one 64-column box of the G tile
constexpr int kMaxTcJobs = 64;
constexpr int kMaxD2 = 8;                      // D2 accumulators (tile epilogues in flight)
constexpr int kMaxStages = 4;                  // pipeline stages at most (host picks 2-4)

struct alignas(64) SteTcJob {
  CUtensorMap g_map;          // G: dims {n, d}, box {64, 128}, 128B swizzle
  CUtensorMap b_map;          // B: dims {n, r}, box {64, RP}, 128B swizzle
  const uint16_t* A;          // d x r bf16
  float* dA;
  float* dB;
  int64_t d, n;
  int32_t r;
  int32_t col_tiles;
  int32_t chunks;             // units per row block
  int32_t pad;
  int64_t unit_begin;
};
struct SteTcBatch {
  SteTcJob job[kMaxTcJobs];
  int32_t count;
  int32_t rp;                 // r rounded up to a multiple of 16 (MMA N)
  int32_t tiles_per_unit;
  int32_t stages;
  int32_t nd2;
  int32_t ctas_per_sm;
  int64_t total_units;
  uint32_t tmem_cols;
  unsigned int* timeouts;
};

__device__ unsigned int g_tc_timeouts;

// Bounded mbarrier wait counted in this kernel family's timeout word.
__device__ __forceinline__ bool mbar_wait_c(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait(bar, parity, abort_flag, &g_tc_timeouts);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M = 128, N = rp.
__host__ __device__ constexpr uint32_t instr_desc(int rp, bool a_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major ? (1u << 15) : 0u) |
         (static_cast<uint32_t>(rp >> 3) << 17) | (static_cast<uint32_t>(kTileRows >> 4) << 24);
}

// Byte offset of element (row k, column i) in a K-major, 128-byte-swizzled
// operand of `rows` rows and 128 K-columns (two 64-column atoms).
__device__ __forceinline__ uint32_t kmajor_offset(int k, int i, int rows) {
  const int atom = i >> 6, ii = i & 63;
  return static_cast<uint32_t>(atom * rows * 128 + (k >> 3) * 1024 + (k & 7) * 128 +
                               ((((ii >> 3) ^ (k & 7)) & 7) << 4) + (ii & 7) * 2);
}

struct Unit {
  int job;
  int64_t i0;
  int ct0, ct1;
};
__device__ __forceinline__ Unit decode_unit(const SteTcBatch& b, int64_t u) {
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].unit_begin <= u) ++j;
  const SteTcJob& J = b.job[j];
  const int64_t local = u - J.unit_begin;
  const int64_t rb = local / J.chunks;
  const int cc = static_cast<int>(local - rb * J.chunks);
  Unit x;
  x.job = j;
  x.i0 = rb * kTileRows;
  x.ct0 = cc * b.tiles_per_unit;
  x.ct1 = min(J.col_tiles, x.ct0 + b.tiles_per_unit);
  return x;
}

__global__ void __launch_bounds__(kTcThreads, 2) ste_tc_kernel(const __grid_constant__ SteTcBatch b) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ __align__(8) uint64_t drain_bar;
  // operands want 1024-byte alignment (the 128-byte swizzle repeats every 8 rows)
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const int RP = b.rp, S = b.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(RP) * 256;     // RP rows x 128 columns bf16
  uint8_t* sG = base;
  uint8_t* sB = sG + S * kGBytes;
  uint8_t* sA = sB + S * b_bytes;                              // [2] A blocks (K-major, RP rows)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sA + 2 * b_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  const int ND2 = b.nd2;                                       // D2 accumulators in the ring
  uint64_t* d2_full = bars + 2 * S;
  uint64_t* d2_empty = d2_full + kMaxD2;
  uint64_t* d1_full = d2_empty + kMaxD2;
  uint64_t* d1_empty = d1_full + 2;
  uint64_t* a_full = d1_full + 4;
  uint64_t* a_empty = d1_full + 6;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < ND2; ++q) {
      mbar_init(&d2_full[q], 1);
      mbar_init(&d2_empty[q], 128);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&d1_full[q], 1);
      mbar_init(&d1_empty[q], 128);
      mbar_init(&a_full[q], 64);
      mbar_init(&a_empty[q], 1);
    }
    abort_flag = 0;
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(b.tmem_cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // TMEM columns: D1[2] at 0 and RP, D2[q] at (2 + q) RP
  const uint32_t idesc1 = instr_desc(RP, false);
  const uint32_t idesc2 = instr_desc(RP, true);

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int armed[kMaxStages];
      for (int q = 0; q < kMaxStages; ++q) armed[q] = -1;
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x) {
        const Unit x = decode_unit(b, u);
        const SteTcJob& J = b.job[x.job];
        for (int ct = x.ct0; ct < x.ct1; ++ct) {
          if (!mbar_wait_c(&empty[stage], ph ^ 1u, &abort_flag)) break;
          mbar_arrive_tx(&full[stage], kGBytes + b_bytes);
          armed[stage] = static_cast<int>(ph);
          uint8_t* g = sG + stage * kGBytes;
          uint8_t* bt = sB + stage * b_bytes;
          const int32_t x0 = ct * kTileCols;
          const int32_t y0 = static_cast<int32_t>(x.i0);
          tma_load_2d(g, &J.g_map, x0, y0, &full[stage]);
          tma_load_2d(g + kBoxBytes, &J.g_map, x0 + 64, y0, &full[stage]);
          tma_load_2d(bt, &J.b_map, x0, 0, &full[stage]);
          tma_load_2d(bt + RP * 128, &J.b_map, x0 + 64, 0, &full[stage]);
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (abort_flag)        // copies in flight land before the CTA goes away
        for (int q = 0; q < S; ++q) drain_phase(&full[q], armed[q]);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0, d2 = 0, ucount = 0;
      uint32_t ph = 0, d2ph = 0;
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x, ++ucount) {
        const Unit x = decode_unit(b, u);
        const int ab = ucount & 1;
        const uint32_t aph = static_cast<uint32_t>(ucount >> 1) & 1u;
        if (!mbar_wait_c(&a_full[ab], aph, &abort_flag)) break;
        if (!mbar_wait_c(&d1_empty[ab], aph ^ 1u, &abort_flag)) break;
        tc_fence_after();
        const uint32_t d1 = tmem + static_cast<uint32_t>(ab * RP);
        const uint64_t a0 = smem_desc(smem_u32(sA + ab * b_bytes), 16, 1024);
        bool ok = true;
        for (int ct = x.ct0; ct < x.ct1; ++ct) {
          if (!mbar_wait_c(&full[stage], ph, &abort_flag) || !mbar_wait_c(&d2_empty[d2], d2ph ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of this stage; the K steps only move the start address
          // (16-byte units): 32 bytes per K step inside a 128-byte row, one
          // 64-column atom further every 4 steps; 16 rows per GEMM2 step
          const uint64_t gk0 = smem_desc(smem_u32(sG + stage * kGBytes), 16, 1024);
          const uint64_t gm0 = smem_desc(smem_u32(sG + stage * kGBytes), kBoxBytes, 1024);
          const uint64_t bt0 = smem_desc(smem_u32(sB + stage * b_bytes), 16, 1024);
          const uint32_t d2t = tmem + static_cast<uint32_t>((2 + d2) * RP);
          const uint32_t acc1 = ct > x.ct0 ? 1u : 0u;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // GEMM1: K = 16 columns of the tile; both operands K-major
            const uint64_t koff = static_cast<uint64_t>((ks & 3) * 2);
            tc_mma(d1, gk0 + static_cast<uint64_t>((ks >> 2) * (kBoxBytes >> 4)) + koff,
                   bt0 + static_cast<uint64_t>((ks >> 2) * (RP * 8)) + koff, idesc1,
                   (acc1 | static_cast<uint32_t>(ks)) != 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // GEMM2: K = 16 rows of the tile; A = G tile MN-major (64-column
            // atoms kBoxBytes apart, 8-row groups 1024 bytes apart), B = A block
            tc_mma(d2t, gm0 + static_cast<uint64_t>(ks * 128),
                   a0 + static_cast<uint64_t>((ks >> 2) * (RP * 8) + (ks & 3) * 2), idesc2, ks > 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          tc_commit(&d2_full[d2]);
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
          if (++d2 == ND2) {
            d2 = 0;
            d2ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&d1_full[ab]);
        tc_commit(&a_empty[ab]);
      }
      if (abort_flag) drain_mma(&drain_bar);   // products in flight complete first
    }
  } else if (warp < 4) {
    // ---------------- A-block staging (64 threads, two rows each)
    const int t = threadIdx.x - 64;
    int ucount = 0;
    for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x, ++ucount) {
      const Unit x = decode_unit(b, u);
      const SteTcJob& J = b.job[x.job];
      const int ab = ucount & 1;
      const uint32_t aph = static_cast<uint32_t>(ucount >> 1) & 1u;
      if (!mbar_wait_c(&a_empty[ab], aph ^ 1u, &abort_flag)) break;
      uint8_t* dst = sA + ab * b_bytes;
      for (int rr = t; rr < kTileRows; rr += 64) {
        const int64_t i = x.i0 + rr;
        for (int k = 0; k < RP; ++k) {
          uint16_t v = 0;
          if (i < J.d && k < J.r) v = __ldg(J.A + i * J.r + k);
          *reinterpret_cast<uint16_t*>(dst + kmajor_offset(k, rr, RP)) = v;
        }
      }
      // generic-proxy writes must be visible to the tensor core's async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&a_full[ab]);
    }
  } else {
    // ---------------- epilogue (TMEM lanes 32 (warp % 4) ..)
    const int e = threadIdx.x - 128;              // TMEM lane = tile row / tile column
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int d2 = 0, ucount = 0;
    uint32_t d2ph = 0;
    float v[16];
    for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x, ++ucount) {
      const Unit x = decode_unit(b, u);
      const SteTcJob& J = b.job[x.job];
      const int r = J.r;
      const int64_t n = J.n;
      bool ok = true;
      for (int ct = x.ct0; ct < x.ct1; ++ct) {
        if (!mbar_wait_c(&d2_full[d2], d2ph, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int64_t j = static_cast<int64_t>(ct) * kTileCols + e;
        for (int c0 = 0; c0 < RP; c0 += 16) {
          tmem_ld16(tmem + lane_base + static_cast<uint32_t>((2 + d2) * RP + c0), v);
          tmem_ld_wait();
          if (j < n) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              if (c0 + k < r) red_add(J.dB + static_cast<int64_t>(c0 + k) * n + j, v[k]);
          }
        }
        tc_fence_before();
        mbar_arrive(&d2_empty[d2]);
        if (++d2 == ND2) {
          d2 = 0;
          d2ph ^= 1u;
        }
      }
      if (!ok) break;
      const int ab = ucount & 1;
      if (!mbar_wait_c(&d1_full[ab], static_cast<uint32_t>(ucount >> 1) & 1u, &abort_flag)) break;
      tc_fence_after();
      const int64_t i = x.i0 + e;
      for (int c0 = 0; c0 < RP; c0 += 16) {
        tmem_ld16(tmem + lane_base + static_cast<uint32_t>(ab * RP + c0), v);
        tmem_ld_wait();
        if (i < J.d) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (c0 + k < r) red_add(J.dA + i * r + c0 + k, v[k]);
        }
      }
      tc_fence_before();
      mbar_arrive(&d1_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(b.tmem_cols)
                 : "memory");
  }
}

// ---- host side ---------------------------------------------------------------
bool encode_bf16(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
  return tc::encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, rows, cols, 64, box_rows);
}

size_t tc_smem_bytes(int rp, int stages) {
  const size_t b_bytes = static_cast<size_t>(rp) * 256;
  return 1024 + stages * (kGBytes + b_bytes) + 2 * b_bytes + (2 * stages + 2 * kMaxD2 + 8) * 8;
}

}  // namespace

bool ste_tc_supported(const SteJob& j) {
  const auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return j.n % 8 == 0 && j.r >= 1 && j.r <= kSteTcMaxRank && al(j.G) && al(j.B) && j.d <= (int64_t{1} << 31) &&
         j.n <= (int64_t{1} << 31) && tc::encode_fn() != nullptr;
}

cudaError_t launch_ste_tc(const SteJob* jobs, int count, cudaStream_t s) {
  static thread_local SteTcBatch b;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  for (int base = 0; base < count; base += kMaxTcJobs) {
    const int m = count - base < kMaxTcJobs ? count - base : kMaxTcJobs;
    std::memset(&b, 0, sizeof b);
    int max_r = 1;
    for (int k = 0; k < m; ++k) max_r = jobs[base + k].r > max_r ? jobs[base + k].r : max_r;
    const int rp = (max_r + 15) / 16 * 16;
    // 128 x 2048 of G (512 KB) per unit at most: units many enough to balance,
    // D1 epilogues rare
    b.tiles_per_unit = 16;
    int64_t units = 0;
    for (int k = 0; k < m; ++k) {
      const SteJob& j = jobs[base + k];
      SteTcJob& t = b.job[k];
      if (!encode_bf16(&t.g_map, j.G, j.d, j.n, kTileRows) || !encode_bf16(&t.b_map, j.B, j.r, j.n, rp))
        return cudaErrorInvalidValue;
      t.A = j.A;
      t.dA = j.dA;
      t.dB = j.dB;
      t.d = j.d;
      t.n = j.n;
      t.r = j.r;
      t.col_tiles = static_cast<int32_t>((j.n + kTileCols - 1) / kTileCols);
      t.chunks = (t.col_tiles + b.tiles_per_unit - 1) / b.tiles_per_unit;
      t.unit_begin = units;
      units += ((j.d + kTileRows - 1) / kTileRows) * t.chunks;
    }
    b.count = m;
    b.rp = rp;
    // two CTAs per SM when their tensor memory fits (two independent
    // load -> MMA -> epilogue chains per SM), else one with deeper buffers
    const int per_sm = 6 * rp <= 256 ? 2 : 1;
    const uint32_t col_budget = 512 / per_sm;
    int nd2 = static_cast<int>(col_budget / rp) - 2;
    nd2 = nd2 > kMaxD2 ? kMaxD2 : nd2;
    int stages = per_sm == 2 ? 3 : 4;
    const size_t smem_cap = (233472 / per_sm) - 1024;
    while (stages > 2 && tc_smem_bytes(rp, stages) > smem_cap) --stages;
    b.stages = stages;
    b.nd2 = nd2;
    b.ctas_per_sm = per_sm;
    b.total_units = units;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>((2 + nd2) * rp)) cols <<= 1;
    b.tmem_cols = cols;
    const size_t smem = tc_smem_bytes(rp, stages);
    cudaError_t e = cudaFuncSetAttribute(ste_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t grid = units < int64_t{per_sm} * sms ? units : int64_t{per_sm} * sms;
    ste_tc_kernel<<<static_cast<unsigned>(grid), kTcThreads, smem, s>>>(b);
    e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

unsigned int ste_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_tc_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
