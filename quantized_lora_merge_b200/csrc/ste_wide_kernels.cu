// STE backward for the larger ranks (r >= 64) on the 5th-generation tensor
// cores [IntLoRA paper notes (ICML2025), method section 2: the STE passes the
// gradient of W' to A B unchanged, so dA = G B^T and dB = A^T G].
//
// The one-pass kernel (ste_tc_kernels.cu) reduces every tile's 128 x r block
// of dB^T into global memory with fp32 reductions: at r >= 64 that is one
// reduction per 2 elements of G or more, and the reductions, not HBM, set its
// pace. Here the two products take separate passes, each accumulating over
// many tiles inside one CTA before it reduces into the (zeroed) outputs. A
// layer is cut into regions of up to 16 row blocks x 16 column tiles (8 MB of
// G); a region's units are
//   pass 1  one per row block: D1 += G_tile B_tile^T over the region's
//           column tiles (both operands K-major), then D1 -> dA rows (+=);
//   pass 2  one per column tile: D2 += G_tile^T A_tile over the region's
//           row blocks (G tile MN-major, the A tile loaded by TMA straight
//           from the row-major A as an MN-major operand), then D2 -> dB (+=).
// Units are numbered region by region and the persistent CTAs walk them in
// that order, so both passes over a region run close together in time and
// the second read of its G tiles is served by L2: HBM sees G about once.
// Every unit is at most 16 tile steps (balanced across the CTAs), and the
// reductions add 128 r fp32 per unit against 16 tiles of G (an eighth of
// G's bytes at r = 128).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>

#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

using namespace tc;

constexpr int kWThreads = 256;
constexpr int kWRows = 128;                       // G tile rows (pass 1 M, pass 2 K)
constexpr int kWCols = 128;                       // G tile columns (pass 1 K, pass 2 M)
constexpr uint32_t kWGBytes = kWRows * kWCols * 2;
constexpr uint32_t kWBox = kWRows * 64 * 2;       // one 64-column box (16 KB)
constexpr int kMaxWJobs = 40;

__device__ unsigned int g_sw_timeouts;

__device__ __forceinline__ bool wait_w(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait(bar, parity, abort_flag, &g_sw_timeouts);
}

constexpr int kRegionBlocks = 16;                // row blocks per region
constexpr int kRegionTiles = 16;                 // column tiles per region

struct alignas(64) WJob {
  CUtensorMap g_map;          // G: dims {n, d}, box {64, 128}
  CUtensorMap b_map;          // B: dims {n, r}, box {64, RP}
  CUtensorMap a_map;          // A: dims {r, d}, box {64, 128}
  float* dA;                  // zeroed before the launch
  float* dB;                  // zeroed before the launch
  int64_t d, n;
  int32_t r;
  int32_t row_blocks;
  int32_t col_tiles;
  int32_t bands;              // region rows: ceil(row_blocks / kRegionBlocks)
  int32_t chunks;             // region columns: ceil(col_tiles / kRegionTiles)
  int32_t pad;
  int64_t band_units;         // units of a full band: chunks kRegionBlocks + col_tiles
  int64_t unit_begin;         // first unit of this job
};
struct WBatch {
  WJob job[kMaxWJobs];
  int32_t count;
  int32_t rp;                 // r rounded up to 64 (MMA N)
  int32_t stages;
  int32_t pad;
  int64_t total_units;
};

struct WUnit {
  int job;
  int pass;                   // 1 or 2
  int64_t fixed;              // pass 1: row block; pass 2: column tile
  int64_t start;              // pass 1: first column tile; pass 2: first row block
  int steps;                  // pass 1: column tiles; pass 2: row blocks
};
__device__ __forceinline__ int64_t wmin(int64_t a, int64_t b) { return a < b ? a : b; }
// Unit u: its job, band (region row), chunk (region column), then the
// region's pass-1 units (one per row block) followed by its pass-2 units
// (one per column tile).
__device__ __forceinline__ WUnit w_unit(const WBatch& b, int64_t u) {
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].unit_begin <= u) ++j;
  const WJob& J = b.job[j];
  int64_t local = u - J.unit_begin;
  const int64_t bi = wmin(local / J.band_units, J.bands - 1);
  local -= bi * J.band_units;
  const int64_t rcount = wmin(kRegionBlocks, J.row_blocks - bi * kRegionBlocks);
  const int64_t ci = wmin(local / (rcount + kRegionTiles), J.chunks - 1);
  local -= ci * (rcount + kRegionTiles);
  const int64_t tcount = wmin(kRegionTiles, J.col_tiles - ci * kRegionTiles);
  WUnit x;
  x.job = j;
  if (local < rcount) {
    x.pass = 1;
    x.fixed = bi * kRegionBlocks + local;
    x.start = ci * kRegionTiles;
    x.steps = static_cast<int>(tcount);
  } else {
    x.pass = 2;
    x.fixed = ci * kRegionTiles + (local - rcount);
    x.start = bi * kRegionBlocks;
    x.steps = static_cast<int>(rcount);
  }
  return x;
}

// kind::f16 (bf16 in, fp32 D), M = 128, N = rp; operand majors per pass.
__device__ __forceinline__ uint32_t w_idesc(int rp, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(rp >> 3) << 17) | (static_cast<uint32_t>(kWRows >> 4) << 24);
}

__global__ void __launch_bounds__(kWThreads, 1) ste_wide_kernel(const __grid_constant__ WBatch b) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ __align__(8) uint64_t drain_bar;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const int RP = b.rp, S = b.stages;
  // a stage: the G tile, then the pass's second operand (B tile: RP rows x
  // 128 columns; A tile: RP / 64 boxes of 128 rows x 64 columns) -- both
  // RP x 256 bytes
  const uint32_t op_bytes = static_cast<uint32_t>(RP) * 256;
  const uint32_t stage_bytes = kWGBytes + op_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* d_full = bars + 2 * S;        // [2]
  uint64_t* d_empty = d_full + 2;         // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&d_full[q], 1);
      mbar_init(&d_empty[q], 128);
    }
    abort_flag = 0;
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const uint32_t tmem_cols = static_cast<uint32_t>(2 * RP);   // 128 or 256 (power of two)
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(tmem_cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;                // D[q] at column q * RP

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int armed[4] = {-1, -1, -1, -1};      // parity last armed per stage (host picks 2-4 stages)
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x) {
        const WUnit x = w_unit(b, u);
        const WJob& J = b.job[x.job];
        bool ok = true;
        for (int st = 0; st < x.steps; ++st) {
          if (!wait_w(&empty[stage], ph ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          const int32_t rb = static_cast<int32_t>(x.pass == 1 ? x.fixed : x.start + st);
          const int32_t ct = static_cast<int32_t>(x.pass == 1 ? x.start + st : x.fixed);
          mbar_arrive_tx(&full[stage], stage_bytes);
          armed[stage] = static_cast<int>(ph);
          uint8_t* g = base + stage * stage_bytes;
          tma_load_2d(g, &J.g_map, ct * kWCols, rb * kWRows, &full[stage]);
          tma_load_2d(g + kWBox, &J.g_map, ct * kWCols + 64, rb * kWRows, &full[stage]);
          uint8_t* o = g + kWGBytes;
          if (x.pass == 1) {
            // B columns of the tile: RP rows x 128 columns (two 64-column boxes)
            tma_load_2d(o, &J.b_map, ct * kWCols, 0, &full[stage]);
            tma_load_2d(o + RP * 128, &J.b_map, ct * kWCols + 64, 0, &full[stage]);
          } else {
            // A rows of the block: 128 rows x RP ranks (RP / 64 boxes)
            for (int at = 0; at < RP / 64; ++at)
              tma_load_2d(o + at * kWBox, &J.a_map, at * 64, rb * kWRows, &full[stage]);
          }
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (abort_flag)        // copies in flight land before the CTA goes away
        for (int q = 0; q < S; ++q) drain_phase(&full[q], armed[q]);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = w_idesc(RP, false, false);
      const uint32_t idesc2 = w_idesc(RP, true, true);
      int stage = 0, buf = 0;
      uint32_t ph = 0, bph = 0;
      for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x) {
        const WUnit x = w_unit(b, u);
        if (!wait_w(&d_empty[buf], bph ^ 1u, &abort_flag)) break;
        tc_fence_after();
        const uint32_t dt = tmem + static_cast<uint32_t>(buf * RP);
        bool ok = true;
        for (int st = 0; st < x.steps; ++st) {
          if (!wait_w(&full[stage], ph, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t g = smem_u32(base + stage * stage_bytes);
          const uint32_t o = g + kWGBytes;
          if (x.pass == 1) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              // K = 16 columns; G tile and B tile K-major (32 bytes per step,
              // a new 64-column atom every 4 steps)
              const uint32_t koff = (ks & 3) * 32u;
              tc_mma(dt, kmajor_desc(g + (ks >> 2) * kWBox + koff),
                     kmajor_desc(o + (ks >> 2) * (RP * 128) + koff), idesc1, (st > 0 || ks > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              // K = 16 rows; both operands MN-major: 64-element atoms 16 KB
              // apart (leading byte offset), 8-row groups 1 KB apart (stride)
              tc_mma(dt, smem_desc(g + ks * 2048, kWBox, 1024), smem_desc(o + ks * 2048, kWBox, 1024), idesc2,
                     (st > 0 || ks > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&d_full[buf]);
        if (++buf == 2) {
          buf = 0;
          bph ^= 1u;
        }
      }
      if (abort_flag) drain_mma(&drain_bar);   // products in flight complete first
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: TMEM lane = row of dA (pass 1) / column of dB (pass 2)
    const int e = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int buf = 0;
    uint32_t bph = 0;
    float v[16];
    for (int64_t u = blockIdx.x; u < b.total_units && !abort_flag; u += gridDim.x) {
      const WUnit x = w_unit(b, u);
      const WJob& J = b.job[x.job];
      const int r = J.r;
      if (!wait_w(&d_full[buf], bph, &abort_flag)) break;
      tc_fence_after();
      const int64_t idx = x.fixed * 128 + e;            // row (pass 1) or column (pass 2)
      for (int c0 = 0; c0 < RP; c0 += 16) {
        tmem_ld16(tmem + lane_base + static_cast<uint32_t>(buf * RP + c0), v);
        tmem_ld_wait();
        if (x.pass == 1) {
          if (idx < J.d) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              if (c0 + k < r) red_add(J.dA + idx * r + c0 + k, v[k]);
          }
        } else if (idx < J.n) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (c0 + k < r) red_add(J.dB + static_cast<int64_t>(c0 + k) * J.n + idx, v[k]);
        }
      }
      tc_fence_before();
      mbar_arrive(&d_empty[buf]);
      if (++buf == 2) {
        buf = 0;
        bph ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols) : "memory");
  }
}

size_t w_smem_bytes(int rp, int stages) {
  return 1024 + static_cast<size_t>(stages) * (kWGBytes + static_cast<size_t>(rp) * 256) + (2 * stages + 4) * 8;
}

}  // namespace

bool ste_wide_supported(const SteJob& j) {
  const auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return j.r >= kSteWideMinRank && j.r <= kSteTcMaxRank && j.r % 8 == 0 && j.n % 8 == 0 && al(j.G) &&
         al(j.A) && al(j.B) && j.d <= (int64_t{1} << 31) && j.n <= (int64_t{1} << 31) &&
         tc::encode_fn() != nullptr;
}

cudaError_t launch_ste_wide(const SteJob* jobs, int count, cudaStream_t s) {
  static thread_local WBatch b;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  for (int k0 = 0; k0 < count; k0 += kMaxWJobs) {
    const int m = count - k0 < kMaxWJobs ? count - k0 : kMaxWJobs;
    std::memset(&b, 0, sizeof b);
    int max_r = 64;
    for (int k = 0; k < m; ++k) max_r = jobs[k0 + k].r > max_r ? jobs[k0 + k].r : max_r;
    const int rp = (max_r + 63) / 64 * 64;
    int64_t units = 0;
    for (int k = 0; k < m; ++k) {
      const SteJob& j = jobs[k0 + k];
      WJob& t = b.job[k];
      const bool ok =
          tc::encode_2d(&t.g_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, j.G, j.d, j.n, 64, kWRows) &&
          tc::encode_2d(&t.b_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, j.B, j.r, j.n, 64, rp) &&
          tc::encode_2d(&t.a_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, j.A, j.d, j.r, 64, kWRows);
      if (!ok) return cudaErrorInvalidValue;
      t.dA = j.dA;
      t.dB = j.dB;
      t.d = j.d;
      t.n = j.n;
      t.r = j.r;
      t.row_blocks = static_cast<int32_t>((j.d + kWRows - 1) / kWRows);
      t.col_tiles = static_cast<int32_t>((j.n + kWCols - 1) / kWCols);
      t.bands = (t.row_blocks + kRegionBlocks - 1) / kRegionBlocks;
      t.chunks = (t.col_tiles + kRegionTiles - 1) / kRegionTiles;
      t.band_units = static_cast<int64_t>(t.chunks) * kRegionBlocks + t.col_tiles;
      t.unit_begin = units;
      // every band but the last is full; a band's units are its chunks' row
      // blocks plus all the column tiles
      const int64_t last_rows = t.row_blocks - static_cast<int64_t>(t.bands - 1) * kRegionBlocks;
      units += static_cast<int64_t>(t.bands - 1) * t.band_units + t.chunks * last_rows + t.col_tiles;
    }
    b.count = m;
    b.rp = rp;
    b.total_units = units;
    const int64_t u2 = units;
    int stages = 4;
    while (stages > 2 && w_smem_bytes(rp, stages) > 232448) --stages;
    b.stages = stages;
    const size_t smem = w_smem_bytes(rp, stages);
    cudaError_t e = cudaFuncSetAttribute(ste_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t grid = u2 < sms ? u2 : sms;
    ste_wide_kernel<<<static_cast<unsigned>(grid), kWThreads, smem, s>>>(b);
    e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

unsigned int ste_wide_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_sw_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
