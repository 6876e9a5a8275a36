// Integer inference on merged IntLoRA weights: Y = X W'^T with W' = s_bar Q
// [IntLoRA paper notes (ICML2025), section 两种实现版本: the merged weight of
// IntLoRA_MUL is s_bar (U_round - z_bar) (.) (W_round - z) and that of
// IntLoRA_SHIFT is s_bar sign(V) (.) ((W_round - z) >> shift), i.e. an
// integer matrix Q times a per-row scale; the efficiency table runs the merged
// model as W8A8 / W4A8 with no post-training quantization].
//
//   Y[t][i] = x_scale[t] * w_scale[i] * sum_j X[t][j] Q[i][j]
//
// X is int8 (tokens x n). Q is held as P base-128 digit planes of int8
// (P = 1 when |Q| <= 127, the SHIFT merge of 4-bit codes; 2 for the MUL
// merge of 4-bit codes, |P| <= 225; 3 for 8-bit codes), packed channel-major
// [d][P][n] so that one TMA box of P C rows holds all planes of C channels.
//
// The GEMM runs on the 5th-generation tensor cores: tcgen05.mma.kind::i8
// (signed x signed, s32 accumulate in TMEM), M = 128 tokens, N = P C <= 256
// digit rows, K = 32 bytes per instruction, 128-byte K slices per pipeline
// stage staged by TMA with the 128-byte swizzle. A persistent CTA per SM:
// warp 0 issues the TMA loads, warp 1 the MMAs, warps 4-11 drain the
// double-buffered accumulator (tcgen05.ld; two warps per 32-lane TMEM
// quarter, each taking half of the tile's channels), add the planes exactly
// in 64-bit integers, scale in fp32 and hand each 32-row x 16-channel block
// of Y to a TMA store through a double-buffered shared-memory stage (64-byte
// swizzle, so the row-per-lane writes are free of bank conflicts and the
// global writes are whole lines instead of 32 scattered rows). The integer part is exact; the only roundings
// are the int -> fp32 conversion, the scale product and the final multiply.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cuda_bf16.h>

#include <cstdint>
#include <cstring>

#include "intlora_device.cuh"
#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

using namespace tc;

constexpr int kIgThreads = 384;
constexpr int kIgEpiThreads = 256;            // warps 4-11
constexpr int kIgRows = 128;                    // tokens per tile (M, TMEM lanes)
constexpr int kIgMaxN = 256;                    // digit rows per tile (N)
constexpr int kIgK = 128;                       // K bytes per stage (one swizzle row)
constexpr uint32_t kIgABytes = kIgRows * kIgK;  // 16 KB
constexpr int kMaxIgJobs = 48;
constexpr int kIgMaxStages = 8;                 // pipeline stages at most (host picks 2-8)
constexpr uint32_t kIgYBox = 32 * 16 * 4;        // one Y block: 32 rows x 16 fp32
constexpr uint32_t kIgYStage = 8 * 2 * kIgYBox;  // 8 epilogue warps x 2 buffers

__device__ unsigned int g_ig_timeouts;

__device__ __forceinline__ bool wait_ig(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait(bar, parity, abort_flag, &g_ig_timeouts);
}

struct alignas(64) IgJob {
  CUtensorMap x_map;          // {n, tokens} int8, box {128, 128}
  CUtensorMap w_map;          // {n, d P} int8, box {128, C P}
  CUtensorMap y_map;          // {d, tokens} fp32 box {16, 32} 64-byte swizzle, or bf16 box
                              // {16, 32} 32-byte swizzle (when y_tma)
  const float* x_scale;
  const float* w_scale;
  void* Y;                    // fp32, or bf16 when y_bf16
  int64_t tokens, d, n;
  int32_t m_tiles, n_tiles, k_stages, y_tma;
  int32_t y_bf16, pad;
  int64_t tile_begin;
};
struct IgBatch {
  IgJob job[kMaxIgJobs];
  int32_t count;
  int32_t planes;             // P
  int32_t chans;              // C: channels per tile
  int32_t stages;
  int64_t total_tiles;
};

struct IgTile {
  int job;
  int64_t t0, i0;
};
__device__ __forceinline__ IgTile ig_tile(const IgBatch& b, int64_t u) {
  int j = 0;
  while (j + 1 < b.count && b.job[j + 1].tile_begin <= u) ++j;
  const IgJob& J = b.job[j];
  const int64_t local = u - J.tile_begin;
  const int64_t nt = local / J.m_tiles;
  IgTile x;
  x.job = j;
  x.t0 = (local - nt * J.m_tiles) * kIgRows;
  x.i0 = nt * b.chans;
  return x;
}

__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::i8: D s32, A and B signed 8-bit, both K-major, M = 128, N = nrows.
__device__ __forceinline__ uint32_t ig_idesc(int nrows) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nrows >> 3) << 17) |
         (static_cast<uint32_t>(kIgRows >> 4) << 24);
}
// kind::f16: D f32, A and B bf16, both K-major, M = 128, N = nrows.
__device__ __forceinline__ uint32_t ig_idesc_bf16(int nrows) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nrows >> 3) << 17) |
         (static_cast<uint32_t>(kIgRows >> 4) << 24);
}

// One 16-channel block of a tile for the calling warp's 32 rows (t = this
// lane's row). ystage: the warp's shared-memory buffer for a TMA store, or
// nullptr for direct stores.
// P = 0: the bf16 GEMM (fp32 accumulators, no scales).
template <int P>
__device__ __forceinline__ void ig_epilogue_chunk(uint32_t taddr, const IgJob& J, int64_t t, float xs,
                                                  int64_t i, bool row_ok, uint8_t* ystage, int lane) {
  constexpr int NP = P == 0 ? 1 : P;
  float raw[16 * NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) tmem_ld16(taddr + static_cast<uint32_t>(16 * q), raw + 16 * q);
  tmem_ld_wait();
  if (i >= J.d) return;                                  // warp-uniform
  if (ystage == nullptr ? !row_ok : t - lane >= J.tokens) return;   // no row of the block in Y
  float y[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    float v;
    if (P == 0) {
      v = raw[c];
    } else if (P == 1) {
      v = static_cast<float>(__float_as_int(raw[c]));
    } else {
      int64_t s = 0;
#pragma unroll
      for (int p = 0; p < P; ++p) s += static_cast<int64_t>(__float_as_int(raw[c * P + p])) << (7 * p);
      v = static_cast<float>(s);
    }
    y[c] = v;
  }
  float ws[16];
  if (P == 0) {
#pragma unroll
    for (int c = 0; c < 16; ++c) ws[c] = 1.0f;
  } else if (i + 16 <= J.d && (reinterpret_cast<uintptr_t>(J.w_scale) & 15u) == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 w4 = __ldg(reinterpret_cast<const float4*>(J.w_scale + i) + q);
      ws[4 * q] = w4.x;
      ws[4 * q + 1] = w4.y;
      ws[4 * q + 2] = w4.z;
      ws[4 * q + 3] = w4.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) ws[c] = i + c < J.d ? __ldg(J.w_scale + i + c) : 0.0f;
  }
  if (P != 0) {
#pragma unroll
    for (int c = 0; c < 16; ++c) y[c] *= xs * ws[c];
  }
  uint32_t yb[8];                                        // bf16 output: pairs, nearest even
  if (J.y_bf16) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * q], y[2 * q + 1]);
      yb[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  if (ystage != nullptr) {
    // the buffer's previous store (two blocks ago) has finished reading it
    if (lane == 0) bulk_wait_read<1>();
    __syncwarp();
    if (J.y_bf16) {
      // 32-byte rows: unit q of row `lane` at lane * 32 + 16 (q ^ ((lane >> 2) & 1))
      const uint32_t row = smem_u32(ystage) + static_cast<uint32_t>(lane) * 32u;
      const uint32_t sw = static_cast<uint32_t>((lane >> 2) & 1);
#pragma unroll
      for (int q = 0; q < 2; ++q)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     ::"r"(row + 16u * (static_cast<uint32_t>(q) ^ sw)), "r"(yb[4 * q]), "r"(yb[4 * q + 1]),
                       "r"(yb[4 * q + 2]), "r"(yb[4 * q + 3])
                     : "memory");
    } else {
      // row `lane`, 16-byte unit q at lane * 64 + 16 (q ^ ((lane >> 1) & 3))
      const uint32_t row = smem_u32(ystage) + static_cast<uint32_t>(lane) * 64u;
      const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};"
                     ::"r"(row + 16u * (static_cast<uint32_t>(q) ^ sw)), "f"(y[4 * q]), "f"(y[4 * q + 1]),
                       "f"(y[4 * q + 2]), "f"(y[4 * q + 3])
                     : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&J.y_map, ystage, static_cast<int32_t>(i), static_cast<int32_t>(t - lane));
      bulk_commit();
    }
    return;
  }
  if (J.y_bf16) {
    uint16_t* dst = static_cast<uint16_t*>(J.Y) + t * J.d + i;
    if (i + 16 <= J.d && (J.d & 7) == 0) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(yb[0], yb[1], yb[2], yb[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(yb[4], yb[5], yb[6], yb[7]);
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (i + c < J.d) dst[c] = static_cast<uint16_t>(yb[c >> 1] >> (16 * (c & 1)));
    }
    return;
  }
  float* dst = static_cast<float*>(J.Y) + t * J.d + i;
  if (i + 16 <= J.d && (J.d & 3) == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      reinterpret_cast<float4*>(dst)[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c)
      if (i + c < J.d) dst[c] = y[c];
  }
}

template <int P>
__global__ void __launch_bounds__(kIgThreads, 1) int_gemm_kernel(const __grid_constant__ IgBatch b) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ __align__(8) uint64_t drain_bar;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const int S = b.stages;
  constexpr int NP = P == 0 ? 1 : P;                    // P = 0: bf16 operands
  constexpr int kElems = P == 0 ? kIgK / 2 : kIgK;      // K elements per stage
  const int nrows = NP * b.chans;                       // digit rows of a tile
  const uint32_t b_bytes = static_cast<uint32_t>(nrows) * kIgK;
  const uint32_t stage_bytes = kIgABytes + b_bytes;     // multiple of 1024
  uint8_t* ystage = base + S * stage_bytes;              // [8 warps][2][32 x 16 fp32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ystage + kIgYStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* d_full = bars + 2 * S;                      // [2]
  uint64_t* d_empty = d_full + 2;                       // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&d_full[q], 1);
      mbar_init(&d_empty[q], kIgEpiThreads);
    }
    abort_flag = 0;
    mbar_init(&drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(2 * kIgMaxN) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;                      // accumulator q at column q * 256

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      int armed[kIgMaxStages];               // parity last armed per stage (-1: never)
      for (int q = 0; q < kIgMaxStages; ++q) armed[q] = -1;
      for (int64_t u = blockIdx.x; u < b.total_tiles && ok && !abort_flag; u += gridDim.x) {
        const IgTile x = ig_tile(b, u);
        const IgJob& J = b.job[x.job];
        const int32_t ty = static_cast<int32_t>(x.t0);
        const int32_t wy = static_cast<int32_t>(x.i0 * NP);
        for (int kb = 0; kb < J.k_stages; ++kb) {
          if (!wait_ig(&empty[stage], ph ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_tx(&full[stage], stage_bytes);
          armed[stage] = static_cast<int>(ph);
          uint8_t* dst = base + stage * stage_bytes;
          tma_load_2d(dst, &J.x_map, kb * kElems, ty, &full[stage]);
          tma_load_2d(dst + kIgABytes, &J.w_map, kb * kElems, wy, &full[stage]);
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
      int stage = 0, buf = 0;
      uint32_t ph = 0, bph = 0;
      const uint32_t idesc = P == 0 ? ig_idesc_bf16(nrows) : ig_idesc(nrows);
      bool ok = true;
      for (int64_t u = blockIdx.x; u < b.total_tiles && ok && !abort_flag; u += gridDim.x) {
        const IgTile x = ig_tile(b, u);
        const int kst = b.job[x.job].k_stages;
        if (!wait_ig(&d_empty[buf], bph ^ 1u, &abort_flag)) break;
        tc_fence_after();
        const uint32_t dt = tmem + static_cast<uint32_t>(buf * kIgMaxN);
        for (int kb = 0; kb < kst; ++kb) {
          if (!wait_ig(&full[stage], ph, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = kmajor_desc(smem_u32(base + stage * stage_bytes));
          const uint64_t b0 = kmajor_desc(smem_u32(base + stage * stage_bytes + kIgABytes));
#pragma unroll
          for (int ks = 0; ks < kIgK / 32; ++ks) {    // 32 bytes (16-byte units x 2) per MMA
            if (P == 0) tc_mma(dt, a0 + 2 * ks, b0 + 2 * ks, idesc, (kb | ks) != 0 ? 1u : 0u);
            else tc_mma_i8(dt, a0 + 2 * ks, b0 + 2 * ks, idesc, (kb | ks) != 0 ? 1u : 0u);
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
    // ---------------- epilogue: TMEM lane = token row of the tile
    const int e = (warp & 3) * 32 + lane;                 // row of the tile
    const int half = (warp - 4) >> 2;                     // channel half of the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int buf = 0;
    uint32_t bph = 0, nstore = 0;
    uint8_t* my_stage = ystage + (warp - 4) * 2 * kIgYBox;
    for (int64_t u = blockIdx.x; u < b.total_tiles && !abort_flag; u += gridDim.x) {
      const IgTile x = ig_tile(b, u);
      const IgJob& J = b.job[x.job];
      const int64_t t = x.t0 + e;
      const bool row_ok = t < J.tokens;
      const float xs = (P != 0 && row_ok) ? __ldg(J.x_scale + t) : 0.0f;
      if (!wait_ig(&d_full[buf], bph, &abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem + lane_base + static_cast<uint32_t>(buf * kIgMaxN);
      const int cbeg = half * (b.chans >> 1), cend = cbeg + (b.chans >> 1);
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        uint8_t* ys = J.y_tma ? my_stage + (nstore++ & 1u) * kIgYBox : nullptr;
        ig_epilogue_chunk<P>(tb + static_cast<uint32_t>(c0 * NP), J, t, xs, x.i0 + c0, row_ok, ys, lane);
      }
      tc_fence_before();
      mbar_arrive(&d_empty[buf]);
      if (++buf == 2) {
        buf = 0;
        bph ^= 1u;
      }
    }
  }

  if (warp >= 4 && lane == 0) bulk_wait<0>();           // this warp's Y stores are done
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kIgMaxN)
                 : "memory");
  }
}

size_t ig_smem_bytes(int planes, int stages) {
  const int np = planes == 0 ? 1 : planes;                // 0: bf16
  const size_t stage = kIgABytes + static_cast<size_t>(np * int_gemm_chans(planes)) * kIgK;
  return 1024 + static_cast<size_t>(stages) * stage + kIgYStage + (2 * stages + 4) * 8;
}

// ---- digit planes ----------------------------------------------------------------
__global__ void int_pack_kernel(const void* w, int w_bytes, int64_t d, int64_t n, int planes, int8_t* out,
                                int32_t* overflow) {
  const int64_t total = d * n;
  int32_t bad = 0;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t v;
    if (w_bytes == 1) v = static_cast<const int8_t*>(w)[e];
    else if (w_bytes == 2) v = static_cast<const int16_t*>(w)[e];
    else v = static_cast<const int32_t*>(w)[e];
    const int64_t i = e / n, j = e - i * n;
    int8_t* o = out + i * planes * n + j;
    for (int k = 0; k < planes; ++k) {
      const int64_t digit = k < planes - 1 ? (v >> (7 * k)) & 127 : v >> (7 * k);
      if (k == planes - 1 && (digit < -128 || digit > 127)) ++bad;
      o[k * n] = static_cast<int8_t>(digit);
    }
  }
  if (overflow != nullptr && bad != 0) atomicAdd(overflow, bad);
}

// W'_bf16 = bf16(fp32(s_bar_i) * q_ij): the merged weight as the bf16 operand
// of a training forward (one fp32 product rounded to nearest, then to bf16
// with ties to even). A CTA step covers kFqRows rows of one job; its threads
// walk those rows' 4-element groups as one flat range (n % 4 == 0), else
// element by element.
constexpr int kFqRows = 8;

struct FqBatch {
  FakeQuantJob job[kMaxBatch];
  int64_t step_begin[kMaxBatch + 1];   // CTA steps before job k
  int32_t count;
};

__device__ __forceinline__ int32_t q_at(const void* q, int q_bytes, int64_t e) {
  if (q_bytes == 1) return static_cast<const int8_t*>(q)[e];
  if (q_bytes == 2) return static_cast<const int16_t*>(q)[e];
  return static_cast<const int32_t*>(q)[e];
}
__device__ __forceinline__ uint16_t fq_one(float s, int32_t v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, static_cast<float>(v))));
}

__global__ void __launch_bounds__(256) fakequant_kernel(const __grid_constant__ FqBatch b) {
  const int64_t total = b.step_begin[b.count];
  int k = 0;
  for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
    while (k + 1 < b.count && b.step_begin[k + 1] <= c) ++k;
    const FakeQuantJob& J = b.job[k];
    const int64_t r0 = (c - b.step_begin[k]) * kFqRows;
    const int rows = static_cast<int>(min64(J.d - r0, kFqRows));
    if (J.n % 4 == 0) {
      const int64_t nq = J.n >> 2;                                // groups per row
      const int64_t groups = nq * rows;
      const bool narrow = groups < (int64_t{1} << 31);             // 32-bit division
      for (int64_t g = threadIdx.x; g < groups; g += blockDim.x) {
        const int64_t rr = narrow ? static_cast<int64_t>(static_cast<uint32_t>(g) / static_cast<uint32_t>(nq))
                                  : g / nq;
        const int64_t i = r0 + rr;
        const int64_t e = i * J.n + 4 * (g - rr * nq);
        const float s = __ldg(J.sbar + i);
        int32_t v[4];
        if (J.q_bytes == 1) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(static_cast<const int8_t*>(J.q) + e);
#pragma unroll
          for (int t = 0; t < 4; ++t) v[t] = static_cast<int8_t>(w >> (8 * t));
        } else if (J.q_bytes == 2) {
          const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const int16_t*>(J.q) + e);
          v[0] = static_cast<int16_t>(w.x);
          v[1] = static_cast<int16_t>(w.x >> 16);
          v[2] = static_cast<int16_t>(w.y);
          v[3] = static_cast<int16_t>(w.y >> 16);
        } else {
          const int4 w = *reinterpret_cast<const int4*>(static_cast<const int32_t*>(J.q) + e);
          v[0] = w.x;
          v[1] = w.y;
          v[2] = w.z;
          v[3] = w.w;
        }
        *reinterpret_cast<uint2*>(J.out + e) =
            make_uint2(fq_one(s, v[0]) | (static_cast<uint32_t>(fq_one(s, v[1])) << 16),
                       fq_one(s, v[2]) | (static_cast<uint32_t>(fq_one(s, v[3])) << 16));
      }
    } else {
      for (int rr = 0; rr < rows; ++rr) {
        const int64_t i = r0 + rr;
        const float s = __ldg(J.sbar + i);
        for (int64_t j = threadIdx.x; j < J.n; j += blockDim.x)
          J.out[i * J.n + j] = fq_one(s, q_at(J.q, J.q_bytes, i * J.n + j));
      }
    }
  }
}

}  // namespace

cudaError_t launch_fakequant(const FakeQuantJob* jobs, int count, cudaStream_t s) {
  static thread_local FqBatch b;
  for (int k0 = 0; k0 < count; k0 += kMaxBatch) {
    const int m = count - k0 < kMaxBatch ? count - k0 : kMaxBatch;
    std::memset(&b, 0, sizeof b);
    int64_t steps = 0;
    for (int k = 0; k < m; ++k) {
      b.job[k] = jobs[k0 + k];
      b.step_begin[k] = steps;
      steps += (jobs[k0 + k].d + kFqRows - 1) / kFqRows;
    }
    b.step_begin[m] = steps;
    b.count = m;
    if (steps == 0) continue;
    fakequant_kernel<<<static_cast<unsigned>(min64(steps, 148 * 8)), 256, 0, s>>>(b);
    const cudaError_t e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int int_gemm_chans(int planes) { return planes <= 1 ? 256 : planes == 2 ? 128 : 64; }

bool int_gemm_supported() { return tc::encode_fn() != nullptr; }

cudaError_t launch_int_pack(const void* w, int w_bytes, int64_t d, int64_t n, int planes, int8_t* out,
                            int32_t* overflow, cudaStream_t s) {
  const int64_t total = d * n;
  if (total <= 0) return cudaSuccess;
  const int64_t blocks = min64((total + 255) / 256, 148 * 16);
  int_pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(w, w_bytes, d, n, planes, out, overflow);
  return counted(cudaGetLastError());
}

// planes = 0: the bf16 GEMM Y = X W^T (X, W bf16 bit patterns, scales unused).
cudaError_t launch_int_gemm(const IntGemmJob* jobs, int count, int planes, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  const bool bf16 = planes == 0;
  const int np = bf16 ? 1 : planes;
  const CUtensorMapDataType dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int esize = bf16 ? 2 : 1;
  const int kelems = kIgK / esize;            // K elements per 128-byte stage
  static thread_local IgBatch b;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int chans = int_gemm_chans(planes);
  for (int k0 = 0; k0 < count; k0 += kMaxIgJobs) {
    const int m = count - k0 < kMaxIgJobs ? count - k0 : kMaxIgJobs;
    std::memset(&b, 0, sizeof b);
    int64_t tiles = 0;
    for (int k = 0; k < m; ++k) {
      const IntGemmJob& j = jobs[k0 + k];
      IgJob& t = b.job[k];
      const bool ok =
          tc::encode_2d(&t.x_map, dt, esize, j.X, j.tokens, j.n, kelems, kIgRows) &&
          tc::encode_2d(&t.w_map, dt, esize, j.W, j.d * np, j.n, kelems, chans * np);
      if (!ok) return cudaErrorInvalidValue;
      // Y through TMA stores when its rows are 16-byte multiples
      t.y_bf16 = j.y_bf16;
      if (j.y_bf16)
        t.y_tma = (j.d % 8 == 0) &&
                  tc::encode_2d_swz(&t.y_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, j.Y, j.tokens, j.d, 16, 32,
                                    CU_TENSOR_MAP_SWIZZLE_32B) ? 1 : 0;
      else
        t.y_tma = (j.d % 4 == 0) &&
                  tc::encode_2d_swz(&t.y_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.Y, j.tokens, j.d, 16, 32,
                                    CU_TENSOR_MAP_SWIZZLE_64B) ? 1 : 0;
      t.x_scale = j.x_scale;
      t.w_scale = j.w_scale;
      t.Y = j.Y;
      t.tokens = j.tokens;
      t.d = j.d;
      t.n = j.n;
      t.m_tiles = static_cast<int32_t>((j.tokens + kIgRows - 1) / kIgRows);
      t.n_tiles = static_cast<int32_t>((j.d + chans - 1) / chans);
      t.k_stages = static_cast<int32_t>((j.n + kelems - 1) / kelems);
      t.tile_begin = tiles;
      tiles += static_cast<int64_t>(t.m_tiles) * t.n_tiles;
    }
    b.count = m;
    b.planes = planes;
    b.chans = chans;
    int stages = 8;
    while (stages > 2 && ig_smem_bytes(planes, stages) > 232448) --stages;
    b.stages = stages;
    b.total_tiles = tiles;
    const size_t smem = ig_smem_bytes(planes, stages);
    const void* fn = planes == 0   ? reinterpret_cast<const void*>(int_gemm_kernel<0>)
                     : planes == 1 ? reinterpret_cast<const void*>(int_gemm_kernel<1>)
                     : planes == 2 ? reinterpret_cast<const void*>(int_gemm_kernel<2>)
                                   : reinterpret_cast<const void*>(int_gemm_kernel<3>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    if (planes == 0) int_gemm_kernel<0><<<grid, kIgThreads, smem, s>>>(b);
    else if (planes == 1) int_gemm_kernel<1><<<grid, kIgThreads, smem, s>>>(b);
    else if (planes == 2) int_gemm_kernel<2><<<grid, kIgThreads, smem, s>>>(b);
    else int_gemm_kernel<3><<<grid, kIgThreads, smem, s>>>(b);
    e = counted(cudaGetLastError());
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

unsigned int int_gemm_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_ig_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
