// Team kernels of the IntLoRA merge path (sm_100a): the same three per-row
// operations as the row-tile kernels (base quantization of W - R*, the MUL
// merge and the SHIFT merge; IntLoRA paper notes (ICML2025), method sections
// 1-3), laid out so that warps do not wait on one another inside a layer.
//
// A team of TW warps owns a group of 4 rows across the whole row. Lane l of
// the team takes the column quads q = l, l + 32 TW, ... ("sweeps"). Phase A
// computes an item of 4 rows x 4 columns (one Philox block per row: the 4
// words of its 4 columns), keeps the running row extrema in registers and
// parks the values (and the code words of the merges) in a lane-private
// stretch of shared memory: only the lane that wrote a value reads it back,
// so no synchronisation is needed for it. The row extrema are reduced over
// the warp with REDUX and over the team through a small slot array and one
// named barrier (none when TW = 1). Phase B quantizes the parked values and
// stores. B is read through the L1 cache (16-byte loads), A and the row
// parameters once per row group.
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "intlora_device.cuh"
#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

constexpr double kLn2 = 0.69314718055994530942;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kSlotWords = 2 * kTeamRows;      // row maxima and negated minima of one warp

__device__ __forceinline__ uint32_t ord(float v) { return __float_as_uint(fabsf(v)); }

__device__ __forceinline__ void team_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 4 x the 4-bit code c of a packed word (a byte offset into a 16-entry table).
__device__ __forceinline__ uint32_t nib4_x4(uint32_t packed, int c) {
  return c == 0 ? (packed << 2) & 0x3Cu : (packed >> (4 * c - 2)) & 0x3Cu;
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

template <int WBITS>
__device__ __forceinline__ int32_t nib(uint32_t packed, int c) {
  return WBITS == 8 ? static_cast<int32_t>((packed >> (8 * c)) & 0xFFu)
                    : static_cast<int32_t>((packed >> (4 * c)) & 0xFu);
}

template <int WBITS>
__device__ __forceinline__ uint32_t load_quad_codes(const uint8_t* row, int64_t j) {
  return WBITS == 8 ? __ldg(reinterpret_cast<const uint32_t*>(row + j))
                    : static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(row + (j >> 1))));
}

// One of the kTeamRows values selected by a small runtime index, without a
// local array (keeps the operands in registers).
template <typename T>
__device__ __forceinline__ T pick_row(const T v[kTeamRows], int k) {
  T x = v[0];
#pragma unroll
  for (int ml = 1; ml < kTeamRows; ++ml) x = k == ml ? v[ml] : x;
  return x;
}

// TMS > 0 (base quantization of wide rows only): sweeps k < TMS of a lane are
// parked in tensor memory, lane 32 (warp % 4) + lane, columns
// 128 (warp / 4) + 16 k .. + 15 (its 4 rows x 4 values); the later sweeps in
// shared memory as usual. Every lane then has the same number of sweeps
// (the host takes only rows that are a whole number of sweeps), so the
// warp-collective tensor-memory accesses are never divergent.
template <int VARIANT, int WBITS, int RANK, int OUTB, int TMS>
__global__ void __launch_bounds__(kTeamThreads, 2) team_kernel(const __grid_constant__ TeamBatch p) {
  static_assert(TMS == 0 || (VARIANT == kGen && TMS * kTeamRows * 4 * 2 <= 256), "tensor-memory parking: kGen, 256 columns");
  extern __shared__ __align__(16) float4 smem4[];
  __shared__ uint32_t tmem_slot;
  const int smax = p.sweeps_max;
  float4* Ubuf = smem4;                                              // [smax][4][256]
  // code words of the merges: [smax][kTeamRows][256]
  uint32_t* Cbuf = reinterpret_cast<uint32_t*>(smem4 + smax * kTeamRows * kTeamThreads);
  // row extrema of every warp: [2][warps][2 kTeamRows] (double buffered)
  uint32_t* slots = Cbuf + (VARIANT == kGen ? 0 : smax * kTeamRows * kTeamThreads);
  float* rcp_tab = reinterpret_cast<float*>(slots + 2 * kTeamWarps * kSlotWords);   // 1/D, D in [-255, 255]
  // 4-bit merges: each warp's 1/(code - z) for its 4 rows x 16 codes (256-byte
  // aligned, so a row entry's address is base | code * 4 + row * 64)
  const uint32_t lut_base =
      (static_cast<uint32_t>(__cvta_generic_to_shared(rcp_tab + 512)) + 255u) & ~255u;
  const uint32_t my_lut = lut_base + static_cast<uint32_t>(threadIdx.x >> 5) * 256u;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qmax = (1 << p.bits) - 1;
  if (VARIANT != kGen)
    for (int k = tid; k < 511; k += kTeamThreads)
      rcp_tab[k] = (k == 255) ? 0.0f : __frcp_rn(static_cast<float>(k - 255));
  uint32_t tpark = 0;                      // this thread's first parking column in tensor memory
  if (TMS > 0) {
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                   ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(&tmem_slot))), "r"(256u) : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::tc_fence_before();
  }
  __syncthreads();
  if (TMS > 0) {
    tc::tc_fence_after();
    tpark = tmem_slot + ((static_cast<uint32_t>(warp & 3) * 32u) << 16) + static_cast<uint32_t>(warp >> 2) * 128u;
  }

  const int64_t t_begin = p.cta_begin[blockIdx.x];
  const int64_t t_end = p.cta_begin[blockIdx.x + 1];
  int li = 0, cur = -1, cur_tw = 0;
  uint32_t phase = 0;
  float c_ln2 = 0.0f;
  for (int64_t t = t_begin; t < t_end; ++t) {
    while (li + 1 < p.count && p.layer[li + 1].tile_begin <= t) ++li;
    const TeamLayer& L = p.layer[li];
    if (li != cur) {
      if (L.team_warps != cur_tw) {
        // teams regroup: nobody may still be reading the slots of the old teams
        __syncthreads();
        cur_tw = L.team_warps;
        phase = 0;
      }
      const double c = pow(*L.sigma_w / *L.sigma_r, static_cast<double>(L.alpha));
      c_ln2 = static_cast<float>(c * kLn2);
      cur = li;
    }
    const int TW = cur_tw;
    const int teams = kTeamWarps / TW;
    const int team = warp / TW;
    const int wi = warp - team * TW;
    const int LT = TW * 32;
    const int lt = wi * 32 + lane;
    const int64_t row0 = ((t - L.tile_begin) * teams + team) * kTeamRows;
    if (row0 >= L.d) continue;                  // the whole team skips together
    const int rows = static_cast<int>(min64(kTeamRows, L.d - row0));
    const int64_t n = L.n;
    const int quads = static_cast<int>(n >> 2);
    const int S = L.sweeps;
    const uint8_t* __restrict__ src = static_cast<const uint8_t*>(L.src);
    const int64_t ld_src = L.ld_src;
    const uint32_t sid = L.stream_id;
    const PhiloxSmall ph = philox_small_setup(sid, p.key0, p.key1);
    // RANK > 0: fixed rank; 0: any rank; < 0: A B precomputed (L.T), no rank loop
    const int r = (VARIANT == kGen || RANK < 0) ? 0 : (RANK > 0 ? RANK : L.r);

    // row parameters and (small fixed rank) the A rows of the group
    int64_t irow[kTeamRows];
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) irow[ml] = row0 + min(ml, rows - 1);
    float sv[kTeamRows];
    int32_t zv[kTeamRows];
    constexpr int AREG = (RANK > 0 && RANK <= 8) ? RANK : 1;
    uint64_t areg[kTeamRows][AREG];          // (a, a) pairs for the f32x2 FMAs
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) {
      sv[ml] = 0.0f;
      zv[ml] = 0;
      if (VARIANT != kGen) {
        sv[ml] = __ldg(L.s + irow[ml]);
        zv[ml] = clamp_i(__ldg(L.z + irow[ml]), 0, (1 << WBITS) - 1);
        if (RANK > 0 && RANK <= 8) {
#pragma unroll
          for (int kk = 0; kk < AREG; ++kk) {
            const float a = __ldg(L.A + irow[ml] * RANK + kk);
            areg[ml][kk] = f2_pack(a, a);
          }
        }
      }
    }

#ifndef TEAM_NO_PREFETCH
    // The team's next row group of this layer is brought into L2 now (its
    // source rows and, for the merges, its row parameters and A rows), so the
    // next tile starts on L2 hits instead of HBM misses.
    {
      const int64_t nrow0 = row0 + static_cast<int64_t>(teams) * kTeamRows;
      if (t + 1 < t_end && nrow0 < L.d) {
        const int nrows = static_cast<int>(min64(kTeamRows, L.d - nrow0));
        const int64_t row_bytes = VARIANT == kGen ? 4 * n : (WBITS == 8 ? n : n / 2);
        const int lines = static_cast<int>((row_bytes + 127) / 128);
        if (VARIANT == kGen) {
          // fp32 rows: many lines per row, walked row by row without a division
          const uint8_t* nsrc = src + nrow0 * ld_src;
          for (int rr = 0; rr < nrows; ++rr, nsrc += ld_src)
            for (int line = lt; line < lines; line += LT) prefetch_l2(nsrc + static_cast<int64_t>(line) * 128);
        } else {
          for (int idx = lt; idx < nrows * lines; idx += LT) {
            const int rr = idx / lines;
            prefetch_l2(src + (nrow0 + rr) * ld_src + static_cast<int64_t>(idx - rr * lines) * 128);
          }
        }
        if (VARIANT != kGen && lt == 0) {
          prefetch_l2(L.s + nrow0);
          prefetch_l2(L.z + nrow0);
          prefetch_l2(L.A + nrow0 * r);
        }
      }
    }
#endif

    if (VARIANT != kGen && WBITS == 4) {
      __syncwarp();
      for (int e = lane; e < kTeamRows * 16; e += 32) {
        const int32_t zr = pick_row(zv, e >> 4);
        st_shared_f32(my_lut + 4u * static_cast<uint32_t>(e), rcp_tab[(e & 15) - zr + 255]);
      }
      __syncwarp();
    }

    uint32_t ctr0[kTeamRows];                   // Philox block of (row, quad 0)
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) ctr0[ml] = static_cast<uint32_t>(irow[ml] * quads);

    // ---- phase A
    // merges: the group's code rows addressed once (measured faster there;
    // the base quantization measured faster addressing each load)
    const uint8_t* srow[kTeamRows];
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) srow[ml] = src + irow[ml] * ld_src;
    float hi[kTeamRows], lo[kTeamRows];
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) hi[ml] = lo[ml] = 0.0f;
    for (int k = 0; k < S; ++k) {
      const int q = lt + k * LT;
      if (q >= quads) break;
      const int64_t j = 4 * static_cast<int64_t>(q);
      uint64_t acc[kTeamRows][2];            // columns (0, 1) and (2, 3) as f32x2 pairs
      uint32_t cw[kTeamRows];
#pragma unroll
      for (int ml = 0; ml < kTeamRows; ++ml) {
        cw[ml] = 0u;
        if (VARIANT == kGen) {
          const float4 w4 = __ldg(reinterpret_cast<const float4*>(src + irow[ml] * ld_src) + q);
          acc[ml][0] = f2_pack(w4.x, w4.y);
          acc[ml][1] = f2_pack(w4.z, w4.w);
        } else {
          cw[ml] = load_quad_codes<WBITS>(srow[ml], j);
          if (RANK < 0) {                        // A B precomputed on the tensor cores
            const float4 t4 = __ldg(reinterpret_cast<const float4*>(L.T + irow[ml] * n) + q);
            acc[ml][0] = f2_pack(t4.x, t4.y);
            acc[ml][1] = f2_pack(t4.z, t4.w);
          } else {
            acc[ml][0] = acc[ml][1] = 0ull;
          }
        }
      }
      if (VARIANT != kGen) {
        if (RANK > 0 && RANK <= 8) {
#pragma unroll
          for (int kk = 0; kk < AREG; ++kk) {
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(L.B + kk * n) + q);
            const uint64_t b01 = f2_pack(b4.x, b4.y), b23 = f2_pack(b4.z, b4.w);
#pragma unroll
            for (int ml = 0; ml < kTeamRows; ++ml) {
              acc[ml][0] = f2_fma(areg[ml][kk], b01, acc[ml][0]);
              acc[ml][1] = f2_fma(areg[ml][kk], b23, acc[ml][1]);
            }
          }
        } else {
#pragma unroll 4
          for (int kk = 0; kk < r; ++kk) {
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(L.B + kk * n) + q);
            const uint64_t b01 = f2_pack(b4.x, b4.y), b23 = f2_pack(b4.z, b4.w);
#pragma unroll
            for (int ml = 0; ml < kTeamRows; ++ml) {
              const float a = __ldg(L.A + irow[ml] * r + kk);
              const uint64_t a2 = f2_pack(a, a);
              acc[ml][0] = f2_fma(a2, b01, acc[ml][0]);
              acc[ml][1] = f2_fma(a2, b23, acc[ml][1]);
            }
          }
        }
      }
#pragma unroll
      for (int ml = 0; ml < kTeamRows; ++ml) {
        // layers here have fewer than 2^34 elements: the block index fits the
        // low counter word and the high word is 0 (rounds 0-1 partly uniform)
        // the folded form measured slower where A is read from L1 (ranks above 8)
        const uint4 w4 = (VARIANT == kGen || (RANK > 0 && RANK <= 8) || RANK < 0)
                             ? philox10_small(ctr0[ml] + static_cast<uint32_t>(q), ph)
                             : philox10(ctr0[ml] + static_cast<uint32_t>(q), 0u, sid, 0u, p.key0, p.key1);
        const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
        float v[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // columns 2h and 2h + 1 as one f32x2 pair
          const uint32_t wa = words[2 * h], wb = words[2 * h + 1];
          const uint64_t lg = laplace_log2_x2(wa, wb);
          uint64_t vp;
          if (VARIANT == kGen) {
            // W - R*: the sign factor negated (bit 31 of the word flipped)
            const uint64_t ncs = f2_pack(laplace_sign(wa ^ 0x80000000u, c_ln2),
                                         laplace_sign(wb ^ 0x80000000u, c_ln2));
            vp = f2_fma(lg, ncs, acc[ml][h]);
          } else {
            const uint64_t cs = f2_pack(laplace_sign(wa, c_ln2), laplace_sign(wb, c_ln2));
            float r0, r1;
            if (WBITS == 4) {
              // code c's entry: base | c * 4 (one shift and one 3-input logic op)
              const uint32_t row_lut = my_lut + static_cast<uint32_t>(ml) * 64u;   // 64-byte aligned
              r0 = ld_shared_f32(row_lut | nib4_x4(cw[ml], 2 * h));
              r1 = ld_shared_f32(row_lut | nib4_x4(cw[ml], 2 * h + 1));
            } else {
              r0 = rcp_tab[nib<WBITS>(cw[ml], 2 * h) - zv[ml] + 255];
              r1 = rcp_tab[nib<WBITS>(cw[ml], 2 * h + 1) - zv[ml] + 255];
            }
            vp = f2_fma(f2_fma(lg, cs, acc[ml][h]), f2_pack(r0, r1), f2_pack(sv[ml], sv[ml]));
          }
          v[2 * h] = f2_lo(vp);
          v[2 * h + 1] = f2_hi(vp);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (VARIANT == kShift) {
            hi[ml] = fmaxf(hi[ml], fabsf(v[c]));
          } else {
            hi[ml] = fmaxf(hi[ml], v[c]);
            lo[ml] = fminf(lo[ml], v[c]);
          }
        }
        if (TMS > 0 && k < TMS)
          tc::tmem_st4(tpark + static_cast<uint32_t>((k * kTeamRows + ml) * 4), make_float4(v[0], v[1], v[2], v[3]));
        else
          Ubuf[((k - TMS) * kTeamRows + ml) * kTeamThreads + tid] = make_float4(v[0], v[1], v[2], v[3]);
        if (VARIANT == kGen && L.r_star_out != nullptr && ml < rows) {
          float* rs = L.r_star_out + irow[ml] * n + j;
          *reinterpret_cast<float4*>(rs) =
              make_float4(laplace_scaled(words[0], c_ln2), laplace_scaled(words[1], c_ln2),
                          laplace_scaled(words[2], c_ln2), laplace_scaled(words[3], c_ln2));
        }
      }
      if (VARIANT != kGen) {
#pragma unroll
        for (int ml = 0; ml < kTeamRows; ++ml) Cbuf[(k * kTeamRows + ml) * kTeamThreads + tid] = cw[ml];
      }
    }

    if (TMS > 0) tc::tmem_st_wait_all();        // this warp's parked values are in

    // ---- row extrema: over the warp (REDUX), then over the team
    uint32_t ehi[kTeamRows], elo[kTeamRows];
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) {
      ehi[ml] = __reduce_max_sync(kFull, ord(hi[ml]));
      elo[ml] = VARIANT == kShift ? 0u : __reduce_max_sync(kFull, ord(lo[ml]));
    }
    if (TW > 1) {
      uint32_t* mine = slots + ((phase & 1u) * kTeamWarps + warp) * kSlotWords;
      if (lane == 0) {
#pragma unroll
        for (int ml = 0; ml < kTeamRows; ++ml) {
          mine[ml] = ehi[ml];
          mine[kTeamRows + ml] = elo[ml];
        }
      }
      team_barrier(1 + team, LT);
      // lane v < 2 kTeamRows gathers value v over the team's warps, then
      // every lane takes the combined values by shuffles
      uint32_t acc = 0u;
      if (lane < kSlotWords) {
        const uint32_t* base = slots + ((phase & 1u) * kTeamWarps + team * TW) * kSlotWords + lane;
        for (int w2 = 0; w2 < TW; ++w2) acc = max(acc, base[w2 * kSlotWords]);
      }
#pragma unroll
      for (int ml = 0; ml < kTeamRows; ++ml) {
        ehi[ml] = __shfl_sync(kFull, acc, ml);
        elo[ml] = __shfl_sync(kFull, acc, kTeamRows + ml);
      }
      ++phase;
    }

    // ---- quantizer parameters: lane ml < 4 works out row ml, then broadcast
    float scale = 1.0f;
    int32_t zero = 0;
    {
      const float top = __uint_as_float(pick_row(ehi, lane & (kTeamRows - 1)));
      const float neg_bottom = __uint_as_float(pick_row(elo, lane & (kTeamRows - 1)));
      if (VARIANT == kShift) {
        scale = top > 0.0f ? top : 1.0f;
      } else {
        scale = __fdiv_rn(top + neg_bottom, static_cast<float>(qmax));
        if (scale > 0.0f) zero = clamp_i(static_cast<int32_t>(rintf(__fdiv_rn(neg_bottom, scale))), 0, qmax);
        else scale = 1.0f;
      }
    }
    const float inv_own = __frcp_rn(scale);
    if (wi == 0 && lane < rows) {
      if (L.scale_out != nullptr) L.scale_out[row0 + lane] = scale;
      if (VARIANT != kShift && L.zero_out != nullptr) L.zero_out[row0 + lane] = zero;
    }
    float inv[kTeamRows];
    int32_t zq[kTeamRows];
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) {
      inv[ml] = __shfl_sync(kFull, inv_own, ml);
      zq[ml] = __shfl_sync(kFull, zero, ml);
    }

    // ---- phase B: quantize the parked values and store
    if (VARIANT == kGen && L.out == nullptr) continue;
    int32_t gen_lo[kTeamRows];                 // base quantization: bias - z per row
    uint8_t* orow[kTeamRows];                  // merges: output rows (bytes)
#pragma unroll
    for (int ml = 0; ml < kTeamRows; ++ml) {
      gen_lo[ml] = kRoundBiasBits - zq[ml];
      orow[ml] = static_cast<uint8_t*>(L.out) + irow[ml] * n * static_cast<int64_t>(OUTB);
    }
    // the merges form the U code bytes only when the layer asks for them
    // (two copies of the loop; the base quantization's output is the codes)
    auto phase_b = [&](auto want_code) {
      constexpr bool WC = decltype(want_code)::value;
      for (int k = 0; k < S; ++k) {
        const int q = lt + k * LT;
        if (q >= quads) break;
        const int64_t j = 4 * static_cast<int64_t>(q);
        uint32_t cw[kTeamRows];
  #pragma unroll
        for (int ml = 0; ml < kTeamRows; ++ml)
          cw[ml] = VARIANT != kGen ? Cbuf[(k * kTeamRows + ml) * kTeamThreads + tid] : 0u;
        float parked[TMS > 0 ? 16 : 1];             // the sweep's 4 rows from tensor memory
        if (TMS > 0 && k < TMS) {
          tc::tmem_ld16(tpark + static_cast<uint32_t>(k * kTeamRows * 4), parked);
          tc::tmem_ld_wait();
        }
  #pragma unroll
        for (int ml = 0; ml < kTeamRows; ++ml) {
          if (ml >= rows) break;
          const float4 u4 = (TMS > 0 && k < TMS)
                                ? make_float4(parked[4 * ml], parked[4 * ml + 1], parked[4 * ml + 2], parked[4 * ml + 3])
                                : Ubuf[((k - TMS) * kTeamRows + ml) * kTeamThreads + tid];
          const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
          const int64_t i = row0 + ml;
          int32_t res[4];
          uint32_t code8[4];
  #pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (VARIANT == kShift) {
              const float vn = uv[c] * inv[ml];
              const int32_t sh = clamp_i(neg_log2_round(vn), 0, qmax);
              const int32_t dcode = nib<WBITS>(cw[ml], c) - zv[ml];
              const int32_t sgn = vn > 0.0f ? 1 : (vn < 0.0f ? -1 : 0);
              res[c] = sgn * (dcode >> sh);
              if (WC) code8[c] = static_cast<uint32_t>(sh);
            } else if (VARIANT == kMul) {
              const int32_t centred = clamp_i(rne_scaled(uv[c], inv[ml]), -zq[ml], qmax - zq[ml]);
              res[c] = centred * (nib<WBITS>(cw[ml], c) - zv[ml]);
              if (WC) code8[c] = static_cast<uint32_t>(centred + zq[ml]);
            } else {
              // the biased rounding word clamped straight to the code range
              // [bias - z, bias - z + qmax]; the bias comes off once per word below
              code8[c] = static_cast<uint32_t>(
                  clamp_i(__float_as_int(fmaf(uv[c], inv[ml], kRoundBias)), gen_lo[ml], gen_lo[ml] + qmax));
              res[c] = 0;
            }
          }
          if (VARIANT == kGen) {
            // sum_c (word_c - lo) 2^(bits c), modulo 2^32 (multiply-adds)
            uint8_t* orow = static_cast<uint8_t*>(L.out) + i * L.ld_out;
            const uint32_t lo = static_cast<uint32_t>(gen_lo[ml]);
            if (WBITS == 8)
              *reinterpret_cast<uint32_t*>(orow + j) =
                  code8[0] + code8[1] * 0x100u + code8[2] * 0x10000u + code8[3] * 0x1000000u - lo * 0x01010101u;
            else
              *reinterpret_cast<uint16_t*>(orow + (j >> 1)) = static_cast<uint16_t>(
                  code8[0] + code8[1] * 16u + code8[2] * 256u + code8[3] * 4096u - lo * 0x1111u);
            continue;
          }
          uint8_t* const op = orow[ml] + j * OUTB;
          if (OUTB == 4) {
            *reinterpret_cast<int4*>(op) = make_int4(res[0], res[1], res[2], res[3]);
          } else if (OUTB == 2) {
            const uint32_t w0 = (static_cast<uint32_t>(res[0]) & 0xFFFFu) | (static_cast<uint32_t>(res[1]) << 16);
            const uint32_t w1 = (static_cast<uint32_t>(res[2]) & 0xFFFFu) | (static_cast<uint32_t>(res[3]) << 16);
            *reinterpret_cast<uint2*>(op) = make_uint2(w0, w1);
          } else {
            *reinterpret_cast<uint32_t*>(op) =
                (static_cast<uint32_t>(res[0]) & 0xFFu) | ((static_cast<uint32_t>(res[1]) & 0xFFu) << 8) |
                ((static_cast<uint32_t>(res[2]) & 0xFFu) << 16) | (static_cast<uint32_t>(res[3]) << 24);
          }
          if (WC)
            *reinterpret_cast<uint32_t*>(L.code_out + i * n + j) = code8[0] | (code8[1] << 8) | (code8[2] << 16) | (code8[3] << 24);
        }
      }
    };
    if (VARIANT == kGen || L.code_out != nullptr) phase_b(std::true_type{});
    else phase_b(std::false_type{});
  }
  if (TMS > 0) {
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc::tc_fence_after();
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_slot), "r"(256u) : "memory");
    }
  }
}

template <int VARIANT, int WBITS, int RANK, int OUTB, int TMS = 0>
struct TeamLaunch {
  static constexpr auto kernel() { return team_kernel<VARIANT, WBITS, RANK, OUTB, TMS>; }
  static cudaError_t launch(const TeamBatch& b, cudaStream_t s) {
    const size_t smem = team_smem_bytes(VARIANT, b.sweeps_max);
    cudaError_t err = cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    kernel()<<<b.num_ctas, kTeamThreads, smem, s>>>(b);
    return counted(cudaGetLastError());
  }
  static int max_ctas(size_t smem) {
    if (cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel(), kTeamThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    int dev = 0, sms = 0, smem_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (TMS > 0 && per_sm < 2) {
      // The occupancy query answers one CTA per SM for the tensor-memory
      // variant at any shared-memory size, yet two fit: 2 x 256 threads x
      // 128 registers is the register file, each CTA takes 256 of the 512
      // tensor-memory columns, and the shared memory is checked here
      // (measured on the 4096 x 14336 layers: 1.27x faster with two).
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kernel()) == cudaSuccess && fa.numRegs * kTeamThreads * 2 <= 65536 &&
          2 * (smem + fa.sharedSizeBytes + 1024) <= static_cast<size_t>(smem_sm))
        per_sm = 2;
    }
    return per_sm * sms;
  }
};

struct TeamQuery {
  int op;                    // 0: launch, 1: resident CTAs
  size_t smem;
  const TeamBatch* batch;
  cudaStream_t stream;
  int result;
  cudaError_t err;
};

template <int VARIANT, int WBITS, int RANK, int OUTB, int TMS = 0>
void team_run(TeamQuery& q) {
  using T = TeamLaunch<VARIANT, WBITS, RANK, OUTB, TMS>;
  if (q.op == 0) q.err = T::launch(*q.batch, q.stream);
  else q.result = T::max_ctas(q.smem);
}

template <int VARIANT, int WBITS, int OUTB>
void team_by_rank(TeamQuery& q, int rank_ct) {
  switch (rank_ct) {
    case 4: team_run<VARIANT, WBITS, 4, OUTB>(q); break;
    case 8: team_run<VARIANT, WBITS, 8, OUTB>(q); break;
    case 16: team_run<VARIANT, WBITS, 16, OUTB>(q); break;
    case -1: team_run<VARIANT, WBITS, -1, OUTB>(q); break;
    default: team_run<VARIANT, WBITS, 0, OUTB>(q); break;
  }
}

void team_dispatch(TeamQuery& q, int variant, int w_bits, int rank_ct, int out_bytes, bool tmem_park) {
  if (variant == kGen) {
    if (tmem_park) {
      if (w_bits == 8) team_run<kGen, 8, 0, 1, kTeamTmemSweeps>(q);
      else team_run<kGen, 4, 0, 1, kTeamTmemSweeps>(q);
    } else if (w_bits == 8) {
      team_run<kGen, 8, 0, 1>(q);
    } else {
      team_run<kGen, 4, 0, 1>(q);
    }
  } else if (variant == kMul) {
    if (w_bits == 8) {
      if (out_bytes == 4) team_by_rank<kMul, 8, 4>(q, rank_ct);
      else team_by_rank<kMul, 8, 2>(q, rank_ct);
    } else {
      team_by_rank<kMul, 4, 2>(q, rank_ct);
    }
  } else {
    if (w_bits == 8) team_by_rank<kShift, 8, 2>(q, rank_ct);
    else team_by_rank<kShift, 4, 1>(q, rank_ct);
  }
}

}  // namespace

size_t team_smem_bytes(int variant, int sweeps_max) {
  const size_t per_sweep = static_cast<size_t>(kTeamRows) * kTeamThreads * 16 +
                           (variant == kGen ? 0 : static_cast<size_t>(kTeamRows) * kTeamThreads * 4);
  return per_sweep * sweeps_max + 2 * kTeamWarps * kSlotWords * 4 +
         (variant == kGen ? 0 : 512 * 4 + 256 + kTeamWarps * 256);
}

cudaError_t launch_team(const TeamBatch& b, int variant, int rank_ct, int out_bytes, cudaStream_t s) {
  TeamQuery q{0, 0, &b, s, 0, cudaSuccess};
  team_dispatch(q, variant, variant == kGen ? b.bits : b.w_bits, rank_ct, out_bytes, b.tmem_sweeps > 0);
  return q.err;
}

int team_max_active_ctas(int variant, int w_bits, int rank_ct, int out_bytes, size_t smem, bool tmem_park) {
  TeamQuery q{1, smem, nullptr, nullptr, 0, cudaSuccess};
  team_dispatch(q, variant, w_bits, rank_ct, out_bytes, tmem_park);
  return q.result;
}

}  // namespace intlora
