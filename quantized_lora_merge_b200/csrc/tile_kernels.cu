// Row-tile kernels of the IntLoRA merge path (sm_100a):
//
//  kGen   base quantization of a layer [IntLoRA paper notes (ICML2025), method
//         section 1, AQS: W' = Q[W - sg(R)] + sg(R) + AB, and section 3, VMC:
//         R* = (sigma_W / sigma_R)^alpha R]: X = W - R*, per-row affine
//         quantizer -> W_round, s, z.
//  kMul   IntLoRA_MUL [same notes, section 2 MLA and "两种实现版本"]:
//         U = s + (R* + A B) / (W_round - z) (quotient 0 where W_round = z),
//         per-row affine quantizer of U -> U_round, s_bar, z_bar, and the
//         integer Hadamard product P = (U_round - z_bar) (W_round - z).
//  kShift IntLoRA_SHIFT [same section]: s_bar = max |U| per row, V = U / s_bar,
//         shift = nearest integer of -log2|V| (clamped), M = sign(V) (D >> shift).
//
// Design. A tile is m rows of one layer; a cluster of C CTAs covers it, CTA k
// owning the column slice [k n_c, (k+1) n_c). Every value of the tile (U or X)
// stays in registers between the two phases: phase A computes it and the
// per-row maxima (reduced with warp REDUX, shared-memory atomics and then
// across the cluster through distributed shared memory), phase B quantizes
// and stores. The layer is therefore read once and R is generated once. The
// B slice stays in shared memory across the tiles of a layer when it fits;
// work items are 4 rows x 4 columns so one B load and one A load feed 16 FMAs
// and one Philox call yields the 4 words of a row's 4 columns. Clusters keep a
// contiguous range of tiles, so B is restaged only at layer changes.
#include <cuda_runtime.h>

#include <cstdint>

#include "intlora_device.cuh"
#include "intlora_kernels.h"

namespace intlora {

namespace {

constexpr double kLn2 = 0.69314718055994530942;

struct SmemLayout {
  int b_floats, a_floats, rcp_floats;
  __host__ __device__ constexpr int b_off() const { return 0; }
  __host__ __device__ constexpr int a_off() const { return b_floats; }
  __host__ __device__ constexpr int rcp_off() const { return b_floats + a_floats; }
  __host__ __device__ constexpr int rows_off() const { return rcp_off() + rcp_floats; }
  // per-row area: s, z, q_inv, q_zero (4 words) + 2 x 2 slots (4 words)
  __host__ __device__ constexpr int total_words() const { return rows_off() + 8 * kMaxTileRows; }
};

__host__ __device__ constexpr SmemLayout layout_for(int variant) {
  return variant == kGen ? SmemLayout{0, 0, 0} : SmemLayout{kBSmemFloats, kASmemFloats, 512};
}

// Load the 4 codes of one item row (columns j .. j+3). aligned: one 32-bit
// (8-bit codes) or 16-bit (4-bit codes) load; otherwise per element.
template <int WBITS>
__device__ __forceinline__ uint32_t load_codes(const uint8_t* row, int64_t j, int valid,
                                               bool aligned) {
  if (WBITS == 8) {
    if (aligned && valid == 4) return __ldg(reinterpret_cast<const uint32_t*>(row + j));
    uint32_t v = 0;
    for (int c = 0; c < valid; ++c) v |= static_cast<uint32_t>(__ldg(row + j + c)) << (8 * c);
    return v;
  } else {
    if (aligned && valid == 4)
      return __ldg(reinterpret_cast<const uint16_t*>(row + (j >> 1)));
    uint32_t v = 0;
    for (int c = 0; c < valid; ++c) {
      const int64_t jj = j + c;
      const uint32_t byte = __ldg(row + (jj >> 1));
      v |= ((jj & 1) ? (byte >> 4) : (byte & 0xFu)) << (4 * c);
    }
    return v;
  }
}

template <int WBITS>
__device__ __forceinline__ int32_t code_at(uint32_t packed, int c) {
  return WBITS == 8 ? static_cast<int32_t>((packed >> (8 * c)) & 0xFFu)
                    : static_cast<int32_t>((packed >> (4 * c)) & 0xFu);
}

// Stores of one item row (4 columns): codes (kGen), P (kMul) or M (kShift),
// plus the optional per-element code output of the merges.
template <int VARIANT, int WBITS, bool ALIGNED>
__device__ __forceinline__ void store_item(const TileLayer& L, int out_bytes, int64_t i, int64_t j,
                                           int vcols, const int32_t res[4], const uint32_t code8[4]) {
  if (VARIANT == kGen) {
    if (L.out == nullptr) return;
    uint8_t* orow = static_cast<uint8_t*>(L.out) + i * L.ld_out;
    if (WBITS == 8) {
      const uint32_t packed = code8[0] | (code8[1] << 8) | (code8[2] << 16) | (code8[3] << 24);
      if (ALIGNED || vcols == 4) {
        *reinterpret_cast<uint32_t*>(orow + j) = packed;
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < vcols) orow[j + c] = static_cast<uint8_t>(code8[c]);
      }
    } else {
      const uint32_t packed = code8[0] | (code8[1] << 4) | (code8[2] << 8) | (code8[3] << 12);
      if (ALIGNED || vcols == 4) {
        *reinterpret_cast<uint16_t*>(orow + (j >> 1)) = static_cast<uint16_t>(packed);
      } else {
        // n is even for 4-bit codes, so a ragged quad holds exactly 2 columns
        orow[j >> 1] = static_cast<uint8_t>(packed & 0xFFu);
      }
    }
    return;
  }
  const int64_t e0 = i * L.n + j;
  const bool vec = ALIGNED || vcols == 4;
  if (vec && !ALIGNED) {
    // an unaligned layer has row starts off the vector boundary
    for (int c = 0; c < 4; ++c) {
      if (out_bytes == 4) static_cast<int32_t*>(L.out)[e0 + c] = res[c];
      else if (out_bytes == 2) static_cast<int16_t*>(L.out)[e0 + c] = static_cast<int16_t>(res[c]);
      else static_cast<int8_t*>(L.out)[e0 + c] = static_cast<int8_t>(res[c]);
      if (L.code_out != nullptr) L.code_out[e0 + c] = static_cast<uint8_t>(code8[c]);
    }
    return;
  }
  if (out_bytes == 4) {   // MUL products beyond the int16 bound
    int32_t* o = static_cast<int32_t*>(L.out) + e0;
    if (vec) {
      *reinterpret_cast<int4*>(o) = make_int4(res[0], res[1], res[2], res[3]);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < vcols) o[c] = res[c];
    }
  } else if (out_bytes == 2) {   // int16 products or merged codes
    int16_t* o = static_cast<int16_t*>(L.out) + e0;
    if (vec) {
      const uint32_t lo = (static_cast<uint32_t>(res[0]) & 0xFFFFu) | (static_cast<uint32_t>(res[1]) << 16);
      const uint32_t hi = (static_cast<uint32_t>(res[2]) & 0xFFFFu) | (static_cast<uint32_t>(res[3]) << 16);
      *reinterpret_cast<uint2*>(o) = make_uint2(lo, hi);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < vcols) o[c] = static_cast<int16_t>(res[c]);
    }
  } else {   // int8 merged codes (SHIFT with a base of at most 7 bits)
    int8_t* o = static_cast<int8_t*>(L.out) + e0;
    if (vec) {
      *reinterpret_cast<uint32_t*>(o) = (static_cast<uint32_t>(res[0]) & 0xFFu) |
                                        ((static_cast<uint32_t>(res[1]) & 0xFFu) << 8) |
                                        ((static_cast<uint32_t>(res[2]) & 0xFFu) << 16) |
                                        (static_cast<uint32_t>(res[3]) << 24);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < vcols) o[c] = static_cast<int8_t>(res[c]);
    }
  }
  if (L.code_out != nullptr) {
    uint8_t* co = L.code_out + e0;
    if (vec) {
      *reinterpret_cast<uint32_t*>(co) = code8[0] | (code8[1] << 8) | (code8[2] << 16) | (code8[3] << 24);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < vcols) co[c] = static_cast<uint8_t>(code8[c]);
    }
  }
}

// Non-negative floats (sign bit clear) order like their bit patterns, so row
// maxima are reduced as unsigned integers (REDUX, shared atomics, DSMEM).
__device__ __forceinline__ uint32_t ord(float v) { return __float_as_uint(v); }

template <int VARIANT, int WBITS, int RANK, bool ALIGNED>
__global__ void __launch_bounds__(kTileThreads, 2) tile_kernel(const __grid_constant__ TileBatch p) {
  constexpr SmemLayout lay = layout_for(VARIANT);
  constexpr int IPT = kItemsPerThread;
  constexpr int RPI = kRowsPerItem;
  extern __shared__ __align__(16) float smem[];
  float* Bs = smem + lay.b_off();
  float* At = smem + lay.a_off();
  float* rcp_tab = smem + lay.rcp_off();
  float* row_s = smem + lay.rows_off();
  int32_t* row_z = reinterpret_cast<int32_t*>(row_s + kMaxTileRows);
  float* q_inv = row_s + 2 * kMaxTileRows;
  int32_t* q_zero = reinterpret_cast<int32_t*>(row_s + 3 * kMaxTileRows);
  uint32_t* slots = reinterpret_cast<uint32_t*>(row_s + 4 * kMaxTileRows);  // [2][rows][2]
  __shared__ float s_cln2;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int C = p.cluster;
  const uint32_t crank = C > 1 ? cluster_ctarank() : 0u;
  const int64_t cl = blockIdx.x / C;
  const int64_t t_begin = cl * p.total_tiles / p.num_clusters;
  const int64_t t_end = (cl + 1) * p.total_tiles / p.num_clusters;
  const int qmax = (1 << p.bits) - 1;   // code range, or the largest shift for kShift

  if (VARIANT != kGen)
    for (int k = tid; k < 511; k += kTileThreads)
      rcp_tab[k] = (k == 255) ? 0.0f : __frcp_rn(static_cast<float>(k - 255));
  for (int k = tid; k < 4 * kMaxTileRows; k += kTileThreads) slots[k] = 0u;

  int li = 0, cur = -1;
  int64_t it_count = 0;
  for (int64_t t = t_begin; t < t_end; ++t, ++it_count) {
    while (li + 1 < p.count && p.layer[li + 1].tile_begin <= t) ++li;
    const TileLayer& L = p.layer[li];
    const int buf = static_cast<int>(it_count & 1);
    const int64_t row0 = (t - L.tile_begin) * L.m;
    const int rows = static_cast<int>(min64(L.m, L.d - row0));
    const int64_t col0 = static_cast<int64_t>(crank) * L.n_c;
    const int ncols = static_cast<int>(max64(0, min64(L.n_c, L.n - col0)));
    const int r = (VARIANT == kGen) ? 0 : (RANK > 0 ? RANK : L.r);
    const int m = L.m;
    const int n_c = L.n_c;

    __syncthreads();  // previous tile is done with At, row params and q params
    if (li != cur) {
      if (tid == 0) {
        const double c = pow(*L.sigma_w / *L.sigma_r, static_cast<double>(L.alpha));
        s_cln2 = static_cast<float>(c * kLn2);
      }
      if (VARIANT != kGen && L.b_resident) {
        for (int idx = tid; idx < r * n_c; idx += kTileThreads) {
          const int k = idx / n_c, jj = idx - k * n_c;
          Bs[idx] = jj < ncols ? __ldg(L.B + static_cast<int64_t>(k) * L.n + col0 + jj) : 0.0f;
        }
      }
      cur = li;
    }
    if (VARIANT != kGen) {
      for (int rr = tid; rr < m; rr += kTileThreads) {
        row_s[rr] = rr < rows ? __ldg(L.s + row0 + rr) : 0.0f;
        // zero-points outside the code range are clamped into it, so the
        // reciprocal table is never indexed outside [-2^b + 1, 2^b - 1]
        row_z[rr] = rr < rows ? clamp_i(__ldg(L.z + row0 + rr), 0, (1 << p.w_bits) - 1) : 0;
      }
      // A rows of the tile, read along the rank (coalesced), stored k-major
      for (int idx = tid; idx < r * m; idx += kTileThreads) {
        const int rr = idx / max(r, 1), k = idx - rr * max(r, 1);
        At[k * m + rr] = rr < rows ? __ldg(L.A + (row0 + rr) * static_cast<int64_t>(L.r) + k) : 0.0f;
      }
    }
    __syncthreads();
    const float c_ln2 = s_cln2;

    // ---- work items of this thread: 4 rows x 4 columns each
    const int quads = n_c >> 2;
    const int G = m / RPI;
    const int nitems = G * quads;
    int ig[IPT], iq[IPT];
    bool iok[IPT];
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
      const int it = tid + k * kTileThreads;
      const int g = it / quads;
      iq[k] = it - g * quads;
      iok[k] = it < nitems && 4 * iq[k] < ncols;
      ig[k] = min(g, G - 1);
    }

    float acc[IPT][RPI][4];
    uint32_t cw[IPT][RPI];

    // ---- phase A.1: codes (merges) or W (base quantization); rows past the
    // layer's end read the last row (their results are masked out)
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
#pragma unroll
      for (int ml = 0; ml < RPI; ++ml) {
        cw[k][ml] = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[k][ml][c] = 0.0f;
      }
      if (!iok[k]) continue;
      const int64_t j = col0 + 4 * iq[k];
      const int vcols = ALIGNED ? 4 : min(4, ncols - 4 * iq[k]);
#pragma unroll
      for (int ml = 0; ml < RPI; ++ml) {
        const int64_t i = row0 + min(ig[k] * RPI + ml, rows - 1);
        if (VARIANT == kGen) {
          const float* wr = static_cast<const float*>(L.src) + i * L.n;
          if (ALIGNED) {
            const float4 w4 = __ldg(reinterpret_cast<const float4*>(wr + j));
            acc[k][ml][0] = w4.x; acc[k][ml][1] = w4.y; acc[k][ml][2] = w4.z; acc[k][ml][3] = w4.w;
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (c < vcols) acc[k][ml][c] = __ldg(wr + j + c);
          }
        } else {
          const uint8_t* wr = static_cast<const uint8_t*>(L.src) + i * L.ld_src;
          cw[k][ml] = load_codes<WBITS>(wr, j, vcols, ALIGNED);
        }
      }
    }

    // ---- phase A.2: T = A B on the tile (CUDA-core FMA), B from shared memory
    if (VARIANT != kGen) {
      auto fma_tile = [&](const float* arow, const float* brow) {
#pragma unroll
        for (int k = 0; k < IPT; ++k) {
          const float4 a4 = *reinterpret_cast<const float4*>(arow + ig[k] * RPI);
          const float4 b4 = *reinterpret_cast<const float4*>(brow + 4 * iq[k]);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
          const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int ml = 0; ml < RPI; ++ml)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[k][ml][c] = fmaf(av[ml], bv[c], acc[k][ml][c]);
        }
      };
      if (L.b_resident) {
        if (RANK > 0) {
#pragma unroll
          for (int kk = 0; kk < RANK; ++kk) fma_tile(At + kk * m, Bs + kk * n_c);
        } else {
#pragma unroll 4
          for (int kk = 0; kk < r; ++kk) fma_tile(At + kk * m, Bs + kk * n_c);
        }
      } else {
        for (int k0 = 0; k0 < r; k0 += L.kc) {
          const int kn = min(L.kc, r - k0);
          __syncthreads();
          for (int idx = tid; idx < kn * n_c; idx += kTileThreads) {
            const int kk = idx / n_c, jj = idx - kk * n_c;
            Bs[idx] = jj < ncols ? __ldg(L.B + static_cast<int64_t>(k0 + kk) * L.n + col0 + jj)
                                 : 0.0f;
          }
          __syncthreads();
#pragma unroll 4
          for (int kk = 0; kk < kn; ++kk) fma_tile(At + (k0 + kk) * m, Bs + kk * n_c);
        }
      }
    }

    // ---- phase A.3: R*, the value to quantize, and the row maxima
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
      float hi[RPI], lo[RPI];
#pragma unroll
      for (int ml = 0; ml < RPI; ++ml) hi[ml] = lo[ml] = 0.0f;
      if (iok[k]) {
        const int jl = 4 * iq[k];
        const int vcols = ALIGNED ? 4 : min(4, ncols - jl);
#pragma unroll
        for (int ml = 0; ml < RPI; ++ml) {
          const int rr = ig[k] * RPI + ml;
          const bool row_ok = rr < rows;
          const int64_t e0 = (row0 + min(rr, rows - 1)) * L.n + col0 + jl;
          uint32_t words[4];
          if (ALIGNED) {
            const uint4 w4 = aux_block(static_cast<uint64_t>(e0) >> 2, L.stream_id, L.key0, L.key1);
            words[0] = w4.x; words[1] = w4.y; words[2] = w4.z; words[3] = w4.w;
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              words[c] = c < vcols ? aux_word(static_cast<uint64_t>(e0 + c), L.stream_id, L.key0,
                                              L.key1)
                                   : 0u;
          }
          float sv = 0.0f;
          int32_t zv = 0;
          if (VARIANT != kGen) {
            sv = row_s[rr];
            zv = row_z[rr];
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float lg = laplace_log2(words[c]);
            const float cs = laplace_sign(words[c], c_ln2);   // +-c ln2
            float v;
            if (VARIANT == kGen) {
              if (L.r_star_out != nullptr && row_ok && (ALIGNED || c < vcols))
                L.r_star_out[e0 + c] = lg * cs;
              v = fmaf(-lg, cs, acc[k][ml][c]);                // W - R*
            } else {
              const int32_t dcode = code_at<WBITS>(cw[k][ml], c) - zv;
              v = fmaf(fmaf(lg, cs, acc[k][ml][c]), rcp_tab[dcode + 255], sv);
            }
            const bool ok = row_ok && (ALIGNED || c < vcols);
            v = ok ? v : 0.0f;
            acc[k][ml][c] = v;
            if (VARIANT == kShift) {
              hi[ml] = fmaxf(hi[ml], fabsf(v));
            } else {
              hi[ml] = fmaxf(hi[ml], v);
              lo[ml] = fminf(lo[ml], v);
            }
          }
        }
      }
      // reduce over the lanes holding the same rows, then one atomic per group
      const int key = iok[k] ? ig[k] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      const int leader = __ffs(peers) - 1;
#pragma unroll
      for (int ml = 0; ml < RPI; ++ml) {
        // hi >= 0 >= lo in value; fabsf drops a possible -0.0, whose bit
        // pattern would otherwise win the unsigned maximum
        const uint32_t a = __reduce_max_sync(peers, ord(fabsf(hi[ml])));
        const uint32_t b = (VARIANT == kShift) ? 0u : __reduce_max_sync(peers, ord(fabsf(lo[ml])));
        const int rr = ig[k] * RPI + ml;
        if (lane == leader && key >= 0 && rr < rows) {
          atomicMax(&slots[(buf * kMaxTileRows + rr) * 2 + 0], a);
          if (VARIANT != kShift) atomicMax(&slots[(buf * kMaxTileRows + rr) * 2 + 1], b);
        }
      }
    }

    // ---- row statistics across the cluster, then quantizer parameters
    __syncthreads();
    if (C > 1) {
      cluster_arrive_release();
      cluster_wait_acquire();
    }
    if (tid < kMaxTileRows) {
      slots[((buf ^ 1) * kMaxTileRows + tid) * 2 + 0] = 0u;
      slots[((buf ^ 1) * kMaxTileRows + tid) * 2 + 1] = 0u;
    }
    for (int rr = tid; rr < rows; rr += kTileThreads) {
      uint32_t a = 0u, b = 0u;
      const uint32_t* sp = &slots[(buf * kMaxTileRows + rr) * 2];
      if (C > 1) {
        for (int k = 0; k < C; ++k) {
          a = max(a, ld_dsmem_u32(map_smem_to_rank(sp, k)));
          b = max(b, ld_dsmem_u32(map_smem_to_rank(sp + 1, k)));
        }
      } else {
        a = sp[0];
        b = sp[1];
      }
      const float top = __uint_as_float(a), neg_bottom = __uint_as_float(b);
      float scale;
      int32_t zero = 0;
      if (VARIANT == kShift) {
        scale = top > 0.0f ? top : 1.0f;
      } else {
        scale = __fdiv_rn(top + neg_bottom, static_cast<float>(qmax));
        if (scale > 0.0f) {
          zero = clamp_i(static_cast<int32_t>(rintf(__fdiv_rn(neg_bottom, scale))), 0, qmax);
        } else {
          scale = 1.0f;
        }
      }
      q_inv[rr] = __frcp_rn(scale);
      q_zero[rr] = zero;
      if (crank == 0) {
        if (L.scale_out != nullptr) L.scale_out[row0 + rr] = scale;
        if (VARIANT != kShift && L.zero_out != nullptr) L.zero_out[row0 + rr] = zero;
      }
    }
    __syncthreads();

    // ---- phase B: quantize from registers and store
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
      if (!iok[k]) continue;
      const int jl = 4 * iq[k];
      const int vcols = ALIGNED ? 4 : min(4, ncols - jl);
      const int64_t j = col0 + jl;
#pragma unroll
      for (int ml = 0; ml < RPI; ++ml) {
        const int rr = ig[k] * RPI + ml;
        if (rr >= rows) continue;
        const int64_t i = row0 + rr;
        const float inv = q_inv[rr];
        const int32_t zero = q_zero[rr];
        const int32_t zv = VARIANT == kGen ? 0 : row_z[rr];
        int32_t res[4];
        uint32_t code8[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float v = acc[k][ml][c];
          if (VARIANT == kShift) {
            const float vn = v * inv;
            const int32_t sh = clamp_i(neg_log2_round(vn), 0, qmax);
            const int32_t dcode = code_at<WBITS>(cw[k][ml], c) - zv;
            const int32_t sgn = vn > 0.0f ? 1 : (vn < 0.0f ? -1 : 0);
            res[c] = sgn * (dcode >> sh);
            code8[c] = static_cast<uint32_t>(sh);
          } else if (VARIANT == kMul) {
            const int32_t centred = clamp_i(rne_scaled(v, inv), -zero, qmax - zero);
            const int32_t dcode = code_at<WBITS>(cw[k][ml], c) - zv;
            res[c] = centred * dcode;
            code8[c] = static_cast<uint32_t>(centred + zero);
          } else {
            code8[c] = static_cast<uint32_t>(clamp_i(rne_scaled(v, inv) + zero, 0, qmax));
            res[c] = 0;
          }
        }
        store_item<VARIANT, WBITS, ALIGNED>(L, p.out_bytes, i, j, vcols, res, code8);
      }
    }
  }
  // No CTA may leave while a cluster peer can still read its row slots.
  if (C > 1) {
    cluster_arrive_release();
    cluster_wait_acquire();
  }
}

template <int VARIANT, int WBITS, int RANK, bool ALIGNED>
cudaError_t launch_one(const TileBatch& b, cudaStream_t s) {
  auto kern = tile_kernel<VARIANT, WBITS, RANK, ALIGNED>;
  const size_t smem = static_cast<size_t>(layout_for(VARIANT).total_words()) * 4;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  if (b.cluster > 8) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(b.num_clusters * b.cluster));
  cfg.blockDim = dim3(kTileThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(b.cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, b);
}

template <int VARIANT, int WBITS, int RANK, bool ALIGNED>
int max_clusters_one(int cluster) {
  auto kern = tile_kernel<VARIANT, WBITS, RANK, ALIGNED>;
  const size_t smem = static_cast<size_t>(layout_for(VARIANT).total_words()) * 4;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return 0;
  if (cluster > 8 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cluster));
  cfg.blockDim = dim3(kTileThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int VARIANT, int WBITS, bool ALIGNED>
cudaError_t dispatch_rank(const TileBatch& b, int rank_ct, cudaStream_t s) {
  switch (rank_ct) {
    case 4: return launch_one<VARIANT, WBITS, 4, ALIGNED>(b, s);
    case 8: return launch_one<VARIANT, WBITS, 8, ALIGNED>(b, s);
    case 16: return launch_one<VARIANT, WBITS, 16, ALIGNED>(b, s);
    case 32: return launch_one<VARIANT, WBITS, 32, ALIGNED>(b, s);
    default: return launch_one<VARIANT, WBITS, 0, ALIGNED>(b, s);
  }
}

template <int VARIANT, int WBITS, bool ALIGNED>
int clusters_rank(int rank_ct, int cluster) {
  switch (rank_ct) {
    case 4: return max_clusters_one<VARIANT, WBITS, 4, ALIGNED>(cluster);
    case 8: return max_clusters_one<VARIANT, WBITS, 8, ALIGNED>(cluster);
    case 16: return max_clusters_one<VARIANT, WBITS, 16, ALIGNED>(cluster);
    case 32: return max_clusters_one<VARIANT, WBITS, 32, ALIGNED>(cluster);
    default: return max_clusters_one<VARIANT, WBITS, 0, ALIGNED>(cluster);
  }
}

template <int VARIANT, bool ALIGNED>
cudaError_t dispatch_bits(const TileBatch& b, int wb, int rank_ct, cudaStream_t s) {
  if constexpr (VARIANT == kGen) {
    return wb == 8 ? launch_one<kGen, 8, 0, ALIGNED>(b, s) : launch_one<kGen, 4, 0, ALIGNED>(b, s);
  } else {
    return wb == 8 ? dispatch_rank<VARIANT, 8, ALIGNED>(b, rank_ct, s)
                   : dispatch_rank<VARIANT, 4, ALIGNED>(b, rank_ct, s);
  }
}

template <int VARIANT, bool ALIGNED>
int clusters_bits(int wb, int rank_ct, int cluster) {
  if constexpr (VARIANT == kGen) {
    return wb == 8 ? max_clusters_one<kGen, 8, 0, ALIGNED>(cluster)
                   : max_clusters_one<kGen, 4, 0, ALIGNED>(cluster);
  } else {
    return wb == 8 ? clusters_rank<VARIANT, 8, ALIGNED>(rank_ct, cluster)
                   : clusters_rank<VARIANT, 4, ALIGNED>(rank_ct, cluster);
  }
}

}  // namespace

size_t tile_kernel_smem_bytes() { return static_cast<size_t>(layout_for(kMul).total_words()) * 4; }

cudaError_t launch_tiles(int variant, const TileBatch& b, int rank_ct, bool aligned, cudaStream_t s) {
  const int wb = variant == kGen ? b.bits : b.w_bits;
  if (variant == kGen)
    return aligned ? dispatch_bits<kGen, true>(b, wb, 0, s) : dispatch_bits<kGen, false>(b, wb, 0, s);
  if (variant == kMul)
    return aligned ? dispatch_bits<kMul, true>(b, wb, rank_ct, s)
                   : dispatch_bits<kMul, false>(b, wb, rank_ct, s);
  return aligned ? dispatch_bits<kShift, true>(b, wb, rank_ct, s)
                 : dispatch_bits<kShift, false>(b, wb, rank_ct, s);
}

int tile_max_active_clusters(int variant, int w_bits, int rank_ct, bool aligned, int cluster) {
  if (variant == kGen)
    return aligned ? clusters_bits<kGen, true>(w_bits, 0, cluster)
                   : clusters_bits<kGen, false>(w_bits, 0, cluster);
  if (variant == kMul)
    return aligned ? clusters_bits<kMul, true>(w_bits, rank_ct, cluster)
                   : clusters_bits<kMul, false>(w_bits, rank_ct, cluster);
  return aligned ? clusters_bits<kShift, true>(w_bits, rank_ct, cluster)
                 : clusters_bits<kShift, false>(w_bits, rank_ct, cluster);
}

}  // namespace intlora
