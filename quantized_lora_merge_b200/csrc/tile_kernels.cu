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
// owning the column slice [k n_c, (k+1) n_c). Phase A computes the tile's
// values (U or X) into a shared-memory tile; a warp per row then reduces the
// row extrema (REDUX), which are combined across the cluster through
// distributed shared memory; phase B quantizes the tile from shared memory and
// stores. The layer is therefore read once and R generated once. Work items
// are 4 rows x 4 columns: one A load and one B load feed 16 FMAs and one
// Philox call yields the 4 words of a row's 4 columns. The B slice stays in
// shared memory across the tiles of a layer when it fits; clusters walk a
// contiguous range of tiles, so B is restaged only at layer changes. The
// shared-memory carve-up (tile, codes, B, A) is chosen per launch by the host.
#include <cuda_runtime.h>

#include <cstdint>

#include "intlora_device.cuh"
#include "intlora_kernels.h"

namespace intlora {

namespace {

constexpr double kLn2 = 0.69314718055994530942;
constexpr int RPI = kRowsPerItem;

// Load the 4 codes of one item row (columns j .. j+3). aligned: one 32-bit
// (8-bit codes) or 16-bit (4-bit codes) load; otherwise per element.
template <int WBITS, bool ALIGNED>
__device__ __forceinline__ uint32_t load_codes(const uint8_t* row, int64_t j, int valid) {
  if (WBITS == 8) {
    if (ALIGNED) return __ldg(reinterpret_cast<const uint32_t*>(row + j));
    uint32_t v = 0;
    for (int c = 0; c < valid; ++c) v |= static_cast<uint32_t>(__ldg(row + j + c)) << (8 * c);
    return v;
  } else {
    if (ALIGNED) return __ldg(reinterpret_cast<const uint16_t*>(row + (j >> 1)));
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
// plus the optional per-element code output of the merges. OUTB = bytes per
// element of `out` for the merges.
template <int VARIANT, int WBITS, int OUTB, bool ALIGNED>
__device__ __forceinline__ void store_item(void* out, uint8_t* code_out, int64_t ld_out, int64_t n,
                                           int64_t i, int64_t j, int vcols, const int32_t res[4],
                                           const uint32_t code8[4]) {
  if (VARIANT == kGen) {
    uint8_t* orow = static_cast<uint8_t*>(out) + i * ld_out;
    if (WBITS == 8) {
      const uint32_t packed = code8[0] | (code8[1] << 8) | (code8[2] << 16) | (code8[3] << 24);
      if (ALIGNED || vcols == 4) {
        *reinterpret_cast<uint32_t*>(orow + j) = packed;
      } else {
        for (int c = 0; c < vcols; ++c) orow[j + c] = static_cast<uint8_t>(code8[c]);
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
  const int64_t e0 = i * n + j;
  if (!ALIGNED) {   // row starts are off the vector boundary: element stores
    for (int c = 0; c < vcols; ++c) {
      if (OUTB == 4) static_cast<int32_t*>(out)[e0 + c] = res[c];
      else if (OUTB == 2) static_cast<int16_t*>(out)[e0 + c] = static_cast<int16_t>(res[c]);
      else static_cast<int8_t*>(out)[e0 + c] = static_cast<int8_t>(res[c]);
      if (code_out != nullptr) code_out[e0 + c] = static_cast<uint8_t>(code8[c]);
    }
    return;
  }
  if (OUTB == 4) {
    *reinterpret_cast<int4*>(static_cast<int32_t*>(out) + e0) = make_int4(res[0], res[1], res[2], res[3]);
  } else if (OUTB == 2) {
    const uint32_t lo = (static_cast<uint32_t>(res[0]) & 0xFFFFu) | (static_cast<uint32_t>(res[1]) << 16);
    const uint32_t hi = (static_cast<uint32_t>(res[2]) & 0xFFFFu) | (static_cast<uint32_t>(res[3]) << 16);
    *reinterpret_cast<uint2*>(static_cast<int16_t*>(out) + e0) = make_uint2(lo, hi);
  } else {
    *reinterpret_cast<uint32_t*>(static_cast<int8_t*>(out) + e0) =
        (static_cast<uint32_t>(res[0]) & 0xFFu) | ((static_cast<uint32_t>(res[1]) & 0xFFu) << 8) |
        ((static_cast<uint32_t>(res[2]) & 0xFFu) << 16) | (static_cast<uint32_t>(res[3]) << 24);
  }
  if (code_out != nullptr)
    *reinterpret_cast<uint32_t*>(code_out + e0) =
        code8[0] | (code8[1] << 8) | (code8[2] << 16) | (code8[3] << 24);
}

// Non-negative floats (sign bit clear) order like their bit patterns, so row
// extrema are reduced as unsigned integers (REDUX, shared atomics, DSMEM).
// fabsf also drops a -0.0, whose pattern would otherwise win the maximum.
__device__ __forceinline__ uint32_t ord(float v) { return __float_as_uint(fabsf(v)); }

// Walk of the items a thread owns: item it = tid + k T, i.e. (g, q) with
// it = g quads + q, advanced without division.
struct ItemWalk {
  int g, q, dg, dq, quads;
  __device__ __forceinline__ void init(int tid, int T, int quads_) {
    quads = quads_;
    g = tid / quads;
    q = tid - g * quads;
    dg = T / quads;
    dq = T - dg * quads;
  }
  __device__ __forceinline__ void next() {
    g += dg;
    q += dq;
    if (q >= quads) {
      q -= quads;
      ++g;
    }
  }
};

template <int VARIANT, int WBITS, int RANK, int OUTB, bool ALIGNED>
__global__ void __launch_bounds__(kTileThreads, 3) tile_kernel(const __grid_constant__ TileBatch p) {
  extern __shared__ __align__(16) float smem[];
  float* Us = smem;                                   // m x n_c tile of U (or X)
  uint32_t* Cs = reinterpret_cast<uint32_t*>(Us + p.smem_u);   // codes, one word per item row
  float* Bs = Us + p.smem_u + (VARIANT == kGen ? 0 : p.smem_u / 4);   // B slice, k-major
  float* At = Bs + p.smem_b;                          // A rows of the tile, k-major
  float* rcp_tab = At + p.smem_a;                     // 1/D for D in [-255, 255]
  float* row_s = rcp_tab + (VARIANT == kGen ? 0 : 512);
  int32_t* row_z = reinterpret_cast<int32_t*>(row_s + kMaxTileRows);
  float* q_inv = row_s + 2 * kMaxTileRows;
  int32_t* q_zero = reinterpret_cast<int32_t*>(row_s + 3 * kMaxTileRows);
  uint32_t* slots = reinterpret_cast<uint32_t*>(row_s + 4 * kMaxTileRows);  // [2][rows][2]
  const int warp = threadIdx.x >> 5;
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
    // RANK > 0: fixed rank; 0: any rank; -1: A B precomputed (L.T); -2: any
    // rank with an auxiliary law other than Laplace (p.dist)
    const int r = (VARIANT == kGen) ? 1 : (RANK == -1 ? 0 : (RANK > 0 ? RANK : L.r));
    const int m = L.m;
    const int n_c = L.n_c;
    // per-layer values used inside the item loops, read once per tile
    const int64_t n = L.n;
    const int64_t ld_src = L.ld_src;
    const uint8_t* __restrict__ src = static_cast<const uint8_t*>(L.src);
    const uint32_t sid = L.stream_id;
    const PhiloxSmall ph = philox_small_setup(sid, p.key0, p.key1);
    void* const out = L.out;
    uint8_t* const code_out = VARIANT == kGen ? nullptr : L.code_out;
    const int64_t ld_out = L.ld_out;
    float* const r_star_out = VARIANT == kGen ? L.r_star_out : nullptr;

    __syncthreads();  // previous tile is done with the tile buffer and row params
    if (li != cur) {
      if (tid == 0) {
        const double c = pow(*L.sigma_w / *L.sigma_r, static_cast<double>(L.alpha));
        s_cln2 = static_cast<float>(RANK == -2 ? c : c * kLn2);   // -2: c itself
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
      const int rdiv = r > 0 ? r : 1;
      for (int idx = tid; idx < r * m; idx += kTileThreads) {
        const int rr = idx / rdiv, k = idx - rr * r;
        At[k * m + rr] = rr < rows ? __ldg(L.A + (row0 + rr) * static_cast<int64_t>(L.r) + k) : 0.0f;
      }
    }
    __syncthreads();
    const float c_ln2 = s_cln2;

    const int quads = n_c >> 2;
    const int G = m / RPI;
    const int nitems = G * quads;

    // B slices that do not stay resident are streamed in chunks; then the
    // items accumulate A B into the tile buffer chunk by chunk first.
    const bool streamed = VARIANT != kGen && !L.b_resident;
    if (streamed) {
      for (int k0 = 0; k0 < r; k0 += L.kc) {
        const int kn = min(L.kc, r - k0);
        __syncthreads();
        for (int idx = tid; idx < kn * n_c; idx += kTileThreads) {
          const int kk = idx / n_c, jj = idx - kk * n_c;
          Bs[idx] = jj < ncols ? __ldg(L.B + static_cast<int64_t>(k0 + kk) * L.n + col0 + jj) : 0.0f;
        }
        __syncthreads();
        ItemWalk w;
        w.init(tid, kTileThreads, quads);
        for (int it = tid; it < nitems; it += kTileThreads, w.next()) {
          float acc[RPI][4];
#pragma unroll
          for (int ml = 0; ml < RPI; ++ml) {
            const float4 u = k0 == 0 ? make_float4(0.f, 0.f, 0.f, 0.f)
                                     : *reinterpret_cast<const float4*>(Us + (w.g * RPI + ml) * n_c + 4 * w.q);
            acc[ml][0] = u.x; acc[ml][1] = u.y; acc[ml][2] = u.z; acc[ml][3] = u.w;
          }
          for (int kk = 0; kk < kn; ++kk) {
            const float4 a4 = *reinterpret_cast<const float4*>(At + (k0 + kk) * m + w.g * RPI);
            const float4 b4 = *reinterpret_cast<const float4*>(Bs + kk * n_c + 4 * w.q);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
            const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int ml = 0; ml < RPI; ++ml)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[ml][c] = fmaf(av[ml], bv[c], acc[ml][c]);
          }
#pragma unroll
          for (int ml = 0; ml < RPI; ++ml)
            *reinterpret_cast<float4*>(Us + (w.g * RPI + ml) * n_c + 4 * w.q) =
                make_float4(acc[ml][0], acc[ml][1], acc[ml][2], acc[ml][3]);
        }
      }
    }

    // ---- phase A: values of the tile (and the code words of the merges)
    {
      const int64_t nq = n >> 2;   // Philox blocks per row (aligned layers)
      ItemWalk w;
      w.init(tid, kTileThreads, quads);
      for (int it = tid; it < nitems; it += kTileThreads, w.next()) {
        const int jl = 4 * w.q;
        if (jl >= ncols) continue;
        const int vcols = ALIGNED ? 4 : min(4, ncols - jl);
        const int64_t j = col0 + jl;
        float acc[RPI][4];
        uint32_t cw[RPI];
        // inputs: codes (merges) or W (base quantization); rows past the
        // layer's end read the last row (those values are never used)
#pragma unroll
        for (int ml = 0; ml < RPI; ++ml) {
          const int64_t i = row0 + min(w.g * RPI + ml, rows - 1);
          cw[ml] = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[ml][c] = 0.0f;
          if (VARIANT == kGen) {
            const float* wr = reinterpret_cast<const float*>(src) + i * n;
            if (ALIGNED) {
              const float4 w4 = __ldg(reinterpret_cast<const float4*>(wr + j));
              acc[ml][0] = w4.x; acc[ml][1] = w4.y; acc[ml][2] = w4.z; acc[ml][3] = w4.w;
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < vcols) acc[ml][c] = __ldg(wr + j + c);
            }
          } else {
            cw[ml] = load_codes<WBITS, ALIGNED>(src + i * ld_src, j, vcols);
          }
        }
        // T = A B on the item: precomputed on the tensor cores, or CUDA-core FMA
        if (VARIANT != kGen && RANK == -1) {
#pragma unroll
          for (int ml = 0; ml < RPI; ++ml) {
            const float* trow = L.T + (row0 + min(w.g * RPI + ml, rows - 1)) * n;
            if (ALIGNED) {
              const float4 t4 = __ldg(reinterpret_cast<const float4*>(trow + j));
              acc[ml][0] = t4.x; acc[ml][1] = t4.y; acc[ml][2] = t4.z; acc[ml][3] = t4.w;
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < vcols) acc[ml][c] = __ldg(trow + j + c);
            }
          }
        } else if (VARIANT != kGen) {
          if (streamed) {
#pragma unroll
            for (int ml = 0; ml < RPI; ++ml) {
              const float4 u = *reinterpret_cast<const float4*>(Us + (w.g * RPI + ml) * n_c + jl);
              acc[ml][0] = u.x; acc[ml][1] = u.y; acc[ml][2] = u.z; acc[ml][3] = u.w;
            }
          } else {
#pragma unroll 4
            for (int kk = 0; kk < r; ++kk) {
              const float4 a4 = *reinterpret_cast<const float4*>(At + kk * m + w.g * RPI);
              const float4 b4 = *reinterpret_cast<const float4*>(Bs + kk * n_c + jl);
              const float av[4] = {a4.x, a4.y, a4.z, a4.w};
              const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
              for (int ml = 0; ml < RPI; ++ml)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[ml][c] = fmaf(av[ml], bv[c], acc[ml][c]);
            }
          }
        }
        // R* and the value to quantize
        const int64_t blk0 = (row0 + w.g * RPI) * nq + (j >> 2);   // aligned layers only
#pragma unroll
        for (int ml = 0; ml < RPI; ++ml) {
          const int rr = w.g * RPI + ml;
          const int64_t e0 = (row0 + min(rr, rows - 1)) * n + j;
          uint32_t words[4];
          if (ALIGNED) {
            // layers below 2^34 elements: block index in the low counter word
            const uint4 w4 = p.small ? philox10_small(static_cast<uint32_t>(blk0 + ml * nq), ph)
                                     : aux_block(static_cast<uint64_t>(blk0 + ml * nq), sid, p.key0, p.key1);
            words[0] = w4.x; words[1] = w4.y; words[2] = w4.z; words[3] = w4.w;
          } else if (RANK != -2) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              words[c] = c < vcols ? aux_word(static_cast<uint64_t>(e0 + c), sid, p.key0, p.key1)
                                   : 0u;
          }
          float rv[4];                                   // RANK -2: R of each element
          if (RANK == -2) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              if (ALIGNED) {
                rv[c] = aux_value_generic(p.dist, words[c & 2], words[c | 1], (c & 1) != 0);
              } else if (c < vcols) {
                // the element's block (the Gaussian pairs words within it)
                const uint64_t e = static_cast<uint64_t>(e0 + c);
                const uint4 bw = aux_block(e >> 2, sid, p.key0, p.key1);
                const uint32_t ww[4] = {bw.x, bw.y, bw.z, bw.w};
                const int cc = static_cast<int>(e & 3u);
                rv[c] = aux_value_generic(p.dist, ww[cc & 2], ww[cc | 1], (cc & 1) != 0);
              } else {
                rv[c] = 0.0f;
              }
            }
          }
          float sv = 0.0f;
          int32_t zv = 0;
          if (VARIANT != kGen) {
            sv = row_s[rr];
            zv = row_z[rr];
          }
          float v[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float x;
            if (RANK == -2) {
              // c_ln2 holds c: R* = c R
              if (VARIANT == kGen) {
                x = fmaf(-c_ln2, rv[c], acc[ml][c]);
              } else {
                const int32_t dcode = code_at<WBITS>(cw[ml], c) - zv;
                x = fmaf(fmaf(c_ln2, rv[c], acc[ml][c]), rcp_tab[dcode + 255], sv);
              }
            } else {
              const float lg = laplace_log2(words[c]);
              const float cs = laplace_sign(words[c], c_ln2);   // +-c ln2
              if (VARIANT == kGen) {
                x = fmaf(-lg, cs, acc[ml][c]);                   // W - R*
              } else {
                const int32_t dcode = code_at<WBITS>(cw[ml], c) - zv;
                x = fmaf(fmaf(lg, cs, acc[ml][c]), rcp_tab[dcode + 255], sv);
              }
            }
            // columns past a ragged layer's end must not reach the extrema
            v[c] = (ALIGNED || c < vcols) ? x : 0.0f;
          }
          *reinterpret_cast<float4*>(Us + rr * n_c + jl) = make_float4(v[0], v[1], v[2], v[3]);
          if (VARIANT != kGen) Cs[rr * quads + w.q] = cw[ml];
          if (VARIANT == kGen && r_star_out != nullptr && rr < rows) {
            for (int c = 0; c < vcols; ++c)
              r_star_out[e0 + c] = RANK == -2 ? c_ln2 * rv[c]
                                              : laplace_log2(words[c]) * laplace_sign(words[c], c_ln2);
          }
        }
      }
    }
    __syncthreads();

    // ---- row extrema of the tile: one warp per row, REDUX over the lanes
    for (int rr = warp; rr < rows; rr += kTileThreads / 32) {
      float hi = 0.0f, lo = 0.0f;
      const float* urow = Us + rr * n_c;
      for (int q = lane; 4 * q < ncols; q += 32) {
        const float4 u = *reinterpret_cast<const float4*>(urow + 4 * q);
        if (VARIANT == kShift) {
          hi = fmaxf(hi, fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(u.z), fabsf(u.w))));
        } else {
          hi = fmaxf(hi, fmaxf(fmaxf(u.x, u.y), fmaxf(u.z, u.w)));
          lo = fminf(lo, fminf(fminf(u.x, u.y), fminf(u.z, u.w)));
        }
      }
      const uint32_t a = __reduce_max_sync(0xffffffffu, ord(hi));
      const uint32_t b = (VARIANT == kShift) ? 0u : __reduce_max_sync(0xffffffffu, ord(lo));
      if (lane == 0) {
        slots[(buf * kMaxTileRows + rr) * 2 + 0] = a;
        slots[(buf * kMaxTileRows + rr) * 2 + 1] = b;
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

    // ---- phase B: quantize the tile and store (one item row per step)
    if (VARIANT == kGen && out == nullptr) continue;
    {
      const int nrow_items = rows * quads;
      ItemWalk w;                            // (row, quad) walk: g is the row here
      w.init(tid, kTileThreads, quads);
      for (int ir = tid; ir < nrow_items; ir += kTileThreads, w.next()) {
        const int rr = w.g;
        const int jl = 4 * w.q;
        if (jl >= ncols) continue;
        const int vcols = ALIGNED ? 4 : min(4, ncols - jl);
        const int64_t i = row0 + rr;
        const int64_t j = col0 + jl;
        const float4 u = *reinterpret_cast<const float4*>(Us + rr * n_c + jl);
        const float uv[4] = {u.x, u.y, u.z, u.w};
        const float inv = q_inv[rr];
        const int32_t zero = q_zero[rr];
        uint32_t cw = 0u;
        int32_t zv = 0;
        if (VARIANT != kGen) {
          cw = Cs[rr * quads + w.q];
          zv = row_z[rr];
        }
        int32_t res[4];
        uint32_t code8[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (VARIANT == kShift) {
            const float vn = uv[c] * inv;
            const int32_t sh = clamp_i(neg_log2_round(vn), 0, qmax);
            const int32_t dcode = code_at<WBITS>(cw, c) - zv;
            const int32_t sgn = vn > 0.0f ? 1 : (vn < 0.0f ? -1 : 0);
            res[c] = sgn * (dcode >> sh);
            code8[c] = static_cast<uint32_t>(sh);
          } else if (VARIANT == kMul) {
            const int32_t centred = clamp_i(rne_scaled(uv[c], inv), -zero, qmax - zero);
            const int32_t dcode = code_at<WBITS>(cw, c) - zv;
            res[c] = centred * dcode;
            code8[c] = static_cast<uint32_t>(centred + zero);
          } else {
            code8[c] = static_cast<uint32_t>(clamp_i(rne_scaled(uv[c], inv) + zero, 0, qmax));
            res[c] = 0;
          }
        }
        store_item<VARIANT, WBITS, OUTB, ALIGNED>(out, code_out, ld_out, n, i, j, vcols, res, code8);
      }
    }
  }
  // No CTA may leave while a cluster peer can still read its row slots.
  if (C > 1) {
    cluster_arrive_release();
    cluster_wait_acquire();
  }
}

template <int VARIANT, int WBITS, int RANK, int OUTB, bool ALIGNED>
struct TileLaunch {
  static constexpr auto kernel() { return tile_kernel<VARIANT, WBITS, RANK, OUTB, ALIGNED>; }

  static cudaError_t prepare(int cluster, size_t smem) {
    auto kern = kernel();
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    if (cluster > 8) err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return err;
  }

  static cudaLaunchConfig_t config(int grid, int cluster, size_t smem, cudaStream_t s,
                                   cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kTileThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
  }

  static cudaError_t launch(const TileBatch& b, cudaStream_t s) {
    const size_t smem = tile_smem_bytes(b.variant, b.smem_u, b.smem_b, b.smem_a);
    cudaError_t err = prepare(b.cluster, smem);
    if (err != cudaSuccess) return err;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = config(b.num_clusters * b.cluster, b.cluster, smem, s, attr);
    return counted(cudaLaunchKernelEx(&cfg, kernel(), b));
  }

  static int max_clusters(int cluster, size_t smem) {
    if (prepare(cluster, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = config(cluster, cluster, smem, nullptr, attr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel(), &cfg) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return n;
  }
};

// Dispatch over the compile-time parameters. op = 0: launch, 1: occupancy.
struct TileQuery {
  int op;
  int cluster;
  size_t smem;
  const TileBatch* batch;
  cudaStream_t stream;
  int result;
  cudaError_t err;
};

template <int VARIANT, int WBITS, int RANK, int OUTB, bool ALIGNED>
void run_query(TileQuery& q) {
  using T = TileLaunch<VARIANT, WBITS, RANK, OUTB, ALIGNED>;
  if (q.op == 0) q.err = T::launch(*q.batch, q.stream);
  else q.result = T::max_clusters(q.cluster, q.smem);
}

template <int VARIANT, int WBITS, int OUTB, bool ALIGNED>
void by_rank(TileQuery& q, int rank_ct) {
  switch (rank_ct) {
    case 4: run_query<VARIANT, WBITS, 4, OUTB, ALIGNED>(q); break;
    case 8: run_query<VARIANT, WBITS, 8, OUTB, ALIGNED>(q); break;
    case 16: run_query<VARIANT, WBITS, 16, OUTB, ALIGNED>(q); break;
    case -1: run_query<VARIANT, WBITS, -1, OUTB, ALIGNED>(q); break;
    case -2: run_query<VARIANT, WBITS, -2, OUTB, ALIGNED>(q); break;
    default: run_query<VARIANT, WBITS, 0, OUTB, ALIGNED>(q); break;
  }
}

template <bool ALIGNED>
void by_variant(TileQuery& q, int variant, int w_bits, int rank_ct, int out_bytes) {
  if (variant == kGen) {
    if (rank_ct == -2) {
      if (w_bits == 8) run_query<kGen, 8, -2, 1, ALIGNED>(q);
      else run_query<kGen, 4, -2, 1, ALIGNED>(q);
    } else if (w_bits == 8) {
      run_query<kGen, 8, 0, 1, ALIGNED>(q);
    } else {
      run_query<kGen, 4, 0, 1, ALIGNED>(q);
    }
  } else if (variant == kMul) {
    if (w_bits == 8) {
      if (out_bytes == 4) by_rank<kMul, 8, 4, ALIGNED>(q, rank_ct);
      else by_rank<kMul, 8, 2, ALIGNED>(q, rank_ct);
    } else {
      by_rank<kMul, 4, 2, ALIGNED>(q, rank_ct);
    }
  } else {
    if (w_bits == 8) by_rank<kShift, 8, 2, ALIGNED>(q, rank_ct);
    else by_rank<kShift, 4, 1, ALIGNED>(q, rank_ct);
  }
}

void dispatch(TileQuery& q, int variant, int w_bits, int rank_ct, int out_bytes, bool aligned) {
  if (aligned) by_variant<true>(q, variant, w_bits, rank_ct, out_bytes);
  else by_variant<false>(q, variant, w_bits, rank_ct, out_bytes);
}

}  // namespace

size_t tile_smem_bytes(int variant, int smem_u, int smem_b, int smem_a) {
  const int codes = variant == kGen ? 0 : smem_u / 4;   // one code word per 4 tile values
  const int words = smem_u + codes + smem_b + smem_a + (variant == kGen ? 0 : 512) + 8 * kMaxTileRows;
  return static_cast<size_t>(words) * 4;
}

cudaError_t launch_tiles(const TileBatch& b, int rank_ct, bool aligned, cudaStream_t s) {
  TileQuery q{0, b.cluster, 0, &b, s, 0, cudaSuccess};
  dispatch(q, b.variant, b.variant == kGen ? b.bits : b.w_bits, rank_ct, b.out_bytes, aligned);
  return q.err;
}

int tile_max_active_clusters(int variant, int w_bits, int rank_ct, int out_bytes, bool aligned,
                             int cluster, size_t smem) {
  TileQuery q{1, cluster, smem, nullptr, nullptr, 0, cudaSuccess};
  dispatch(q, variant, w_bits, rank_ct, out_bytes, aligned);
  return q.result;
}

}  // namespace intlora
