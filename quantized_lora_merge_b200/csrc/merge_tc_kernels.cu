// Fused IntLoRA merge with the low-rank product on the 5th-generation tensor
// cores (sm_100a). One kernel per batch of layers computes, for every element
// of W, the adaptation term
//     U = s + (R* + A B) / (W_round - z)      (quotient 0 where W_round = z)
// [IntLoRA paper notes (ICML2025), method section 2, MLA], the per-row
// quantizer of U and the integer merged weight: MUL, P = (U_round - z_bar) D,
// or SHIFT, M = sign(U) (D >> shift) [same page, the two variants], with R
// regenerated from Philox4x32-10 and the Laplace inverse CDF [section 1, AQS]
// and scaled by the VMC factor c = (sigma_W / sigma_R)^alpha [section 3].
//
// Layout of the work. A unit is 128 rows of one layer. A group of G CTAs
// covers the unit's whole rows: CTA k of the group owns the column slice
// [k S, (k + 1) S), S <= 512. Tensor memory (128 lanes x 512 fp32 columns)
// holds T = A B for the slice, lane i = row i of the unit, written by the
// MMAs; every quantizer thread reads its lane (one row, 16 consecutive
// columns per tcgen05.ld: four Philox blocks of that row), forms U, keeps the
// row's running extrema in registers and writes U back in place
// (tcgen05.st). The extrema of the G CTAs are combined through a small
// exchange area in the caller's workspace: each CTA stores its 128 row
// extrema as one 64-bit word per row (both extrema and a 2-bit tag that
// tells this unit from the one two back, which used the same slot set), and
// the quantizer threads of a row read the other CTAs' words, two in flight
// at a time, until every tag matches; no fence, flag or extra barrier hop
// lies on that path. Then the same thread reads U back, quantizes it and
// stores its row's merged weights.
// Nothing else of the merge touches global memory.
//
// The launch is cooperative (every CTA resident, one per SM), so a CTA may
// wait for the other CTAs of its group; groups walk their units in lockstep.
// Groups are not hardware clusters: any G packs onto the 148 SMs (a cluster
// of 8 CTAs at one CTA per SM leaves 28 SMs idle).
//
// Low-rank product. T = A_hi B_hi + A_hi B_lo + A_lo B_hi on tf32 (the
// "three-term split": each fp32 operand split exactly into a tf32 head and a
// tf32 tail, written by t_split_kernel into the caller's workspace, K padded
// to kp = 32, 64 or 128 with zeros). tcgen05.mma.cta_group::1.kind::tf32,
// M = 128 (the unit's rows), N <= 128 columns per instruction ("part"), K = 8,
// fp32 accumulation in tensor memory. Tensor memory is handed back to the
// MMA issuer part by part as the quantizers finish reading U, so the next
// unit's products overlap the current unit's last parts.
//
// Roles (16 warps): warp 0 issues TMA loads (the unit's A tile once, B^T
// tiles through a ring of stages), warp 1 allocates tensor memory and issues
// the MMAs (one thread), warps 4-15 quantize: warps 4 + q, 8 + q and 12 + q
// serve lane quarter q (rows 32 q .. 32 q + 31) and take every third
// 16-column group (three warps per scheduler keep the issue slots busier
// than two; 128 registers a thread suffice without spills). Every wait is bounded (2 s); a wait that gives up is
// counted, the CTA drains its copies and products and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include "intlora_device.cuh"
#include "intlora_kernels.h"
#include "tcgen05_util.cuh"

namespace intlora {

namespace {

using namespace tc;

constexpr double kLn2 = 0.69314718055994530942;
#ifndef INTLORA_MTC_QUANT_WARPS
#define INTLORA_MTC_QUANT_WARPS 12
#endif
constexpr int kQuantWarps = INTLORA_MTC_QUANT_WARPS;   // a multiple of 4: kMembers warps per lane quarter
static_assert(kQuantWarps % 4 == 0 && kQuantWarps >= 4 && kQuantWarps <= 16, "quantizer warps: 4, 8, 12 or 16");
constexpr int kMembers = kQuantWarps / 4;
constexpr int kQuantThreads = 32 * kQuantWarps;
constexpr int kMtcThreads = 32 * (4 + kQuantWarps);
constexpr int kRows = 128;                               // rows per unit = tensor-memory lanes
constexpr uint32_t kPartCols = 128;                      // columns per MMA (N) and per hand-off
constexpr int kMaxParts = 4;
constexpr uint32_t kABytes = kRows * 128;                // one tf32 part of one K atom of A (16 KB)
constexpr uint32_t kBPart = kPartCols * 128;             // one tf32 part of a B^T stage (16 KB)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxMtcJobs = 32;
constexpr uint32_t kOutStage = 2048;                     // one 32 x 16 output block (int32), 1 KB aligned
#ifndef INTLORA_MTC_GATHER
#define INTLORA_MTC_GATHER 2
#endif
constexpr int kGather = INTLORA_MTC_GATHER;              // exchange slots in flight per thread

__device__ unsigned int g_mtc_timeouts;

// Every wait of this kernel sleeps between checks: a waiting warp (the TMA
// and MMA threads wait most of the time) takes no issue slots from the
// quantizer warps that share its scheduler.
__device__ __forceinline__ bool wait_m(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait_sleep(bar, parity, abort_flag, &g_mtc_timeouts);
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

struct alignas(64) MtcLayerDev {
  CUtensorMap a_hi, a_lo;        // {kp, d}, box {32, 128}, 128B swizzle
  CUtensorMap b_hi, b_lo;        // {kp, n}, box {32, 128}, 128B swizzle
  CUtensorMap out_map;           // {n, d} of P or M, box {16, 32}, swizzle = row bytes (16 B: none)
  const uint8_t* codes;
  int64_t ld_w;
  const float* s;
  const int32_t* z;
  const double* sigma_w;
  const double* sigma_r;
  void* out;
  float* scale_out;
  int32_t* zero_out;
  uint8_t* code_out;
  int64_t d, n;
  int64_t unit_begin;
  float alpha;
  uint32_t stream_id;
  int32_t atoms;                 // kp / 32
  int32_t pad;
};
struct MtcBatch {
  MtcLayerDev layer[kMaxMtcJobs];
  uint64_t* slots;               // [groups][2][G][128] tagged row extrema (zeroed before the launch)
  int32_t count;
  uint32_t key0, key1;
  int32_t bits;                  // MUL: u_bits; SHIFT: shift_bits
  int32_t group;                 // G
  int32_t slice;                 // S: columns per CTA (multiple of 32, <= 512)
  int32_t atoms_max;
  int32_t stages;
  int32_t obufs;                 // output staging blocks per quantizer warp (2, or 1 at rank > 64)
  int32_t num_groups;
  int64_t total_units;
};

// ---- small PTX helpers ---------------------------------------------------------
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float v[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// kind::tf32, fp32 D, both operands K-major, M = 128, N columns.
__device__ __forceinline__ uint32_t idesc_tf32(uint32_t n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

// Exchange area accesses, L2-coherent (another SM wrote them). A slot is one
// 64-bit word: the row maximum and negated minimum as |value| bit patterns
// (31 bits each) and a 2-bit tag. An aligned 64-bit access is single-copy
// atomic, so a word whose tag matches carries its own values and no fence or
// flag is needed to publish it.
__device__ __forceinline__ uint64_t slot_word(uint32_t top, uint32_t negb, uint32_t tag) {
  return (static_cast<uint64_t>(top) << 33) | (static_cast<uint64_t>(negb) << 2) | tag;
}
__device__ __forceinline__ void st_slot(uint64_t* p, uint64_t w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_slot(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

__device__ __forceinline__ uint32_t ord_abs(float v) { return __float_as_uint(fabsf(v)); }

// 16 codes of one row from global memory (read-only path): 8-bit codes are
// 16 bytes, 4-bit codes 8 bytes (even column in the low nibble).
template <int WBITS>
__device__ __forceinline__ uint4 load_codes16(const uint8_t* p) {
  if (WBITS == 8) return __ldg(reinterpret_cast<const uint4*>(p));
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  return make_uint4(v.x, v.y, 0u, 0u);
}
template <int WBITS>
__device__ __forceinline__ int32_t code_at(const uint4& c, int k) {
  if (WBITS == 8) {
    // byte k & 3 of the word, zero-extended (one byte permute)
    const uint32_t w = k < 4 ? c.x : k < 8 ? c.y : k < 12 ? c.z : c.w;
    return static_cast<int32_t>(__byte_perm(w, 0u, 0x4440u | static_cast<uint32_t>(k & 3)));
  }
  const uint32_t w = k < 8 ? c.x : c.y;
  return static_cast<int32_t>((w >> (4 * (k & 7))) & 0xFu);
}

struct Unit {
  int li;
  int64_t i0;
};
__device__ __forceinline__ Unit unit_of(const MtcBatch& b, int64_t u) {
  int j = 0;
  while (j + 1 < b.count && b.layer[j + 1].unit_begin <= u) ++j;
  Unit x;
  x.li = j;
  x.i0 = (u - b.layer[j].unit_begin) * kRows;
  return x;
}

// CODE: some layer of the launch asks for the U codes as well (code_out);
// the instantiation without it forms no code bytes at all.
template <int VARIANT, int WBITS, int OUTB, bool CODE>
__global__ void __launch_bounds__(kMtcThreads, 1) merge_tc_kernel(const __grid_constant__ MtcBatch b) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t{1023});
  const int S = b.slice;
  const int NP = (S + static_cast<int>(kPartCols) - 1) / static_cast<int>(kPartCols);
  const int NS = b.stages;
  const int G = b.group;
  uint8_t* sA = base;                                                   // [atom][hi, lo]
  uint8_t* sB = sA + static_cast<size_t>(b.atoms_max) * 2 * kABytes;  // [stage][hi, lo]
  uint8_t* ostage = sB + static_cast<size_t>(NS) * 2 * kBPart;           // [quantizer warp][2] output blocks
  uint2* ext = reinterpret_cast<uint2*>(ostage + static_cast<size_t>(kQuantWarps) * b.obufs * kOutStage);   // [kMembers][128]
  float* rcp_tab = reinterpret_cast<float*>(ext + 2 * kMembers * kRows);   // 1/D, D in [-255, 255]; ext, then gat
  uint64_t* bars = reinterpret_cast<uint64_t*>(rcp_tab + 512);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* ext_bar = bars + 2;            // the quantizers' partial extrema are in ext
  uint64_t* got_bar = bars + 4;            // every member's share of the group's extrema is in gat
  uint64_t* drain = bars + 5;
  uint64_t* t_full = bars + 6;             // [kMaxParts]
  uint64_t* t_empty = t_full + kMaxParts;  // [kMaxParts]
  uint64_t* b_full = t_empty + kMaxParts;  // [NS]
  uint64_t* b_empty = b_full + NS;         // [NS]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = static_cast<int>(blockIdx.x) / G;
  const int rank = static_cast<int>(blockIdx.x) - grp * G;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    mbar_init(ext_bar, kQuantThreads);
    mbar_init(got_bar, kQuantThreads);
    mbar_init(drain, 1);
    for (int p = 0; p < kMaxParts; ++p) {
      mbar_init(&t_full[p], 1);
      mbar_init(&t_empty[p], kQuantThreads);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp >= 4)
    for (int k = threadIdx.x - 128; k < 511; k += kQuantThreads)
      rcp_tab[k] = (k == 255) ? 0.0f : __frcp_rn(static_cast<float>(k - 255));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0, ucount = 0;
      uint32_t sph = 0;
      // parity of the last phase armed on each barrier (-1: never armed), so
      // that an aborted CTA can wait for its copies in flight
      int armed_b[4] = {-1, -1, -1, -1};
      int armed_a = -1;
      for (int64_t u = grp; u < b.total_units && !abort_flag; u += b.num_groups, ++ucount) {
        const Unit x = unit_of(b, u);
        const MtcLayerDev& L = b.layer[x.li];
        if (!wait_m(a_empty, (static_cast<uint32_t>(ucount) & 1u) ^ 1u, &abort_flag)) break;
        mbar_arrive_tx(a_full, static_cast<uint32_t>(L.atoms) * 2u * kABytes);
        armed_a = ucount & 1;
        const int32_t y0 = static_cast<int32_t>(x.i0);
        for (int a = 0; a < L.atoms; ++a) {
          uint8_t* dst = sA + static_cast<size_t>(2 * a) * kABytes;
          tma_load_2d(dst, &L.a_hi, a * 32, y0, a_full);
          tma_load_2d(dst + kABytes, &L.a_lo, a * 32, y0, a_full);
        }
        bool ok = true;
        for (int p = 0; p < NP && ok; ++p)
          for (int a = 0; a < L.atoms; ++a) {
            if (!wait_m(&b_empty[stage], sph ^ 1u, &abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_tx(&b_full[stage], 2u * kBPart);
            armed_b[stage] = static_cast<int>(sph);
            const int32_t y = static_cast<int32_t>(static_cast<int64_t>(rank) * S + p * static_cast<int>(kPartCols));
            uint8_t* dst = sB + static_cast<size_t>(stage) * 2 * kBPart;
            tma_load_2d(dst, &L.b_hi, a * 32, y, &b_full[stage]);
            tma_load_2d(dst + kBPart, &L.b_lo, a * 32, y, &b_full[stage]);
            if (++stage == NS) {
              stage = 0;
              sph ^= 1u;
            }
          }
        if (!ok) break;
      }
      if (abort_flag) {
        // every copy this thread started lands before the CTA goes away: the
        // last phase armed on each barrier completes when its bytes arrive
        for (int s = 0; s < NS; ++s) {
          if (armed_b[s] < 0) continue;
          const uint64_t t0 = global_ns();
          while (!mbar_try(&b_full[s], static_cast<uint32_t>(armed_b[s])) && global_ns() - t0 < kWaitNs) {
          }
        }
        if (armed_a >= 0) {
          const uint64_t t0 = global_ns();
          while (!mbar_try(a_full, static_cast<uint32_t>(armed_a)) && global_ns() - t0 < kWaitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0, ucount = 0;
      uint32_t sph = 0;
      for (int64_t u = grp; u < b.total_units && !abort_flag; u += b.num_groups, ++ucount) {
        const Unit x = unit_of(b, u);
        const int atoms = b.layer[x.li].atoms;
        const uint32_t up = static_cast<uint32_t>(ucount) & 1u;
        if (!wait_m(a_full, up, &abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int p = 0; p < NP && ok; ++p) {
          // the quantizers have read this part of the last unit
          if (!wait_m(&t_empty[p], up ^ 1u, &abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ncols = static_cast<uint32_t>(min(static_cast<int>(kPartCols), S - p * static_cast<int>(kPartCols)));
          const uint32_t idesc = idesc_tf32(ncols);
          const uint32_t dt = tmem + static_cast<uint32_t>(p) * kPartCols;
          for (int a = 0; a < atoms; ++a) {
            if (!wait_m(&b_full[stage], sph, &abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint8_t* ar = sA + static_cast<size_t>(2 * a) * kABytes;
            const uint64_t ahi = kmajor_desc(smem_u32(ar));
            const uint64_t alo = kmajor_desc(smem_u32(ar + kABytes));
            const uint8_t* br = sB + static_cast<size_t>(stage) * 2 * kBPart;
            const uint64_t bhi = kmajor_desc(smem_u32(br));
            const uint64_t blo = kmajor_desc(smem_u32(br + kBPart));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t off = static_cast<uint64_t>(ks * 2);       // 32 bytes of K per step
              mma_tf32(dt, ahi + off, bhi + off, idesc, (a == 0 && ks == 0) ? 0u : 1u);
              mma_tf32(dt, ahi + off, blo + off, idesc, 1u);
              mma_tf32(dt, alo + off, bhi + off, idesc, 1u);
            }
            tc_commit(&b_empty[stage]);
            if (++stage == NS) {
              stage = 0;
              sph ^= 1u;
            }
          }
          if (ok) tc_commit(&t_full[p]);
        }
        if (!ok) break;
        tc_commit(a_empty);
      }
      if (abort_flag) {
        // every product issued so far completes before tensor memory is freed
        tc_commit(drain);
        const uint64_t t0 = global_ns();
        while (!mbar_try(drain, 0u) && global_ns() - t0 < kWaitNs) {
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------- quantizers: lane i of quarter q = row 32 q + i of the unit
    const int quarter = warp & 3;
    const int member = (warp - 4) >> 2;            // 0 .. kMembers - 1: every kMembers-th 16-column group
    const int row_u = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int qmax = (1 << b.bits) - 1;
    const bool sender = member == 0;
    uint64_t* my_slots = b.slots + static_cast<int64_t>(grp) * 2 * G * kRows;
    uint2* gat = ext + kMembers * kRows;           // [kMembers][128] partial group extrema
    int cur = -1, ucount = 0;
    uint32_t nstore = 0;                           // output blocks this warp has sent
    float c_ln2 = 0.0f;
    PhiloxSmall ph{};
    for (int64_t u = grp; u < b.total_units && !abort_flag; u += b.num_groups, ++ucount) {
      const Unit x = unit_of(b, u);
      const MtcLayerDev& L = b.layer[x.li];
      if (x.li != cur) {
        const double c = pow(*L.sigma_w / *L.sigma_r, static_cast<double>(L.alpha));
        c_ln2 = static_cast<float>(c * kLn2);
        ph = philox_small_setup(L.stream_id, b.key0, b.key1);
        cur = x.li;
      }
      const uint32_t up = static_cast<uint32_t>(ucount) & 1u;
      const int64_t n = L.n;
      const int64_t row = x.i0 + row_u;
      const bool valid = row < L.d;
      const int64_t rrow = valid ? row : L.d - 1;         // clamped for loads
      const int64_t col0 = static_cast<int64_t>(rank) * S;
      const int cols = col0 < n ? static_cast<int>(min64(S, n - col0)) : 0;   // multiple of 32
      const float sv = __ldg(L.s + rrow);
      const int32_t zv = clamp_i(__ldg(L.z + rrow), 0, (1 << WBITS) - 1);
      const uint32_t rb = smem_u32(rcp_tab) + 4u * static_cast<uint32_t>(255 - zv);   // 1/(code - z) at rb + 4 code
      const uint8_t* crow = L.codes + rrow * L.ld_w;
      const uint32_t ctr_row = static_cast<uint32_t>(rrow * (n >> 2));
      const uint64_t s2 = f2_pack(sv, sv);

      // this thread's next code row into L2 (the group's next unit)
      {
        const int64_t un = u + b.num_groups;
        if (un < b.total_units) {
          const Unit y = unit_of(b, un);
          const MtcLayerDev& L2 = b.layer[y.li];
          const int64_t nrow = y.i0 + row_u;
          const int64_t ncol0 = static_cast<int64_t>(rank) * S;
          if (nrow < L2.d && ncol0 < L2.n) {
            const int64_t bytes = (min64(S, L2.n - ncol0) * WBITS) >> 3;
            const uint8_t* q = L2.codes + nrow * L2.ld_w + ((ncol0 * WBITS) >> 3);
            for (int64_t o = member * 128; o < bytes; o += 128 * kMembers) prefetch_l2(q + o);
          }
        }
      }

      // ---- phase A: T -> U, row extrema, U parked in tensor memory
      // This thread's 16-column groups are g = 0 .. ng - 1 at slice column
      // 16 (kMembers g + member), in part order; each group's codes are
      // loaded two groups ahead (the loads are the longest latency of the loop).
      constexpr int kStep = 16 * kMembers;                      // columns between a thread's groups
      const int ng = (cols >> 4) > member ? ((cols >> 4) - member + kMembers - 1) / kMembers : 0;
      float hi = 0.0f, lo = 0.0f;
      bool ok = true;
      {
        uint4 cw0 = make_uint4(0u, 0u, 0u, 0u), cw1 = cw0;
        if (ng > 0) cw0 = load_codes16<WBITS>(crow + (((col0 + 16 * member) * WBITS) >> 3));
        if (ng > 1) cw1 = load_codes16<WBITS>(crow + (((col0 + kStep + 16 * member) * WBITS) >> 3));
        int have_part = -1;
        for (int g = 0; g < ng; ++g) {
          const int cc = kStep * g + 16 * member;              // column in the slice
          const int p = cc >> 7;
          if (p != have_part) {
            if (!wait_m(&t_full[p], up, &abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            have_part = p;
          }
          const int64_t j = col0 + cc;
          const uint4 cw = cw0;
          cw0 = cw1;
          if (g + 2 < ng) cw1 = load_codes16<WBITS>(crow + (((j + 2 * kStep) * WBITS) >> 3));
          float v[16];
          tmem_ld16(tmem + lane_base + static_cast<uint32_t>(cc), v);
          tmem_ld_wait();
          const uint32_t blk = ctr_row + static_cast<uint32_t>(j >> 2);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w4 = philox10_small(blk + static_cast<uint32_t>(q), ph);
            const uint32_t words[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t wa = words[2 * h], wb = words[2 * h + 1];
              const int k0 = 4 * q + 2 * h;
              const uint64_t lg = laplace_log2_x2(wa, wb);
              const uint64_t cs = f2_pack(laplace_sign(wa, c_ln2), laplace_sign(wb, c_ln2));
              const float r0 = ld_shared_f32(rb + 4u * static_cast<uint32_t>(code_at<WBITS>(cw, k0)));
              const float r1 = ld_shared_f32(rb + 4u * static_cast<uint32_t>(code_at<WBITS>(cw, k0 + 1)));
              const uint64_t vp = f2_fma(f2_fma(lg, cs, f2_pack(v[k0], v[k0 + 1])), f2_pack(r0, r1), s2);
              v[k0] = f2_lo(vp);
              v[k0 + 1] = f2_hi(vp);
            }
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (VARIANT == kShift) {
              hi = fmaxf(hi, fabsf(v[k]));
            } else {
              hi = fmaxf(hi, v[k]);
              lo = fminf(lo, v[k]);
            }
          }
          tmem_st16(tmem + lane_base + static_cast<uint32_t>(cc), v);
        }
      }
      tmem_st_wait();
      if (!valid) hi = lo = 0.0f;

      // ---- row extrema: the members of this CTA, then the group
      ext[member * kRows + row_u] = make_uint2(ord_abs(hi), ord_abs(lo));
      mbar_arrive(ext_bar);
      if (!wait_m(ext_bar, up, &abort_flag) || !ok) break;
      // this CTA's extrema of the row (every member reads them from ext)
      uint2 own = ext[row_u];
#pragma unroll
      for (int m = 1; m < kMembers; ++m) {
        const uint2 f = ext[m * kRows + row_u];
        own = make_uint2(max(own.x, f.x), max(own.y, f.y));
      }
      // this unit's tag: the slot set (parity) alternates every unit, so the
      // stale word a slot can hold is the unit two back's (other tag) or the
      // launch's zero fill (tag 0)
      const uint32_t want = ((static_cast<uint32_t>(ucount) >> 1) & 1u) + 1u;
      if (sender) st_slot(my_slots + (static_cast<int64_t>(up) * G + rank) * kRows + row_u, slot_word(own.x, own.y, want));
      // member m gathers the other CTAs k = m, m + kMembers, ... of the group,
      // kGather slots in flight at a time; a slot is read again (sleeping
      // between reads, bounded) until it carries this unit's tag
      uint2 part = own;
      {
        const uint64_t* sp = my_slots + static_cast<int64_t>(up) * G * kRows + row_u;
        uint64_t t0 = 0;
        for (int k0 = member; k0 < G && !abort_flag; k0 += kGather * kMembers) {
          uint64_t e[kGather];
#pragma unroll
          for (int i = 0; i < kGather; ++i) {
            const int k = k0 + i * kMembers;
            if (k < G && k != rank) e[i] = ld_slot(sp + static_cast<int64_t>(k) * kRows);
          }
#pragma unroll
          for (int i = 0; i < kGather; ++i) {
            const int k = k0 + i * kMembers;
            if (k >= G || k == rank) continue;
            for (uint32_t it = 1; static_cast<uint32_t>(e[i] & 3u) != want; ++it) {
              __nanosleep(64);
              e[i] = ld_slot(sp + static_cast<int64_t>(k) * kRows);
              if ((it & 63u) == 0u) {
                if (t0 == 0) {
                  t0 = global_ns();
                } else if (global_ns() - t0 > kWaitNs) {
                  atomicAdd(&g_mtc_timeouts, 1u);
                  abort_flag = 1;
                }
                if (abort_flag) break;
              }
            }
            part = make_uint2(max(part.x, static_cast<uint32_t>(e[i] >> 33)),
                              max(part.y, static_cast<uint32_t>(e[i] >> 2) & 0x7FFFFFFFu));
          }
        }
      }
      gat[member * kRows + row_u] = part;
      mbar_arrive(got_bar);
      if (!wait_m(got_bar, up, &abort_flag) || abort_flag) break;
      uint32_t top_b = part.x, negb_b = part.y;
#pragma unroll
      for (int m = 0; m < kMembers; ++m) {
        const uint2 f = gat[m * kRows + row_u];
        top_b = max(top_b, f.x);
        negb_b = max(negb_b, f.y);
      }
      const float top = __uint_as_float(top_b), neg_bottom = __uint_as_float(negb_b);
      float scale = 1.0f;
      int32_t zero = 0;
      if (VARIANT == kShift) {
        scale = top > 0.0f ? top : 1.0f;
      } else {
        scale = __fdiv_rn(top + neg_bottom, static_cast<float>(qmax));
        if (scale > 0.0f) zero = clamp_i(static_cast<int32_t>(rintf(__fdiv_rn(neg_bottom, scale))), 0, qmax);
        else scale = 1.0f;
      }
      const float inv = __frcp_rn(scale);
      if (rank == 0 && sender && valid) {
        if (L.scale_out != nullptr) L.scale_out[row] = scale;
        if (VARIANT == kMul && L.zero_out != nullptr) L.zero_out[row] = zero;
      }

      // ---- phase B: quantize the parked U and store the row's merged weights
      const int32_t bias_lo = kRoundBiasBits - zero;
      const int32_t bias_hi = bias_lo + qmax;
      // Each part in turn: this thread's groups of the part (16-column groups
      // 16 member + kStep i), their codes loaded one part ahead; the part of
      // tensor memory goes back to the MMA issuer once they have been read.
      constexpr int kGpp = (static_cast<int>(kPartCols) / 16 + kMembers - 1) / kMembers;   // groups per part, at most
      uint4 cwn[kGpp];
      auto load_part = [&](int p) {
        const int pc = min(static_cast<int>(kPartCols), cols - p * static_cast<int>(kPartCols));
#pragma unroll
        for (int i = 0; i < kGpp; ++i) {
          const int c = 16 * member + kStep * i;
          cwn[i] = c < pc ? load_codes16<WBITS>(crow + (((col0 + p * static_cast<int>(kPartCols) + c) * WBITS) >> 3))
                          : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      if (NP > 0) load_part(0);
      for (int p = 0; p < NP; ++p) {
        uint4 cwc[kGpp];
#pragma unroll
        for (int i = 0; i < kGpp; ++i) cwc[i] = cwn[i];
        if (p + 1 < NP) load_part(p + 1);
        const int pc = min(static_cast<int>(kPartCols), cols - p * static_cast<int>(kPartCols));
#pragma unroll
        for (int i = 0; i < kGpp; ++i) {
          const int c = 16 * member + kStep * i;
          if (c >= pc) break;
          const int cc = p * static_cast<int>(kPartCols) + c;
          const int64_t j = col0 + cc;
          const uint4 cw = cwc[i];
          float v[16];
          tmem_ld16(tmem + lane_base + static_cast<uint32_t>(cc), v);
          tmem_ld_wait();
          int32_t res[16];
          uint32_t code8[CODE ? 16 : 1];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int32_t dcode = code_at<WBITS>(cw, k) - zv;
            if (VARIANT == kShift) {
              const float vn = v[k] * inv;
              const int32_t sh = clamp_i(neg_log2_round(vn), 0, qmax);
              const int32_t sgn = vn > 0.0f ? 1 : (vn < 0.0f ? -1 : 0);
              res[k] = sgn * (dcode >> sh);
              if (CODE) code8[CODE ? k : 0] = static_cast<uint32_t>(sh);
            } else {
              // biased rounding word clamped to the code range, bias taken off after
              const int32_t cb = clamp_i(__float_as_int(fmaf(v[k], inv, kRoundBias)), bias_lo, bias_hi);
              res[k] = (cb - kRoundBiasBits) * dcode;
              if (CODE) code8[CODE ? k : 0] = static_cast<uint32_t>(cb - bias_lo);
            }
          }
          if (OUTB == 1) {
            // 16 bytes per row and group: one direct store per lane
            if (valid) {
              uint32_t wv[4];
#pragma unroll
              for (int q = 0; q < 4; ++q)
                wv[q] = (static_cast<uint32_t>(res[4 * q]) & 0xFFu) | ((static_cast<uint32_t>(res[4 * q + 1]) & 0xFFu) << 8) |
                        ((static_cast<uint32_t>(res[4 * q + 2]) & 0xFFu) << 16) | (static_cast<uint32_t>(res[4 * q + 3]) << 24);
              *reinterpret_cast<uint4*>(static_cast<uint8_t*>(L.out) + row * n + j) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          } else {
            // the warp's 32 rows x 16 columns go out as one TMA store through a
            // swizzled staging block (double-buffered when shared memory
            // allows), one whole 32- or 64-byte segment per row
            const bool two = b.obufs == 2;
            uint8_t* stage = ostage + static_cast<size_t>(warp - 4) * b.obufs * kOutStage + (two ? (nstore & 1u) : 0u) * kOutStage;
            if (lane == 0) {                         // this block's last store has read it
              if (two) bulk_wait_read<1>();
              else bulk_wait_read<0>();
            }
            __syncwarp();
            const uint32_t rowp = smem_u32(stage) + static_cast<uint32_t>(lane) * (16u * OUTB);
            if (OUTB == 4) {
              const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);     // 64-byte swizzle
#pragma unroll
              for (int q = 0; q < 4; ++q)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                             ::"r"(rowp + 16u * (static_cast<uint32_t>(q) ^ sw)), "r"(res[4 * q]), "r"(res[4 * q + 1]),
                               "r"(res[4 * q + 2]), "r"(res[4 * q + 3])
                             : "memory");
            } else {
              uint32_t wv[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                wv[q] = (static_cast<uint32_t>(res[2 * q]) & 0xFFFFu) | (static_cast<uint32_t>(res[2 * q + 1]) << 16);
              const uint32_t sw = static_cast<uint32_t>((lane >> 2) & 1);     // 32-byte swizzle
#pragma unroll
              for (int q = 0; q < 2; ++q)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                             ::"r"(rowp + 16u * (static_cast<uint32_t>(q) ^ sw)), "r"(wv[4 * q]), "r"(wv[4 * q + 1]),
                               "r"(wv[4 * q + 2]), "r"(wv[4 * q + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              // rows past d are clipped by the tensor map
              tma_store_2d(&L.out_map, stage, static_cast<int32_t>(j), static_cast<int32_t>(x.i0 + quarter * 32));
              bulk_commit();
            }
            ++nstore;
          }
          if (CODE && valid) {
            if (L.code_out != nullptr) {
              uint32_t cv[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int k0 = CODE ? 4 * q : 0;
                cv[q] = code8[k0] | (code8[k0 + (CODE ? 1 : 0)] << 8) | (code8[k0 + (CODE ? 2 : 0)] << 16) |
                        (code8[k0 + (CODE ? 3 : 0)] << 24);
              }
              *reinterpret_cast<uint4*>(L.code_out + row * n + j) = make_uint4(cv[0], cv[1], cv[2], cv[3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&t_empty[p]);
      }
    }
    if (lane == 0) bulk_wait<0>();                 // this warp's output stores are done
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Dynamic shared memory of a launch. At least 120 KB, so that two CTAs never
// share an SM: each allocates all 512 tensor-memory columns.
int mtc_obufs(int atoms_max) { return atoms_max > 2 ? 1 : 2; }

size_t mtc_smem_bytes(int atoms_max, int stages) {
  const size_t need = 1024 + static_cast<size_t>(atoms_max) * 2 * kABytes + static_cast<size_t>(stages) * 2 * kBPart +
                      static_cast<size_t>(kQuantWarps) * mtc_obufs(atoms_max) * kOutStage + 2 * kMembers * kRows * 8 +
                      512 * 4 + (6 + 2 * kMaxParts + 2 * stages) * 8;
  return need < 120 * 1024 ? 120 * 1024 : need;
}

int mtc_stages(int atoms_max) {
  for (int st = 4; st >= 2; --st)
    if (mtc_smem_bytes(atoms_max, st) <= 227 * 1024) return st;
  return 0;
}

int mtc_atoms(int32_t r) { return r <= 32 ? 1 : (r <= 64 ? 2 : 4); }

template <int VARIANT, int WBITS, int OUTB, bool CODE>
struct MtcLaunch {
  static constexpr auto kernel() { return merge_tc_kernel<VARIANT, WBITS, OUTB, CODE>; }
  static int blocks_per_sm(size_t smem) {
    if (cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel(), kMtcThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return per_sm;
  }
  static cudaError_t launch(const MtcBatch& b, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(kernel(), cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(b.num_groups * b.group));
    cfg.blockDim = dim3(kMtcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;     // every CTA resident: group members wait on one another
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return counted(cudaLaunchKernelEx(&cfg, kernel(), b));
  }
};

struct MtcQuery {
  int op;              // 0 launch, 1 CTAs per SM
  size_t smem;
  const MtcBatch* batch;
  cudaStream_t stream;
  int result;
  cudaError_t err;
};
template <int VARIANT, int WBITS, int OUTB>
void mtc_run(MtcQuery& q, bool code) {
  if (code) {
    using T = MtcLaunch<VARIANT, WBITS, OUTB, true>;
    if (q.op == 0) q.err = T::launch(*q.batch, q.smem, q.stream);
    else q.result = T::blocks_per_sm(q.smem);
  } else {
    using T = MtcLaunch<VARIANT, WBITS, OUTB, false>;
    if (q.op == 0) q.err = T::launch(*q.batch, q.smem, q.stream);
    else q.result = T::blocks_per_sm(q.smem);
  }
}
bool mtc_dispatch(MtcQuery& q, int variant, int w_bits, int out_bytes, bool code) {
  if (variant == kMul) {
    if (w_bits == 8 && out_bytes == 4) mtc_run<kMul, 8, 4>(q, code);
    else if (w_bits == 8 && out_bytes == 2) mtc_run<kMul, 8, 2>(q, code);
    else if (w_bits == 4 && out_bytes == 2) mtc_run<kMul, 4, 2>(q, code);
    else return false;
  } else {
    if (w_bits == 4 && out_bytes == 1) mtc_run<kShift, 4, 1>(q, code);
    else if (w_bits == 8 && out_bytes == 2) mtc_run<kShift, 8, 2>(q, code);
    else return false;
  }
  return true;
}

int num_sms() {
  static std::atomic<int> cached{0};
  int v = cached.load();
  if (v == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cached.store(v);
  }
  return v;
}

}  // namespace

int64_t merge_tc_kp(int32_t r) { return 32 * mtc_atoms(r); }

bool merge_tc_plan(int64_t n, int32_t r, MtcPlan* plan) {
  if (r < 1 || r > kMergeTcMaxRank || n % 32 != 0 || n < 32) return false;
  const int64_t g = (n + kTmemCols - 1) / kTmemCols;
  if (g > kMergeTcMaxGroup) return false;
  int64_t slice = (n + g - 1) / g;
  slice = (slice + 31) / 32 * 32;
  plan->group = static_cast<int>(g);
  plan->slice = static_cast<int32_t>(slice);
  return mtc_stages(mtc_atoms(r)) > 0;
}

size_t merge_tc_exchange_bytes() {
  // the double-buffered tagged row extrema of up to kMergeTcMaxCtas CTAs
  return static_cast<size_t>(kMergeTcMaxCtas) * 2 * kRows * sizeof(uint64_t);
}

cudaError_t launch_merge_tc(const MtcJob* jobs, int count, int variant, int w_bits, int out_bytes, int bits,
                            uint32_t key0, uint32_t key1, const MtcPlan& plan, void* exchange, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  static thread_local MtcBatch b;
  const int G = plan.group;
  for (int k0 = 0; k0 < count; k0 += kMaxMtcJobs) {
    const int m = count - k0 < kMaxMtcJobs ? count - k0 : kMaxMtcJobs;
    std::memset(&b, 0, sizeof b);
    int atoms_max = 1;
    int64_t units = 0;
    bool code = false;
    for (int k = 0; k < m; ++k) {
      const MtcJob& j = jobs[k0 + k];
      MtcLayerDev& t = b.layer[k];
      const int kp = static_cast<int>(j.kp);
      const bool ok = tc::encode_2d(&t.a_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.a_hi, j.d, kp, 32, kRows) &&
                      tc::encode_2d(&t.a_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.a_lo, j.d, kp, 32, kRows) &&
                      tc::encode_2d(&t.b_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.b_hi, j.n, kp, 32, kPartCols) &&
                      tc::encode_2d(&t.b_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, j.b_lo, j.n, kp, 32, kPartCols);
      const CUtensorMapDataType odt = out_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                      : out_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
      const CUtensorMapSwizzle osw = out_bytes == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                     : out_bytes == 2 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE;
      if (!ok || !tc::encode_2d_swz(&t.out_map, odt, out_bytes, j.out, j.d, j.n, 16, 32, osw))
        return cudaErrorInvalidValue;
      t.codes = j.codes;
      t.ld_w = j.ld_w;
      t.s = j.s;
      t.z = j.z;
      t.sigma_w = j.sigma_w;
      t.sigma_r = j.sigma_r;
      t.out = j.out;
      t.scale_out = j.scale_out;
      t.zero_out = j.zero_out;
      t.code_out = j.code_out;
      code = code || j.code_out != nullptr;
      t.d = j.d;
      t.n = j.n;
      t.unit_begin = units;
      t.alpha = j.alpha;
      t.stream_id = j.stream_id;
      t.atoms = kp / 32;
      atoms_max = t.atoms > atoms_max ? t.atoms : atoms_max;
      units += (j.d + kRows - 1) / kRows;
    }
    b.count = m;
    b.key0 = key0;
    b.key1 = key1;
    b.bits = bits;
    b.group = G;
    b.slice = plan.slice;
    b.atoms_max = atoms_max;
    b.stages = mtc_stages(atoms_max);
    b.obufs = mtc_obufs(atoms_max);
    if (b.stages == 0) return cudaErrorInvalidValue;
    b.total_units = units;
    const size_t smem = mtc_smem_bytes(atoms_max, b.stages);
    MtcQuery q{1, smem, nullptr, s, 0, cudaSuccess};
    if (!mtc_dispatch(q, variant, w_bits, out_bytes, code)) return cudaErrorInvalidValue;
    if (q.result < 1) return cudaErrorInvalidConfiguration;
    // one CTA per SM (shared memory and tensor memory allow no more)
    const int64_t fit = std::min<int64_t>(num_sms(), kMergeTcMaxCtas) / G;
    if (fit < 1) return cudaErrorInvalidConfiguration;
    b.num_groups = static_cast<int32_t>(units < fit ? units : fit);
    // tag 0 matches no unit: the slots this launch uses start zeroed
    b.slots = static_cast<uint64_t*>(exchange);
    cudaError_t e = cudaMemsetAsync(b.slots, 0, static_cast<size_t>(b.num_groups) * G * 2 * kRows * sizeof(uint64_t), s);
    if (e != cudaSuccess) return e;
    q.op = 0;
    q.batch = &b;
    mtc_dispatch(q, variant, w_bits, out_bytes, code);
    if (q.err != cudaSuccess) return q.err;
  }
  return cudaSuccess;
}

unsigned int merge_tc_timeouts() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_mtc_timeouts, sizeof v);
  return v;
}

}  // namespace intlora
