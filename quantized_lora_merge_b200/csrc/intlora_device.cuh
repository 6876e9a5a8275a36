// Device-side building blocks of the IntLoRA merge kernels (sm_100a).
//
//  * Philox4x32-10 counter-based generator [Salmon et al., SC'11]: the
//    auxiliary matrix R is regenerated from (seed, stream id, element index)
//    instead of being stored ("R is generated online from distribution
//    statistics and a fixed seed, with no extra storage": IntLoRA paper notes,
//    ICML2025, method section 1, AQS).
//  * Laplace(0,1) by the inverse CDF (the auxiliary law the IntLoRA ablation
//    selects: atlas.scime.ai summary, "Measured effects").
//  * Rounding and order-preserving helpers used by the row quantizers.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace intlora {

// Philox4x32 multipliers and Weyl key increments (published constants of the
// generator).
constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

// Ten rounds of Philox4x32 on counter (c0, c1, c2, c3) under key (k0, k1).
// Each round multiplies words 0 and 2 by the two constants (32x32 -> 64),
// swaps the halves around with words 1 and 3 and the round key, and bumps
// the key by the Weyl increments.
__device__ __forceinline__ uint4 philox10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                          uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * c0;   // one wide multiply each
    const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * c2;
    c0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ (k0 + round * kPhiloxW0);
    c2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ (k1 + round * kPhiloxW1);
    c1 = static_cast<uint32_t>(p1);
    c3 = static_cast<uint32_t>(p0);
  }
  return make_uint4(c0, c1, c2, c3);
}

// Philox4x32-10 for counters (c0, 0, sid, 0) under a fixed key and stream id
// (layers below 2^34 elements): everything that does not depend on c0 is
// formed once per layer. Round 0 multiplies sid (the same for the whole
// layer), so its word-0 output u0 and word-1 output u1 are constants; round 1
// multiplies u0, so its high and low products are constants too. The round
// keys k + r W of rounds 2-9 are formed here as well. Bit-identical to
// philox10(c0, 0, sid, 0, k0, k1).
struct PhiloxSmall {
  uint32_t u0, u1;           // words 0 and 1 after round 0
  uint32_t x1, y1, l1;       // round 1: u1 ^ key0(1), hi(M0 u0) ^ key1(1), lo(M0 u0)
  uint32_t k1;               // key word 1 (round 0)
  uint32_t rk0[8], rk1[8];   // round keys of rounds 2-9: k + r W
};
__device__ __forceinline__ PhiloxSmall philox_small_setup(uint32_t sid, uint32_t k0, uint32_t k1) {
  PhiloxSmall p;
  const uint64_t q = static_cast<uint64_t>(kPhiloxM1) * sid;
  p.u0 = static_cast<uint32_t>(q >> 32) ^ k0;          // c1 = 0
  p.u1 = static_cast<uint32_t>(q);
  const uint64_t h = static_cast<uint64_t>(kPhiloxM0) * p.u0;
  p.x1 = p.u1 ^ (k0 + kPhiloxW0);
  p.y1 = static_cast<uint32_t>(h >> 32) ^ (k1 + kPhiloxW1);
  p.l1 = static_cast<uint32_t>(h);
  p.k1 = k1;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    p.rk0[r] = k0 + static_cast<uint32_t>(r + 2) * kPhiloxW0;
    p.rk1[r] = k1 + static_cast<uint32_t>(r + 2) * kPhiloxW1;
  }
  return p;
}
__device__ __forceinline__ uint4 philox10_small(uint32_t c0, const PhiloxSmall& p) {
  // round 0: word 2 from the product of c0 (c3 = 0)
  const uint64_t a = static_cast<uint64_t>(kPhiloxM0) * c0;
  const uint32_t c2 = static_cast<uint32_t>(a >> 32) ^ p.k1;
  const uint32_t c3 = static_cast<uint32_t>(a);
  // round 1: the product of word 0 (= u0) is a layer constant
  const uint64_t b = static_cast<uint64_t>(kPhiloxM1) * c2;
  uint32_t w0 = static_cast<uint32_t>(b >> 32) ^ p.x1;
  uint32_t w1 = static_cast<uint32_t>(b);
  uint32_t w2 = c3 ^ p.y1;
  uint32_t w3 = p.l1;
#pragma unroll
  for (int round = 2; round < 10; ++round) {
    const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * w0;
    const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * w2;
    w0 = static_cast<uint32_t>(p1 >> 32) ^ w1 ^ p.rk0[round - 2];
    w2 = static_cast<uint32_t>(p0 >> 32) ^ w3 ^ p.rk1[round - 2];
    w1 = static_cast<uint32_t>(p1);
    w3 = static_cast<uint32_t>(p0);
  }
  return make_uint4(w0, w1, w2, w3);
}

// Four consecutive words of the auxiliary stream, starting at a flat index
// that is a multiple of 4: block = e / 4, counter (block lo, block hi,
// stream id, 0).
__device__ __forceinline__ uint4 aux_block(uint64_t block, uint32_t stream_id, uint32_t k0,
                                           uint32_t k1) {
  return philox10(static_cast<uint32_t>(block), static_cast<uint32_t>(block >> 32), stream_id,
                  0u, k0, k1);
}

// One word of the auxiliary stream at any flat index (ragged shapes).
__device__ __forceinline__ uint32_t aux_word(uint64_t e, uint32_t stream_id, uint32_t k0,
                                             uint32_t k1) {
  const uint4 w = aux_block(e >> 2, stream_id, k0, k1);
  const uint32_t sel = static_cast<uint32_t>(e & 3u);
  return sel == 0 ? w.x : sel == 1 ? w.y : sel == 2 ? w.z : w.w;
}

// Base-2 logarithm on the special-function unit for a normal, positive
// argument (flush-to-zero form: no denormal guard around the instruction;
// the Laplace argument below is at least 2^-23, so it is never denormal and
// the result is the one the guarded form gives).
__device__ __forceinline__ float lg2_normal(float w) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(w));
  return r;
}

// c * R for the Laplace sample of word x, with c_ln2 = c * ln 2 (fp32).
//
// With k = x >> 9 (23 bits), u = (2k + 1) 2^-24 and v = u - 1/2, the inverse
// CDF gives R = -sign(v) ln(1 - 2|v|). Every step below is exact in fp32:
//   f  = 1 + k 2^-23                     (the bits 0x3F800000 | k, built by one
//                                         funnel shift of 0x7F:x by 9)
//   u2 = 2 f - (2 - 2^-23) = (2k + 1) 2^-23 = 2u
//   w  = 1 - |u2 - 1|      = 1 - 2|v|   (an odd multiple of 2^-23 in (0, 1))
// so log2(w) is taken of the exact argument; the sign of R is that of -v,
// i.e. + exactly when bit 31 of x is clear. Most of the work sits on the FMA
// pipe rather than the integer/logic pipe.
__device__ __forceinline__ float laplace_log2(uint32_t x) {
  const float f = __uint_as_float(__funnelshift_r(x, 0x7Fu, 9));
  const float u2 = fmaf(2.0f, f, -1.99999988079071044921875f);   // -(2 - 2^-23)
  const float w = 1.0f - fabsf(u2 - 1.0f);
  return lg2_normal(w);                                           // log2(1 - 2|v|) < 0
}
// +-c ln2: the factor that turns laplace_log2(x) into c * R.
__device__ __forceinline__ float laplace_sign(uint32_t x, float c_ln2) {
  return __uint_as_float(__float_as_uint(c_ln2) ^ (x & 0x80000000u));
}
__device__ __forceinline__ float laplace_scaled(uint32_t x, float c_ln2) {
  return laplace_log2(x) * laplace_sign(x, c_ln2);
}

// The auxiliary laws the ablation compares with Laplace (IntLoRA summary,
// "Measured effects": Gaussian, Cauchy and Student-t auxiliary matrices),
// read from the same Philox words through u = (2 (x >> 9) + 1) 2^-24:
//   Gaussian: Box-Muller on the word pair (2p, 2p + 1) of a block: radius
//     sqrt(-2 ln u_2p), angle 2 pi u_2p+1; word 2p takes the cosine, word
//     2p + 1 the sine;
//   Cauchy: tan(pi (u - 1/2)) = -cos(pi u) / sin(pi u) (sinpi / cospi keep
//     the argument exact near the poles);
//   Student-t with 2 degrees of freedom: (2u - 1) / sqrt(2 u (1 - u)).
constexpr int kDistLaplace = 0;
constexpr int kDistGaussian = 1;
constexpr int kDistCauchy = 2;
constexpr int kDistStudentT2 = 3;

// u of a word, exactly: 1 + k 2^-23 built from the bits, minus (1 - 2^-24).
__device__ __forceinline__ float unit_from_word(uint32_t x) {
  return __uint_as_float(0x3F800000u | (x >> 9)) - 0.999999940395355224609375f;
}
// R of the element whose word is word `odd` of the pair (w_even, w_odd).
__device__ __forceinline__ float aux_value_generic(int dist, uint32_t w_even, uint32_t w_odd, bool odd) {
  if (dist == kDistGaussian) {
    const float rho = sqrtf(-2.0f * logf(unit_from_word(w_even)));
    const float t = 2.0f * unit_from_word(w_odd);
    return odd ? rho * sinpif(t) : rho * cospif(t);
  }
  const float u = unit_from_word(odd ? w_odd : w_even);
  if (dist == kDistCauchy) return -cospif(u) / sinpif(u);
  return (2.0f * u - 1.0f) / sqrtf(2.0f * u * (1.0f - u));
}

// Packed pairs of fp32 (sm_100 f32x2 instructions): two lanes' worth of
// fma/add/mul per instruction, each half rounded exactly like its scalar
// counterpart (round to nearest even).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v));
}
__device__ __forceinline__ float f2_hi(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Two Laplace log2 values (laplace_log2 of words x and y) with the FMA-pipe
// steps done pairwise; bit-identical to two laplace_log2 calls.
__device__ __forceinline__ uint64_t laplace_log2_x2(uint32_t x, uint32_t y) {
  const uint64_t f = f2_pack(__uint_as_float(__funnelshift_r(x, 0x7Fu, 9)),
                             __uint_as_float(__funnelshift_r(y, 0x7Fu, 9)));
  const uint64_t u2 = f2_fma(f2_pack(2.0f, 2.0f), f, f2_pack(-1.99999988079071044921875f,
                                                           -1.99999988079071044921875f));
  const uint64_t t = f2_add(u2, f2_pack(-1.0f, -1.0f));
  return f2_pack(lg2_normal(1.0f - fabsf(f2_lo(t))), lg2_normal(1.0f - fabsf(f2_hi(t))));
}

// Round to nearest, ties to even, for |x| < 2^22, via the 1.5 * 2^23 bias:
// the fused multiply-add rounds x * inv + bias once, leaving the integer in
// the low mantissa bits.
constexpr float kRoundBias = 12582912.0f;          // 1.5 * 2^23
constexpr int32_t kRoundBiasBits = 0x4B400000;
__device__ __forceinline__ int32_t rne_scaled(float x, float inv) {
  return __float_as_int(fmaf(x, inv, kRoundBias)) - kRoundBiasBits;
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ int32_t clamp_i(int32_t v, int32_t lo, int32_t hi) {
  return min(max(v, lo), hi);
}

// Non-negative floats order like their bit patterns: row maxima of
// non-negative quantities are reduced as unsigned integers.
__device__ __forceinline__ uint32_t nonneg_bits(float v) { return __float_as_uint(fmaxf(v, 0.0f)); }

// Threshold on the fp32 mantissa for "1.f > sqrt(2)": floor((sqrt2 - 1) 2^23).
constexpr uint32_t kSqrt2Mantissa = 0x3504F3u;

// Nearest integer of -log2|v| for 0 < |v| <= 1 (and +large for v = 0 or
// subnormal v), decided exactly on the exponent and mantissa bits: with
// |v| = 2^E * 1.f, -log2|v| = -E - log2(1.f) rounds to -E - 1 exactly when
// 1.f > sqrt(2) (the half-integer threshold of the log domain).
__device__ __forceinline__ int32_t neg_log2_round(float v) {
  const uint32_t a = __float_as_uint(v) & 0x7FFFFFFFu;
  const int32_t e = static_cast<int32_t>(a >> 23) - 127;
  const int32_t up = (a & 0x7FFFFFu) > kSqrt2Mantissa ? 1 : 0;
  return -e - up;
}

__device__ __forceinline__ void warp_sum2(double& a, double& b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
}

// Cluster helpers (inline PTX; sm_90+).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_smem_to_rank(const void* p, uint32_t rank) {
  uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  return remote;
}
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

}  // namespace intlora
