// C ABI of the IntLoRA merge library: host-side validation, launch geometry
// and kernel launches. Every entry point validates all of its arguments before
// enqueuing anything, never synchronizes, and never allocates: scratch space is
// the caller's workspace. See include/intlora.h for the contract.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "intlora.h"
#include "intlora_kernels.h"

using namespace intlora;

// Two-pass tensor-core A B helpers (tgemm_kernels.cu).
namespace intlora {
cudaError_t launch_copy_cols(const float* src, int64_t ld_src, int32_t col0, int32_t cols, int64_t d, float* dst,
                             cudaStream_t s);
cudaError_t launch_add_f32(float* t, const float* t2, int64_t count, cudaStream_t s);
}  // namespace intlora

namespace {

thread_local char g_last_error[512] = "";

intlora_status fail(intlora_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

intlora_status cuda_fail(cudaError_t e, const char* what) {
  return fail(INTLORA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

constexpr int64_t kMaxElements = int64_t{1} << 40;
constexpr int kStatsMaxBlocksPerJob = 148 * 8;

int64_t stats_blocks(int64_t numel) {
  return std::min<int64_t>(kStatsMaxBlocksPerJob, std::max<int64_t>(1, ceil_div(numel, kStatsElementsPerCta)));
}
size_t stats_partial_bytes(int64_t numel) {
  return round256(static_cast<size_t>(stats_blocks(numel)) * kStatsPartialBytes);
}

// ------------------------------------------------------------------------
// tile geometry: cluster size, column slice, rows per tile
// ------------------------------------------------------------------------
int max_active_clusters_cached(int variant, int w_bits, int rank_ct, int out_bytes, bool aligned,
                               int cluster, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, size_t>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(dev, variant * 16 + w_bits, rank_ct, out_bytes, aligned ? 1 : 0,
                                   cluster, smem);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int v = tile_max_active_clusters(variant, w_bits, rank_ct, out_bytes, aligned, cluster, smem);
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = v;
  return v;
}

int slice_cols(int64_t n, int cluster) { return static_cast<int>(ceil_div(ceil_div(n, cluster), 4) * 4); }

// Shared memory an SM offers to `occ` CTAs of the tile kernel (B200: 228 KB
// per SM, 1 KB reserved per CTA, 227 KB per CTA at most).
constexpr int64_t kSmemPerSm = 233472;
constexpr int64_t kSmemPerCtaMax = 232448;
constexpr int kMiscWords = 512 + 8 * kMaxTileRows;

// Geometry of every layer for one (cluster, occupancy) choice. Returns false
// when the slices do not fit. B stays resident when `resident` is asked for.
// *efficiency receives the element-weighted fraction of thread slots that do
// useful work in the item loops (the tile's items spread over kTileThreads).
bool plan_layers(int variant, std::vector<TileLayer>& L, int cluster, int occ, bool resident,
                 TileBatch* b, int64_t* tiles_out, double* efficiency) {
  const int64_t budget_words = (std::min(kSmemPerCtaMax, kSmemPerSm / occ - 1024) - 64) / 4;
  int64_t max_nc = 0, max_b = 0, max_r = 1;
  for (auto& l : L) {
    const int n_c = slice_cols(l.n, cluster);
    max_nc = std::max<int64_t>(max_nc, n_c);
    if (variant != kGen) {
      max_r = std::max<int64_t>(max_r, l.r);
      max_b = std::max<int64_t>(max_b, resident ? int64_t{l.r} * n_c : int64_t{n_c} * std::min(l.r, 8));
    }
  }
  // rows of A a tile may stage: all kMaxTileRows up to rank 32, fewer above
  const int64_t a_rows = variant == kGen ? kMaxTileRows
      : std::min<int64_t>(kMaxTileRows, std::max<int64_t>(kRowsPerItem, (4096 / max_r) / 4 * 4));
  const int64_t free_words = budget_words - max_b - (variant == kGen ? 0 : max_r * a_rows) - kMiscWords;
  // merges stash one code word per 4 tile values next to the tile buffer
  const int64_t u_words = (variant == kGen ? free_words : free_words * 4 / 5) / 16 * 16;
  if (u_words < kRowsPerItem * max_nc) return false;
  int64_t smem_a = 0, tiles = 0;
  double useful = 0.0, total = 0.0;
  for (auto& l : L) {
    const int n_c = slice_cols(l.n, cluster);
    const int64_t quads = n_c / 4;
    int64_t gmax = std::min<int64_t>(u_words / n_c, std::min<int64_t>(kMaxTileRows, a_rows)) / kRowsPerItem;
    gmax = std::max<int64_t>(1, std::min<int64_t>(gmax, ceil_div(l.d, kRowsPerItem)));
    // rows per tile: the item count that fills whole rounds of the block best,
    // then the largest such tile
    int64_t best_g = 1;
    double best_e = -1.0;
    for (int64_t g = 1; g <= gmax; ++g) {
      const int64_t items = g * quads;
      const double e = static_cast<double>(items) / static_cast<double>(ceil_div(items, kTileThreads) * kTileThreads);
      if (e > best_e + 1e-9 || (e > best_e - 1e-9 && g > best_g)) {
        best_e = e;
        best_g = g;
      }
    }
    const int m = static_cast<int>(best_g * kRowsPerItem);
    l.n_c = n_c;
    l.m = m;
    l.aligned = (l.n % 4 == 0) ? 1 : 0;
    if (variant != kGen) {
      l.b_resident = resident ? 1 : 0;
      l.kc = resident ? l.r : static_cast<int>(std::max<int64_t>(1, max_b / n_c));
      smem_a = std::max<int64_t>(smem_a, int64_t{l.r} * m);
    }
    l.tile_begin = tiles;
    const int64_t nt = ceil_div(l.d, m);
    tiles += nt;
    const double numel = static_cast<double>(l.d) * static_cast<double>(l.n);
    useful += numel * best_e * (static_cast<double>(l.d) / static_cast<double>(nt * m));
    total += numel;
  }
  b->smem_u = static_cast<int32_t>(u_words);
  b->smem_b = static_cast<int32_t>(max_b);
  b->smem_a = static_cast<int32_t>(smem_a);
  *tiles_out = tiles;
  if (efficiency) *efficiency = total > 0 ? useful / total : 0.0;
  return true;
}

// ------------------------------------------------------------------------
// team kernels: layers with n % 4 == 0 and n <= kTeamMaxCols
// ------------------------------------------------------------------------
// INTLORA_ROW_KERNEL=tile sends every layer to the row-tile kernels (both
// kernel families stay testable on the same shapes); unset or "auto": the
// team kernels take the layers they support.
bool team_path_enabled() {
  const char* v = std::getenv("INTLORA_ROW_KERNEL");
  return v == nullptr || std::strcmp(v, "tile") != 0;
}

// Base quantization of a row wider than kTeamMaxCols that is a whole number
// of 8-warp sweeps: the team kernel with tensor-memory parking takes it.
bool team_wide(int variant, const TileLayer& l) {
  return variant == kGen && l.n > kTeamMaxCols && l.n <= kTeamWideMaxCols && l.n % (4 * kTeamThreads) == 0;
}

bool team_eligible(int variant, const TileLayer& l) {
  if (l.n % 4 != 0 || (l.n > kTeamMaxCols && !team_wide(variant, l))) return false;
  if (l.d > (int64_t{1} << 24)) return false;      // keeps tile indices of a batch in int32
  if (l.d * l.n >= (int64_t{1} << 34)) return false; // Philox block index fits 32 bits
  if (variant != kGen && l.r > 0 && !aligned16(l.B)) return false;
  if (l.T != nullptr && !aligned16(l.T)) return false;
  return true;
}

// Team width and sweeps of one layer: the most even spread of the row's
// column quads over the team's lanes, then the fewest sweeps (less shared
// memory, more resident CTAs), then the narrower team.
void team_shape(int64_t n, int* tw_out, int* sweeps_out) {
  const int64_t quads = n / 4;
  double best_e = -1.0;
  int best_tw = kTeamWarps, best_s = kTeamMaxSweeps;
  for (int tw = 1; tw <= kTeamWarps; tw *= 2) {
    const int64_t s = ceil_div(quads, int64_t{32} * tw);
    if (s > kTeamMaxSweeps) continue;
    const double e = static_cast<double>(quads) / static_cast<double>(32 * tw * s);
    const bool better = e > best_e + 0.1 || (e > best_e - 0.1 && s < best_s);
    if (better) {
      best_e = std::max(best_e, e);
      best_tw = tw;
      best_s = static_cast<int>(s);
    }
  }
  *tw_out = best_tw;
  *sweeps_out = best_s;
}

int team_ctas_cached(int variant, int w_bits, int rank_ct, int out_bytes, int sweeps_max, bool wide) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, bool>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(dev, variant, w_bits, rank_ct, out_bytes, sweeps_max, wide);
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int v = team_max_active_ctas(variant, w_bits, rank_ct, out_bytes,
                                     team_smem_bytes(variant, sweeps_max), wide);
  std::lock_guard<std::mutex> g(mu);
  cache[key] = v;
  return v;
}

intlora_status launch_team_batch(int variant, const std::vector<TileLayer>& L, int rank_ct, int bits,
                                 int w_bits, int out_bytes, uint64_t seed, cudaStream_t stream, bool wide = false) {
  static thread_local TeamBatch b;
  std::memset(&b, 0, sizeof b);
  int smax = wide ? 0 : 1;
  int64_t tiles = 0;
  std::vector<double> layer_cost(L.size()), tile_cost(L.size());
  std::vector<int64_t> layer_tiles(L.size());
  double total_cost = 0.0;
  for (size_t k = 0; k < L.size(); ++k) {
    const TileLayer& s = L[k];
    TeamLayer& t = b.layer[k];
    t.src = s.src;
    t.ld_src = s.ld_src;
    t.s = s.s;
    t.z = s.z;
    t.A = s.A;
    t.B = s.B;
    t.sigma_w = s.sigma_w;
    t.sigma_r = s.sigma_r;
    t.alpha = s.alpha;
    t.stream_id = s.stream_id;
    t.out = s.out;
    t.ld_out = s.ld_out;
    t.scale_out = s.scale_out;
    t.zero_out = s.zero_out;
    t.code_out = s.code_out;
    t.r_star_out = s.r_star_out;
    t.T = s.T;
    t.d = s.d;
    t.n = s.n;
    t.r = s.r;
    if (wide) {
      // the whole CTA is the team; sweeps past the tensor-memory ones in shared memory
      t.team_warps = kTeamWarps;
      t.sweeps = static_cast<int32_t>(s.n / (4 * kTeamThreads));
      smax = std::max(smax, t.sweeps - kTeamTmemSweeps);
    } else {
      team_shape(s.n, &t.team_warps, &t.sweeps);
      smax = std::max(smax, t.sweeps);
    }
    const int64_t groups = ceil_div(s.d, kTeamRows);
    const int64_t teams = kTeamWarps / t.team_warps;
    t.tile_begin = tiles;
    layer_tiles[k] = ceil_div(groups, teams);
    tiles += layer_tiles[k];
    // cost of a tile: its elements plus a fixed per-row-group overhead
    tile_cost[k] = static_cast<double>(teams) * (kTeamRows * static_cast<double>(s.n) + 512.0);
    layer_cost[k] = tile_cost[k] * static_cast<double>(layer_tiles[k]);
    total_cost += layer_cost[k];
  }
  const int resident = team_ctas_cached(variant, w_bits, rank_ct, out_bytes, smax, wide);
  if (resident <= 0) return fail(INTLORA_ERR_UNSUPPORTED, "team kernel cannot be made resident");
  const int ctas = static_cast<int>(std::min<int64_t>({int64_t{resident}, int64_t{kTeamMaxCtas}, tiles}));
  // contiguous tile ranges of about equal cost, one per CTA
  size_t li = 0;
  double c_acc = 0.0;
  int64_t t_acc = 0;
  for (int k = 0; k < ctas; ++k) {
    const double target = total_cost * static_cast<double>(k) / static_cast<double>(ctas);
    while (li < L.size() && c_acc + layer_cost[li] <= target) {
      c_acc += layer_cost[li];
      t_acc += layer_tiles[li];
      ++li;
    }
    int64_t begin = tiles;
    if (li < L.size())
      begin = t_acc + std::min<int64_t>(layer_tiles[li],
                                        static_cast<int64_t>(std::ceil((target - c_acc) / tile_cost[li] - 1e-9)));
    if (k > 0) begin = std::max<int64_t>(begin, b.cta_begin[k - 1]);
    b.cta_begin[k] = static_cast<int32_t>(begin);
  }
  b.cta_begin[0] = 0;
  b.cta_begin[ctas] = static_cast<int32_t>(tiles);
  b.count = static_cast<int32_t>(L.size());
  b.key0 = static_cast<uint32_t>(seed);
  b.key1 = static_cast<uint32_t>(seed >> 32);
  b.bits = bits;
  b.w_bits = w_bits;
  b.sweeps_max = smax;
  b.tmem_sweeps = wide ? kTeamTmemSweeps : 0;
  b.num_ctas = ctas;
  b.total_tiles = tiles;
  cudaError_t e = launch_team(b, variant, rank_ct, out_bytes, stream);
  if (e != cudaSuccess) return cuda_fail(e, "team kernel launch");
  return INTLORA_OK;
}

intlora_status launch_tile_batch(int variant, std::vector<TileLayer>& L, int bits, int w_bits,
                                 int out_bytes, uint64_t seed, int dist, cudaStream_t stream) {
  // layers whose A B was precomputed run in launches of their own (the
  // kernels' rank-free specialisation)
  bool any_t = false, all_t = true;
  for (auto& l : L) {
    any_t = any_t || l.T != nullptr;
    all_t = all_t && l.T != nullptr;
  }
  if (any_t && !all_t) {
    std::vector<TileLayer> with_t, without;
    for (auto& l : L) (l.T != nullptr ? with_t : without).push_back(l);
    const intlora_status s = launch_tile_batch(variant, with_t, bits, w_bits, out_bytes, seed, dist, stream);
    if (s != INTLORA_OK) return s;
    return launch_tile_batch(variant, without, bits, w_bits, out_bytes, seed, dist, stream);
  }
  // layers the team kernel takes go there (one launch); the rest stay here
  // (the team kernels draw Laplace R only)
  if (team_path_enabled() && dist == INTLORA_DIST_LAPLACE) {
    std::vector<TileLayer> team, rest, wide;
    for (auto& l : L) (team_eligible(variant, l) ? (team_wide(variant, l) ? wide : team) : rest).push_back(l);
    if (!wide.empty()) {
      const intlora_status s = launch_team_batch(variant, wide, 0, bits, w_bits, out_bytes, seed, stream, true);
      if (s != INTLORA_OK) return s;
    }
    if (!team.empty()) {
      int rank_t = 0;
      if (variant != kGen) {
        rank_t = team[0].r;
        for (auto& l : team)
          if (l.r != rank_t) rank_t = 0;
        if (rank_t != 4 && rank_t != 8 && rank_t != 16) rank_t = 0;
        if (all_t) rank_t = -1;
      }
      const intlora_status s = launch_team_batch(variant, team, rank_t, bits, w_bits, out_bytes, seed, stream);
      if (s != INTLORA_OK) return s;
    }
    if (rest.empty()) return INTLORA_OK;
    L = rest;
  }
  int rank_ct = 0;
  if (variant != kGen) {
    rank_ct = L[0].r;
    for (auto& l : L)
      if (l.r != rank_ct) rank_ct = 0;
    if (rank_ct != 4 && rank_ct != 8 && rank_ct != 16) rank_ct = 0;
    if (all_t) rank_ct = -1;
  }
  if (dist != INTLORA_DIST_LAPLACE) rank_ct = -2;    // any rank, another auxiliary law
  bool aligned = true;
  for (auto& l : L) aligned = aligned && (l.n % 4 == 0);
  TileBatch b;
  std::memset(&b, 0, sizeof b);
  static const int kClusters[] = {1, 2, 4, 8, 16};
  bool found = false;
  int64_t total = 0;
  int max_clusters = 0;
  // Prefer B resident, then more CTAs per SM, then the smaller cluster; the
  // rows per tile of each layer are picked for balanced item rounds.
  for (int pass = 0; pass < 2 && !found; ++pass) {
    const bool resident = (pass == 0) || variant == kGen;
    for (int occ = 3; occ >= 1 && !found; --occ) {
      for (int c : kClusters) {
        if (!plan_layers(variant, L, c, occ, resident, &b, &total, nullptr)) continue;
        const size_t smem = tile_smem_bytes(variant, b.smem_u, b.smem_b, b.smem_a);
        max_clusters = max_active_clusters_cached(variant, w_bits, rank_ct, out_bytes, aligned, c, smem);
        if (max_clusters <= 0) continue;
        b.cluster = c;
        found = true;
        break;
      }
    }
  }
  if (!found) return fail(INTLORA_ERR_UNSUPPORTED, "no launchable tile geometry for this batch");
  for (size_t k = 0; k < L.size(); ++k) b.layer[k] = L[k];
  b.count = static_cast<int32_t>(L.size());
  b.variant = variant;
  b.total_tiles = total;
  b.num_clusters = static_cast<int32_t>(std::min<int64_t>(total, max_clusters));
  b.bits = bits;
  b.w_bits = w_bits;
  b.out_bytes = out_bytes;
  b.key0 = static_cast<uint32_t>(seed);
  b.key1 = static_cast<uint32_t>(seed >> 32);
  b.small = 1;
  for (auto& l : L)
    if (l.d * l.n >= (int64_t{1} << 34)) b.small = 0;
  b.dist = dist;
  cudaError_t e = launch_tiles(b, rank_ct, aligned, stream);
  if (e != cudaSuccess) return cuda_fail(e, "row-tile kernel launch");
  return INTLORA_OK;
}

uint32_t lo32(uint64_t v) { return static_cast<uint32_t>(v); }
uint32_t hi32(uint64_t v) { return static_cast<uint32_t>(v >> 32); }

// ------------------------------------------------------------------------
// gen_aux
// ------------------------------------------------------------------------
intlora_status check_aux_job(const intlora_aux_job& j, int idx) {
  if (j.W == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "job %d: W is NULL", idx);
  if (j.d < 1 || j.n < 1) return fail(INTLORA_ERR_INVALID_ARG, "job %d: d and n must be >= 1", idx);
  if (j.d > kMaxElements / j.n) return fail(INTLORA_ERR_INVALID_ARG, "job %d: d*n exceeds 2^40", idx);
  if (j.w_bits != 4 && j.w_bits != 8)
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: w_bits must be 4 or 8", idx);
  if (j.w_bits == 4 && (j.n % 2) != 0)
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: n must be even for 4-bit codes", idx);
  if (!(j.alpha >= 0.0f) || !std::isfinite(j.alpha))
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: alpha must be finite and >= 0", idx);
  if (j.sigma_w_out == nullptr || j.sigma_r_out == nullptr)
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: sigma outputs are required", idx);
  if (j.distribution < INTLORA_DIST_LAPLACE || j.distribution > INTLORA_DIST_STUDENT_T2)
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: distribution must be one of INTLORA_DIST_*", idx);
  if (!aligned16(j.W)) return fail(INTLORA_ERR_INVALID_ARG, "job %d: W must be 16-byte aligned", idx);
  if (j.r_star_out != nullptr && !aligned16(j.r_star_out))
    return fail(INTLORA_ERR_INVALID_ARG, "job %d: r_star_out must be 16-byte aligned", idx);
  if (j.w_round_out != nullptr) {
    const int64_t need = j.w_bits == 8 ? j.n : j.n / 2;
    if (j.ld_w_out < need || j.ld_w_out % 16 != 0)
      return fail(INTLORA_ERR_INVALID_ARG,
                  "job %d: ld_w_out must be >= %lld bytes and a multiple of 16", idx,
                  static_cast<long long>(need));
    if (!aligned16(j.w_round_out))
      return fail(INTLORA_ERR_INVALID_ARG, "job %d: w_round_out must be 16-byte aligned", idx);
    if (j.s_out == nullptr || j.z_out == nullptr)
      return fail(INTLORA_ERR_INVALID_ARG, "job %d: s_out and z_out are required with w_round_out", idx);
  }
  return INTLORA_OK;
}

size_t aux_ws_bytes(const intlora_aux_job* jobs, int32_t count) {
  size_t total = 0;
  for (int32_t k = 0; k < count; ++k) total += stats_partial_bytes(jobs[k].d * jobs[k].n);
  return total;
}

// Indices of `count` items grouped by (seed, auxiliary law), in
// first-appearance order: every launch carries one Philox key (uniform round
// keys) and one law at batch level.
template <typename T>
std::vector<std::vector<int32_t>> group_by_seed(const T* items, int32_t count) {
  std::vector<std::pair<uint64_t, int32_t>> keys;
  std::vector<std::vector<int32_t>> groups;
  for (int32_t k = 0; k < count; ++k) {
    const std::pair<uint64_t, int32_t> key(items[k].seed, items[k].distribution);
    size_t g = 0;
    while (g < keys.size() && keys[g] != key) ++g;
    if (g == keys.size()) {
      keys.push_back(key);
      groups.emplace_back();
    }
    groups[g].push_back(k);
  }
  return groups;
}

// The launches of one chunk of at most kMaxBatch jobs: per seed, statistics,
// finalize and the base quantization (grouped by code width).
intlora_status gen_aux_chunk(const intlora_aux_job* jobs, int32_t count, char* ws, cudaStream_t st) {
  std::vector<size_t> offset(count);
  size_t off = 0;
  for (int32_t k = 0; k < count; ++k) {
    offset[k] = off;
    off += stats_partial_bytes(jobs[k].d * jobs[k].n);
  }
  for (const auto& grp : group_by_seed(jobs, count)) {
    StatsBatch sb;
    std::memset(&sb, 0, sizeof sb);
    int64_t blocks = 0;
    for (size_t q = 0; q < grp.size(); ++q) {
      const intlora_aux_job& j = jobs[grp[q]];
      StatsJob& s = sb.job[q];
      s.W = j.W;
      s.numel = j.d * j.n;
      s.stream_id = j.stream_id;
      s.nblocks = static_cast<int32_t>(stats_blocks(s.numel));
      s.block_begin = blocks;
      s.partial = reinterpret_cast<double*>(ws + offset[grp[q]]);
      s.sigma_w_out = j.sigma_w_out;
      s.sigma_r_out = j.sigma_r_out;
      blocks += s.nblocks;
    }
    sb.count = static_cast<int32_t>(grp.size());
    sb.key0 = lo32(jobs[grp[0]].seed);
    sb.key1 = hi32(jobs[grp[0]].seed);
    sb.dist = jobs[grp[0]].distribution;
    cudaError_t e = launch_stats(sb, blocks, st);
    if (e != cudaSuccess) return cuda_fail(e, "statistics kernel launch");
    e = launch_stats_finalize(sb, st);
    if (e != cudaSuccess) return cuda_fail(e, "statistics finalize launch");

    // base quantization for the jobs that want codes or R*, grouped by w_bits
    for (int wb : {4, 8}) {
      std::vector<TileLayer> L;
      for (int32_t k : grp) {
        const intlora_aux_job& j = jobs[k];
        if (j.w_bits != wb || (j.w_round_out == nullptr && j.r_star_out == nullptr)) continue;
        TileLayer l;
        std::memset(&l, 0, sizeof l);
        l.src = j.W;
        l.ld_src = j.n * 4;
        l.sigma_w = j.sigma_w_out;
        l.sigma_r = j.sigma_r_out;
        l.alpha = j.alpha;
        l.stream_id = j.stream_id;
        l.out = j.w_round_out;
        l.ld_out = j.ld_w_out;
        l.scale_out = j.s_out;
        l.zero_out = j.z_out;
        l.r_star_out = j.r_star_out;
        l.d = j.d;
        l.n = j.n;
        L.push_back(l);
      }
      if (L.empty()) continue;
      const intlora_status s =
          launch_tile_batch(kGen, L, wb, wb, 1, jobs[grp[0]].seed, jobs[grp[0]].distribution, st);
      if (s != INTLORA_OK) return s;
    }
  }
  return INTLORA_OK;
}

// ------------------------------------------------------------------------
// merges
// ------------------------------------------------------------------------
intlora_status check_layer(const intlora_layer* l, int idx) {
  if (l == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "layer %d is NULL", idx);
  if (l->d < 1 || l->n < 1) return fail(INTLORA_ERR_INVALID_ARG, "layer %d: d and n must be >= 1", idx);
  if (l->d > kMaxElements / l->n) return fail(INTLORA_ERR_INVALID_ARG, "layer %d: d*n exceeds 2^40", idx);
  if (l->r < 1 || l->r > INTLORA_MAX_RANK)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: r must be in [1, %d]", idx, INTLORA_MAX_RANK);
  if (l->w_bits != 4 && l->w_bits != 8)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: w_bits must be 4 or 8", idx);
  if (l->w_bits == 4 && (l->n % 2) != 0)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: n must be even for 4-bit codes", idx);
  if (l->w_round == nullptr || l->s == nullptr || l->z == nullptr || l->A == nullptr ||
      l->B == nullptr || l->sigma_w == nullptr)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: w_round, s, z, A, B and sigma_w are required", idx);
  const int64_t need = l->w_bits == 8 ? l->n : l->n / 2;
  if (l->ld_w < need || l->ld_w % 16 != 0)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: ld_w must be >= %lld bytes and a multiple of 16",
                idx, static_cast<long long>(need));
  if (!aligned16(l->w_round)) return fail(INTLORA_ERR_INVALID_ARG, "layer %d: w_round must be 16-byte aligned", idx);
  if (!(l->alpha >= 0.0f) || !std::isfinite(l->alpha))
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: alpha must be finite and >= 0", idx);
  if (l->distribution < INTLORA_DIST_LAPLACE || l->distribution > INTLORA_DIST_STUDENT_T2)
    return fail(INTLORA_ERR_INVALID_ARG, "layer %d: distribution must be one of INTLORA_DIST_*", idx);
  return INTLORA_OK;
}

intlora_status check_out(const intlora_merge_out* o, bool mul, int idx) {
  if (o == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "output %d is NULL", idx);
  if (o->out == nullptr || o->sbar == nullptr)
    return fail(INTLORA_ERR_INVALID_ARG, "output %d: out and sbar are required", idx);
  if (mul && o->zbar == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "output %d: zbar is required for MUL", idx);
  if (!aligned16(o->out) || (o->code != nullptr && !aligned16(o->code)))
    return fail(INTLORA_ERR_INVALID_ARG, "output %d: out and code must be 16-byte aligned", idx);
  return INTLORA_OK;
}

// INTLORA_T_KERNEL=cuda keeps T = A B on the CUDA cores inside the row
// kernels; unset or "auto": ranks in [kTensorTMinRank, kTensorTMaxRank] get T
// from the tensor-core pass.
bool tensor_t_enabled() {
  const char* v = std::getenv("INTLORA_T_KERNEL");
  return v == nullptr || std::strcmp(v, "cuda") != 0;
}
// Ranks in (kTensorTMaxRank, 2 kTensorTMaxRank] take two tensor-core passes
// over the rank (the second product added into T).
constexpr int32_t kTwoPassMaxRank = 2 * kTensorTMaxRank;
bool two_pass_t(const intlora_layer& l) { return l.r > kTensorTMaxRank; }
bool uses_tensor_t(const intlora_layer& l) {
  if (!tensor_t_enabled() || l.distribution != INTLORA_DIST_LAPLACE) return false;
  if (l.r > kTensorTMaxRank && l.r <= kTwoPassMaxRank)
    return t_gemm_supported(l.d, l.n, kTensorTMaxRank);
  return t_gemm_supported(l.d, l.n, l.r);
}
// INTLORA_MERGE_KERNEL=rows keeps every merge on the row kernels (team and
// row-tile kernels, A B on the CUDA cores or from the tensor-core T pass);
// "tc" sends every layer the fused tensor-core kernel takes there, whatever
// its rank; unset or "auto": the fused kernel takes the layers it supports
// from rank kMergeTcAutoMinRank up (below it the CUDA-core FMAs of the team
// kernels cost less than the tensor-core hand-offs), and at any rank the rows
// too wide for the team kernels (the row-tile kernels are slower than the
// fused one there: measured on 4096 x 14336 layers at r = 4 and 8).
constexpr int32_t kMergeTcAutoMinRank = 16;   // measured: the team kernels win at r = 8, the fused kernel at r = 16
int merge_kernel_mode() {
  const char* v = std::getenv("INTLORA_MERGE_KERNEL");
  if (v == nullptr) return 0;
  if (std::strcmp(v, "rows") == 0) return 1;
  if (std::strcmp(v, "tc") == 0) return 2;
  return 0;
}
bool uses_merge_tc(const intlora_layer& l) {
  const int mode = merge_kernel_mode();
  if (mode == 1 || l.distribution != INTLORA_DIST_LAPLACE) return false;
  if (mode == 0 && l.r < kMergeTcAutoMinRank && l.n <= kTeamMaxCols) return false;
  // 32-bit Philox block index and tensor-map extents
  if (l.d * l.n >= (int64_t{1} << 34) || l.d >= (int64_t{1} << 31)) return false;
  MtcPlan plan;
  return merge_tc_plan(l.n, l.r, &plan) && t_gemm_supported(l.d, l.n, kTensorTMinRank);
}

// A call whose workspace does not cover the tensor-core buffers still runs,
// with A B on the CUDA cores (set per call by merge_batched).
thread_local bool g_t_allowed = true;

// Workspace of one layer of a merge: the sigma_R scratch when sigma_r is not
// passed, then (tensor-core T) T, A_hi, A_lo, B^T_hi, B^T_lo; for two-pass
// ranks also the second product T2 and A's two column blocks (d x 64 each).
struct MergeWs {
  size_t sigma, T, a, bt, t2, ablk, total;
  bool tc;                   // fused tensor-core merge: only the split A, B^T
};
MergeWs merge_ws_layout(const intlora_layer& l) {
  MergeWs w{0, 0, 0, 0, 0, 0, 0, false};
  if (l.sigma_r == nullptr) w.sigma = 256 + stats_partial_bytes(l.d * l.n);
  if (g_t_allowed && uses_merge_tc(l)) {
    const int64_t kp = merge_tc_kp(l.r);
    w.tc = true;
    w.a = round256(static_cast<size_t>(l.d * kp) * 4);
    w.bt = round256(static_cast<size_t>(l.n * kp) * 4);
  } else if (g_t_allowed && uses_tensor_t(l)) {
    const int64_t kp = t_gemm_kp(std::min(l.r, kTensorTMaxRank));
    w.T = round256(static_cast<size_t>(l.d * l.n) * 4);
    w.a = round256(static_cast<size_t>(l.d * kp) * 4);
    w.bt = round256(static_cast<size_t>(l.n * kp) * 4);
    if (two_pass_t(l)) {
      w.t2 = w.T;
      w.ablk = round256(static_cast<size_t>(l.d * kTensorTMaxRank) * 4);
    }
  }
  w.total = w.sigma + w.T + 2 * w.a + 2 * w.bt + w.t2 + 2 * w.ablk;
  return w;
}

// Per-layer regions in order, then (when a layer takes the fused kernel) the
// fused kernel's exchange area.
size_t merge_layers_ws_bytes(const intlora_layer* layers, int32_t count) {
  size_t total = 0;
  for (int32_t k = 0; k < count; ++k) total += merge_ws_layout(layers[k]).total;
  return total;
}
size_t merge_ws_bytes(const intlora_layer* layers, int32_t count) {
  bool tc = false;
  for (int32_t k = 0; k < count && !tc; ++k) tc = merge_ws_layout(layers[k]).tc;
  return merge_layers_ws_bytes(layers, count) + (tc ? round256(merge_tc_exchange_bytes()) : 0);
}

int32_t out_bytes_for(int variant, int w_bits, int out_bits) {
  if (variant == 0) {
    const int64_t bound = ((int64_t{1} << w_bits) - 1) * ((int64_t{1} << out_bits) - 1);
    return bound <= 32767 ? 2 : 4;
  }
  return w_bits <= 7 ? 1 : 2;
}

intlora_status merge_chunk(int variant, const intlora_layer* layers, const intlora_merge_out* outs,
                           int32_t count, int32_t bits, char* ws, cudaStream_t st) {
  std::vector<const double*> sig_r(count);
  std::vector<size_t> offset(count);
  std::vector<const float*> t_of(count, nullptr);
  std::vector<TGemmJob> tjobs, tjobs2;        // second passes of two-pass ranks
  std::vector<TGemmJob> sjobs;                // split operands of the fused-kernel layers
  std::vector<const TGemmJob*> split_of(count, nullptr);
  std::vector<std::pair<float*, const float*>> adds;   // T += T2 after the passes
  std::vector<int64_t> add_count;
  size_t off = 0;
  for (int32_t k = 0; k < count; ++k) {
    sig_r[k] = layers[k].sigma_r;
    offset[k] = off;
    const MergeWs w = merge_ws_layout(layers[k]);
    if (w.tc) {
      const intlora_layer& y = layers[k];
      char* p = ws + off + w.sigma;
      TGemmJob j;
      std::memset(&j, 0, sizeof j);
      j.A = y.A;
      j.B = y.B;
      j.d = y.d;
      j.n = y.n;
      j.r = y.r;
      j.kp = static_cast<int32_t>(merge_tc_kp(y.r));
      j.a_hi = reinterpret_cast<float*>(p);
      j.a_lo = reinterpret_cast<float*>(p + w.a);
      j.b_hi = reinterpret_cast<float*>(p + 2 * w.a);
      j.b_lo = reinterpret_cast<float*>(p + 2 * w.a + w.bt);
      sjobs.push_back(j);
    } else if (w.T > 0) {
      const intlora_layer& y = layers[k];
      char* p = ws + off + w.sigma;
      TGemmJob j;
      j.A = y.A;
      j.B = y.B;
      j.d = y.d;
      j.n = y.n;
      j.r = std::min(y.r, kTensorTMaxRank);
      j.kp = static_cast<int32_t>(t_gemm_kp(j.r));
      j.T = reinterpret_cast<float*>(p);
      j.a_hi = reinterpret_cast<float*>(p + w.T);
      j.a_lo = reinterpret_cast<float*>(p + w.T + w.a);
      j.b_hi = reinterpret_cast<float*>(p + w.T + 2 * w.a);
      j.b_lo = reinterpret_cast<float*>(p + w.T + 2 * w.a + w.bt);
      if (two_pass_t(y)) {
        // A's column blocks [0, 64) and [64, r) as dense matrices; the second
        // pass reuses the split buffers after the first has run
        float* t2 = reinterpret_cast<float*>(p + w.T + 2 * w.a + 2 * w.bt);
        float* a1 = reinterpret_cast<float*>(p + w.T + 2 * w.a + 2 * w.bt + w.t2);
        float* a2 = reinterpret_cast<float*>(p + w.T + 2 * w.a + 2 * w.bt + w.t2 + w.ablk);
        cudaError_t e = launch_copy_cols(y.A, y.r, 0, kTensorTMaxRank, y.d, a1, st);
        if (e == cudaSuccess) e = launch_copy_cols(y.A, y.r, kTensorTMaxRank, y.r - kTensorTMaxRank, y.d, a2, st);
        if (e != cudaSuccess) return cuda_fail(e, "A column copy launch");
        j.A = a1;
        TGemmJob j2 = j;
        j2.A = a2;
        j2.B = y.B + static_cast<int64_t>(kTensorTMaxRank) * y.n;
        j2.r = y.r - kTensorTMaxRank;
        j2.kp = static_cast<int32_t>(t_gemm_kp(j2.r));
        j2.T = t2;
        tjobs2.push_back(j2);
        adds.emplace_back(j.T, t2);
        add_count.push_back(y.d * y.n);
      }
      t_of[k] = j.T;
      tjobs.push_back(j);
    }
    off += w.total;
  }
  {
    size_t q = 0;
    for (int32_t k = 0; k < count; ++k)
      if (merge_ws_layout(layers[k]).tc) split_of[k] = &sjobs[q++];
  }
  if (!sjobs.empty()) {
    cudaError_t e = launch_t_split(sjobs.data(), static_cast<int>(sjobs.size()), st);
    if (e != cudaSuccess) return cuda_fail(e, "A B operand split launch");
  }
  if (!tjobs.empty()) {
    cudaError_t e = launch_t_gemm(tjobs.data(), static_cast<int>(tjobs.size()), st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core A B launch");
  }
  if (!tjobs2.empty()) {
    cudaError_t e = launch_t_gemm(tjobs2.data(), static_cast<int>(tjobs2.size()), st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core A B (second pass) launch");
    for (size_t q = 0; q < adds.size(); ++q) {
      e = launch_add_f32(adds[q].first, adds[q].second, add_count[q], st);
      if (e != cudaSuccess) return cuda_fail(e, "A B pass add launch");
    }
  }
  for (const auto& grp : group_by_seed(layers, count)) {
    // sigma_R on the device for layers that did not pass it in
    StatsBatch sb;
    std::memset(&sb, 0, sizeof sb);
    int32_t ns = 0;
    int64_t blocks = 0;
    for (int32_t k : grp) {
      if (layers[k].sigma_r != nullptr) continue;
      StatsJob& s = sb.job[ns++];
      s.W = nullptr;
      s.numel = layers[k].d * layers[k].n;
      s.stream_id = layers[k].stream_id;
      s.nblocks = static_cast<int32_t>(stats_blocks(s.numel));
      s.block_begin = blocks;
      s.sigma_w_out = nullptr;
      s.sigma_r_out = reinterpret_cast<double*>(ws + offset[k]);
      s.partial = reinterpret_cast<double*>(ws + offset[k] + 256);
      sig_r[k] = s.sigma_r_out;
      blocks += s.nblocks;
    }
    if (ns > 0) {
      sb.count = ns;
      sb.key0 = lo32(layers[grp[0]].seed);
      sb.key1 = hi32(layers[grp[0]].seed);
      sb.dist = layers[grp[0]].distribution;
      cudaError_t e = launch_stats(sb, blocks, st);
      if (e != cudaSuccess) return cuda_fail(e, "statistics kernel launch");
      e = launch_stats_finalize(sb, st);
      if (e != cudaSuccess) return cuda_fail(e, "statistics finalize launch");
    }
    // fused tensor-core merge: one launch per (geometry, code width)
    {
      std::map<std::tuple<int, int, int>, std::vector<MtcJob>> tc_groups;
      for (int32_t k : grp) {
        if (split_of[k] == nullptr) continue;
        const intlora_layer& y = layers[k];
        const TGemmJob& sj = *split_of[k];
        MtcPlan plan;
        merge_tc_plan(y.n, y.r, &plan);
        MtcJob j;
        std::memset(&j, 0, sizeof j);
        j.codes = static_cast<const uint8_t*>(y.w_round);
        j.ld_w = y.ld_w;
        j.s = y.s;
        j.z = y.z;
        j.a_hi = sj.a_hi;
        j.a_lo = sj.a_lo;
        j.b_hi = sj.b_hi;
        j.b_lo = sj.b_lo;
        j.sigma_w = y.sigma_w;
        j.sigma_r = sig_r[k];
        j.alpha = y.alpha;
        j.stream_id = y.stream_id;
        j.out = outs[k].out;
        j.scale_out = outs[k].sbar;
        j.zero_out = variant == kMul ? outs[k].zbar : nullptr;
        j.code_out = outs[k].code;
        j.d = y.d;
        j.n = y.n;
        j.kp = sj.kp;
        tc_groups[std::make_tuple(plan.group, static_cast<int>(plan.slice), y.w_bits)].push_back(j);
      }
      for (auto& kv : tc_groups) {
        MtcPlan plan;
        plan.group = std::get<0>(kv.first);
        plan.slice = std::get<1>(kv.first);
        const int wb = std::get<2>(kv.first);
        const int ob = out_bytes_for(variant == kMul ? 0 : 1, wb, bits);
        cudaError_t e = launch_merge_tc(kv.second.data(), static_cast<int>(kv.second.size()), variant, wb, ob, bits,
                                        lo32(layers[grp[0]].seed), hi32(layers[grp[0]].seed), plan,
                                        ws + merge_layers_ws_bytes(layers, count), st);
        if (e != cudaSuccess) return cuda_fail(e, "fused tensor-core merge launch");
      }
    }
    for (int wb : {4, 8}) {
      std::vector<TileLayer> L;
      for (int32_t k : grp) {
        const intlora_layer& y = layers[k];
        if (y.w_bits != wb || split_of[k] != nullptr) continue;
        TileLayer l;
        std::memset(&l, 0, sizeof l);
        l.src = y.w_round;
        l.ld_src = y.ld_w;
        l.s = y.s;
        l.z = y.z;
        l.A = y.A;
        l.B = y.B;
        l.sigma_w = y.sigma_w;
        l.sigma_r = sig_r[k];
        l.alpha = y.alpha;
        l.stream_id = y.stream_id;
        l.out = outs[k].out;
        l.ld_out = y.n;
        l.scale_out = outs[k].sbar;
        l.zero_out = variant == kMul ? outs[k].zbar : nullptr;
        l.code_out = outs[k].code;
        l.d = y.d;
        l.n = y.n;
        l.r = y.r;
        if (t_of[k] != nullptr) {          // the row kernels read T, no A B on the CUDA cores
          l.T = t_of[k];
          l.r = 0;
        }
        L.push_back(l);
      }
      if (L.empty()) continue;
      const intlora_status s = launch_tile_batch(variant, L, bits, wb,
                                                 out_bytes_for(variant == kMul ? 0 : 1, wb, bits),
                                                 layers[grp[0]].seed, layers[grp[0]].distribution, st);
      if (s != INTLORA_OK) return s;
    }
  }
  return INTLORA_OK;
}

intlora_status merge_batched(int variant, const intlora_layer* layers, const intlora_merge_out* outs,
                             int32_t count, int32_t bits, void* ws, size_t ws_bytes, void* stream) {
  if (count < 0 || (count > 0 && (layers == nullptr || outs == nullptr)))
    return fail(INTLORA_ERR_INVALID_ARG, "layers/outs must be non-NULL arrays, count >= 0");
  if (variant == kMul && (bits < 2 || bits > 8))
    return fail(INTLORA_ERR_INVALID_ARG, "u_bits must be in [2, 8]");
  if (variant == kShift && (bits < 1 || bits > 5))
    return fail(INTLORA_ERR_INVALID_ARG, "shift_bits must be in [1, 5]");
  for (int32_t k = 0; k < count; ++k) {
    intlora_status s = check_layer(&layers[k], k);
    if (s != INTLORA_OK) return s;
    s = check_out(&outs[k], variant == kMul, k);
    if (s != INTLORA_OK) return s;
  }
  g_t_allowed = true;
  size_t need = merge_ws_bytes(layers, count);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) {
    // without room for the tensor-core T buffers, form A B on the CUDA cores
    g_t_allowed = false;
    need = merge_ws_bytes(layers, count);
    if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) {
      g_t_allowed = true;
      return fail(INTLORA_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required", need);
    }
  }
  char* w = static_cast<char*>(ws);
  for (int32_t k0 = 0; k0 < count; k0 += kMaxBatch) {
    const int32_t c = std::min<int32_t>(kMaxBatch, count - k0);
    const intlora_status s = merge_chunk(variant, layers + k0, outs + k0, c, bits, w,
                                         static_cast<cudaStream_t>(stream));
    if (s != INTLORA_OK) return s;
    w += merge_ws_bytes(layers + k0, c);
  }
  g_t_allowed = true;
  return INTLORA_OK;
}

// ------------------------------------------------------------------------
// STE
// ------------------------------------------------------------------------
intlora_status check_ste(const intlora_ste_job& j, int idx) {
  if (j.G == nullptr || j.A == nullptr || j.B == nullptr || j.dA == nullptr || j.dB == nullptr)
    return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: G, A, B, dA, dB are required", idx);
  if (j.d < 1 || j.n < 1) return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: d and n must be >= 1", idx);
  if (j.d > kMaxElements / j.n) return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: d*n exceeds 2^40", idx);
  if (j.r < 1 || j.r > INTLORA_MAX_RANK)
    return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: r must be in [1, %d]", idx, INTLORA_MAX_RANK);
  if (!aligned16(j.G) || !aligned16(j.A) || !aligned16(j.B))
    return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: G, A, B must be 16-byte aligned", idx);
  if (j.mask_codes != nullptr) {
    if (j.mask_bits != 4 && j.mask_bits != 8)
      return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: mask_bits must be 4 or 8", idx);
    if (j.mask_bits == 4 && j.n % 2 != 0)
      return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: n must be even for 4-bit mask codes", idx);
    const int64_t need = j.mask_bits == 8 ? j.n : j.n / 2;
    if (j.mask_ld < need || j.mask_ld % 16 != 0 || !aligned16(j.mask_codes))
      return fail(INTLORA_ERR_INVALID_ARG,
                  "STE job %d: mask_codes must be 16-byte aligned with mask_ld >= %lld, a multiple of 16",
                  idx, static_cast<long long>(need));
    if (j.mask_z == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "STE job %d: mask_z is required", idx);
  }
  return INTLORA_OK;
}

// The kernels' descriptor of one STE job (tiling fields left 0).
SteJob ste_job_of(const intlora_ste_job& j) {
  SteJob s;
  std::memset(&s, 0, sizeof s);
  s.G = static_cast<const uint16_t*>(j.G);
  s.A = static_cast<const uint16_t*>(j.A);
  s.B = static_cast<const uint16_t*>(j.B);
  s.d = j.d;
  s.n = j.n;
  s.r = j.r;
  s.dA = j.dA;
  s.dB = j.dB;
  s.mcodes = static_cast<const uint8_t*>(j.mask_codes);
  s.mld = j.mask_ld;
  s.mbits = j.mask_bits;
  s.mz = j.mask_z;
  return s;
}

constexpr int kSteBM = 64, kSteRB = 32, kSteTargetCtas = 148 * 4;

// INTLORA_STE_KERNEL=cuda keeps the STE backward on the CUDA-core kernels;
// unset or "auto": the tensor-core kernel takes every batch it supports.
bool ste_tc_enabled() {
  const char* v = std::getenv("INTLORA_STE_KERNEL");
  return v == nullptr || std::strcmp(v, "cuda") != 0;
}

intlora_status ste_chunk(const intlora_ste_job* jobs, int32_t count, cudaStream_t st) {
  bool masked = false;                     // masked jobs run on the CUDA cores
  for (int32_t k = 0; k < count; ++k) masked = masked || jobs[k].mask_codes != nullptr;
  if (ste_tc_enabled() && !masked) {
    // tensor-core pass: both products from one read of G
    SteBatch b;
    std::memset(&b, 0, sizeof b);
    bool ok = true;
    for (int32_t k = 0; k < count && ok; ++k) {
      const intlora_ste_job& j = jobs[k];
      SteJob& s = b.job[k];
      s = ste_job_of(j);
      ok = ste_tc_supported(s);
    }
    if (ok) {
      // ranks >= 64: two passes over L2-sized regions; the rest one pass.
      // Both reduce into outputs zeroed first.
      b.count = count;
      cudaError_t e = launch_ste_zero(b, st);
      if (e != cudaSuccess) return cuda_fail(e, "STE zero launch");
      SteBatch one;
      std::memset(&one, 0, sizeof one);
      std::vector<SteJob> wide;
      for (int32_t k = 0; k < count; ++k) {
        if (ste_wide_supported(b.job[k])) wide.push_back(b.job[k]);
        else one.job[one.count++] = b.job[k];
      }
      if (!wide.empty()) {
        e = launch_ste_wide(wide.data(), static_cast<int>(wide.size()), st);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core STE (two-pass) launch");
      }
      if (one.count > 0) {
        e = launch_ste_tc(one.job, one.count, st);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core STE kernel launch");
      }
      return INTLORA_OK;
    }
  }
  // Ranks up to 8 with n % 8 == 0: one fused pass over G (both outputs).
  int max_r = 0;
  bool fusable = true;
  for (int32_t k = 0; k < count; ++k) {
    max_r = std::max(max_r, jobs[k].r);
    fusable = fusable && jobs[k].n % 8 == 0;
  }
  fusable = fusable && max_r <= 8;
  if (fusable) {
    SteBatch b;
    std::memset(&b, 0, sizeof b);
    int64_t tiles = 0;
    for (int32_t k = 0; k < count; ++k) {
      const intlora_ste_job& j = jobs[k];
      SteJob& s = b.job[k];
      s = ste_job_of(j);
      const int64_t strips = ceil_div(j.n, 128);
      // row ranges of at least 256 rows, enough CTAs to fill the GPU a few times
      int64_t ranges = std::max<int64_t>(1, ceil_div(kSteTargetCtas * 2, strips));
      ranges = std::min<int64_t>(ranges, std::max<int64_t>(1, ceil_div(j.d, 256)));
      s.ksplit = static_cast<int32_t>(ranges);
      s.tile_begin = tiles;
      tiles += strips * ranges;
    }
    b.count = count;
    b.fused = max_r <= 4 ? 4 : 8;
    b.total_tiles = tiles;
    cudaError_t e = launch_ste(b, st);
    if (e != cudaSuccess) return cuda_fail(e, "STE kernel launch");
    return INTLORA_OK;
  }
  for (int dir = 0; dir < 2; ++dir) {
    SteBatch b;
    std::memset(&b, 0, sizeof b);
    int64_t tiles = 0;
    for (int32_t k = 0; k < count; ++k) {
      const intlora_ste_job& j = jobs[k];
      SteJob& s = b.job[k];
      s = ste_job_of(j);
      const int64_t M = dir ? j.n : j.d, K = dir ? j.d : j.n;
      const int64_t base = ceil_div(M, kSteBM) * ceil_div(j.r, kSteRB);
      int64_t ks = std::max<int64_t>(1, ceil_div(kSteTargetCtas, base));
      ks = std::min<int64_t>(ks, std::max<int64_t>(1, ceil_div(K, 512)));
      s.ksplit = static_cast<int32_t>(ks);
      s.tile_begin = tiles;
      tiles += base * ks;
    }
    b.count = count;
    b.transposed = dir;
    b.total_tiles = tiles;
    cudaError_t e = launch_ste(b, st);
    if (e != cudaSuccess) return cuda_fail(e, "STE kernel launch");
  }
  return INTLORA_OK;
}

}  // namespace

void intlora::set_last_error(const char* message) {
  snprintf(g_last_error, sizeof g_last_error, "%s", message);
}

namespace {
std::atomic<uint64_t> g_launches{0};
}
void intlora::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" {

const char* intlora_status_string(int status) {
  switch (status) {
    case INTLORA_OK: return "ok";
    case INTLORA_ERR_INVALID_ARG: return "invalid argument";
    case INTLORA_ERR_UNSUPPORTED: return "unsupported";
    case INTLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case INTLORA_ERR_CUDA: return "CUDA error";
    case INTLORA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

const char* intlora_last_error(void) { return g_last_error; }

int intlora_version(void) { return 200; }   // 0.2.0: descriptors gained trailing fields

uint64_t intlora_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

uint32_t intlora_device_timeouts(void) {
  return intlora::ste_tc_timeouts() + intlora::ste_wide_timeouts() + intlora::t_gemm_timeouts() +
         intlora::int_gemm_timeouts() + intlora::merge_tc_timeouts() + intlora::selftest_timeouts();
}

namespace {

// Workspace regions of one training-backward job, in order (each 256-byte aligned):
// W'^T, [A^T; 0], [B; 0], a zero tokens x 2r operand, the tokens x 2r fp32
// product of the current pass, the two split operands, the two 2r-row
// products that become dA and dB.
struct TbWs {
  size_t wt, at, bp, zz, zw, zs1, zs2, o1, o2, total;
};
TbWs tb_ws_layout(const intlora_train_backward_job& j) {
  TbWs w;
  const size_t T = static_cast<size_t>(j.tokens), d = static_cast<size_t>(j.d), n = static_cast<size_t>(j.n);
  const size_t r = static_cast<size_t>(j.r);
  w.wt = round256(n * d * 2);
  w.at = round256(2 * r * d * 2);
  w.bp = round256(2 * r * n * 2);
  w.zz = round256(T * 2 * r * 2);
  w.zw = round256(T * 2 * r * 4);
  w.zs1 = w.zs2 = round256(T * 2 * r * 2);
  w.o1 = round256(2 * r * d * 4);
  w.o2 = round256(2 * r * n * 4);
  w.total = w.wt + w.at + w.bp + w.zz + w.zw + w.zs1 + w.zs2 + w.o1 + w.o2;
  return w;
}

intlora_status check_tb(const intlora_train_backward_job& j, int k) {
  if (j.tokens < 1 || j.d < 8 || j.n < 8 || j.d % 8 != 0 || j.n % 8 != 0)
    return fail(INTLORA_ERR_INVALID_ARG, "train-backward job %d: tokens >= 1, d and n multiples of 8 required", k);
  if (j.r < 1 || j.r > 64)
    return fail(INTLORA_ERR_INVALID_ARG, "train-backward job %d: r must be in [1, 64]", k);
  if (j.tokens > (int64_t{1} << 31) || j.d > (int64_t{1} << 31) || j.n > (int64_t{1} << 31))
    return fail(INTLORA_ERR_INVALID_ARG, "train-backward job %d: tokens, d, n must be <= 2^31", k);
  if (j.X == nullptr || j.dY == nullptr || j.W == nullptr || j.A == nullptr || j.B == nullptr ||
      j.dX == nullptr || j.dA == nullptr || j.dB == nullptr)
    return fail(INTLORA_ERR_INVALID_ARG, "train-backward job %d: every pointer is required", k);
  if (!aligned16(j.X) || !aligned16(j.dY) || !aligned16(j.W) || !aligned16(j.B) || !aligned16(j.dX) ||
      !aligned16(j.dA) || !aligned16(j.dB) || (reinterpret_cast<uintptr_t>(j.A) & 1u) != 0)
    return fail(INTLORA_ERR_INVALID_ARG, "train-backward job %d: X, dY, W, B and outputs must be 16-byte aligned", k);
  return INTLORA_OK;
}

std::mutex g_status_mutex;
uint32_t g_timeouts_reported = 0;
}

intlora_status intlora_device_status(void) {
  const cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "device synchronization");
  const uint32_t now = intlora_device_timeouts();
  std::lock_guard<std::mutex> lock(g_status_mutex);
  if (now != g_timeouts_reported) {
    const uint32_t fresh = now - g_timeouts_reported;
    g_timeouts_reported = now;
    return fail(INTLORA_ERR_TIMEOUT,
                "%u bounded device wait(s) gave up since the last check; the results of the "
                "calls in between are not valid",
                fresh);
  }
  return INTLORA_OK;
}

size_t intlora_train_backward_workspace_size(const intlora_train_backward_job* jobs, int32_t count) {
  size_t total = 0;
  for (int32_t k = 0; k < count && jobs != nullptr; ++k) total += tb_ws_layout(jobs[k]).total;
  return total;
}

intlora_status intlora_train_backward_batched(const intlora_train_backward_job* jobs, int32_t count, void* ws,
                                              size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  for (int32_t k = 0; k < count; ++k) {
    const intlora_status s = check_tb(jobs[k], k);
    if (s != INTLORA_OK) return s;
  }
  if (count == 0) return INTLORA_OK;
  const size_t need = intlora_train_backward_workspace_size(jobs, count);
  if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(INTLORA_ERR_WORKSPACE, "workspace of %zu bytes (256-byte aligned) required", need);
  if (!int_gemm_supported())
    return fail(INTLORA_ERR_UNSUPPORTED, "training backward: the driver's tensor-map encoder is unavailable");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<TransposeJob> tr;
  std::vector<intlora_linear_job> lin;
  std::vector<intlora_ste_job> pass_x1, pass_y, pass_x2;
  std::vector<SplitZJob> split1, split2;
  std::vector<CombineJob> comb;
  char* p = static_cast<char*>(ws);
  for (int32_t k = 0; k < count; ++k) {
    const intlora_train_backward_job& j = jobs[k];
    const TbWs w = tb_ws_layout(j);
    char* q = p;
    uint16_t* wt = reinterpret_cast<uint16_t*>(q);
    q += w.wt;
    uint16_t* at = reinterpret_cast<uint16_t*>(q);      // [A^T; 0]: 2r x d
    q += w.at;
    uint16_t* bp = reinterpret_cast<uint16_t*>(q);      // [B; 0]: 2r x n
    q += w.bp;
    uint16_t* zz = reinterpret_cast<uint16_t*>(q);      // zeros: tokens x 2r
    q += w.zz;
    float* zw = reinterpret_cast<float*>(q);            // tokens x 2r: [Z1 | 0], then [Z2 | 0]
    q += w.zw;
    uint16_t* zs1 = reinterpret_cast<uint16_t*>(q);
    q += w.zs1;
    uint16_t* zs2 = reinterpret_cast<uint16_t*>(q);
    q += w.zs2;
    float* o1 = reinterpret_cast<float*>(q);            // [Z1_hi | Z1_lo]^T dY: 2r x d
    q += w.o1;
    float* o2 = reinterpret_cast<float*>(q);            // [Z2_hi | Z2_lo]^T X: 2r x n
    // the padded operands: zero rows r .. 2r - 1, then A^T and B in rows 0 .. r - 1
    cudaError_t e = cudaMemsetAsync(at, 0, w.at + w.bp + w.zz, st);
    if (e != cudaSuccess) return cuda_fail(e, "zero operand fill");
    e = cudaMemcpyAsync(bp, j.B, static_cast<size_t>(j.r) * j.n * 2, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "B operand copy");
    tr.push_back(TransposeJob{static_cast<const uint16_t*>(j.W), wt, j.d, j.n, 0});
    tr.push_back(TransposeJob{static_cast<const uint16_t*>(j.A), at, j.d, j.r, 0});
    // dX = dY W' (K = d), fp32 out
    lin.push_back(intlora_linear_job{j.dY, wt, j.tokens, j.n, j.d, j.dX, 0});
    // pass over X: its product with [B; 0] is [Z1 | 0] (the other product, against zeros, is discarded)
    intlora_ste_job s;
    std::memset(&s, 0, sizeof s);
    s.G = j.X; s.A = zz; s.B = bp; s.d = j.tokens; s.n = j.n; s.r = 2 * j.r; s.dA = zw; s.dB = o2;
    pass_x1.push_back(s);
    split1.push_back(SplitZJob{zw, zs1, j.tokens, j.r, 2 * j.r});
    // pass over dY: [Z2 | 0] = dY [A^T; 0]^T and [Z1_hi | Z1_lo]^T dY (-> dA)
    s.G = j.dY; s.A = zs1; s.B = at; s.n = j.d; s.dA = zw; s.dB = o1;
    pass_y.push_back(s);
    split2.push_back(SplitZJob{zw, zs2, j.tokens, j.r, 2 * j.r});
    // pass over X: [Z2_hi | Z2_lo]^T X (-> dB); the other product is discarded
    s.G = j.X; s.A = zs2; s.B = bp; s.n = j.n; s.dA = zw; s.dB = o2;
    pass_x2.push_back(s);
    comb.push_back(CombineJob{o1, j.dA, j.d, j.r, 1});     // dA = (top + bottom)^T
    comb.push_back(CombineJob{o2, j.dB, j.n, j.r, 0});     // dB = top + bottom
    p += w.total;
  }
  cudaError_t e = launch_transpose_bf16(tr.data(), static_cast<int>(tr.size()), st);
  if (e != cudaSuccess) return cuda_fail(e, "transpose launch");
  intlora_status s = intlora_linear_bf16_batched(lin.data(), static_cast<int32_t>(lin.size()), stream);
  if (s != INTLORA_OK) return s;
  s = intlora_ste_backward_batched(pass_x1.data(), static_cast<int32_t>(pass_x1.size()), nullptr, 0, stream);
  if (s != INTLORA_OK) return s;
  e = launch_split_hilo(split1.data(), static_cast<int>(split1.size()), st);
  if (e != cudaSuccess) return cuda_fail(e, "split launch");
  s = intlora_ste_backward_batched(pass_y.data(), static_cast<int32_t>(pass_y.size()), nullptr, 0, stream);
  if (s != INTLORA_OK) return s;
  e = launch_split_hilo(split2.data(), static_cast<int>(split2.size()), st);
  if (e != cudaSuccess) return cuda_fail(e, "split launch");
  s = intlora_ste_backward_batched(pass_x2.data(), static_cast<int32_t>(pass_x2.size()), nullptr, 0, stream);
  if (s != INTLORA_OK) return s;
  e = launch_combine_halves(comb.data(), static_cast<int>(comb.size()), st);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return INTLORA_OK;
}

intlora_status intlora_selftest_bounded_wait(uint32_t limit_us, void* stream) {
  g_last_error[0] = '\0';
  if (limit_us < 1 || limit_us > 1000000)
    return fail(INTLORA_ERR_INVALID_ARG, "limit_us must be in [1, 1000000]");
  const cudaError_t e = intlora::launch_selftest_wait(uint64_t{limit_us} * 1000u, nullptr,
                                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test kernel launch");
  return INTLORA_OK;
}

int32_t intlora_int_planes(int64_t max_abs) {
  if (max_abs < 0) return 0;
  for (int32_t p = 1; p <= 3; ++p)
    if (max_abs <= (int64_t{1} << (7 * p)) - 1) return p;
  return 0;
}

intlora_status intlora_int_pack(const void* q, int32_t q_bytes, int64_t d, int64_t n, int32_t planes,
                                int8_t* packed, int32_t* overflow, void* stream) {
  g_last_error[0] = '\0';
  if (q_bytes != 1 && q_bytes != 2 && q_bytes != 4)
    return fail(INTLORA_ERR_INVALID_ARG, "q_bytes must be 1, 2 or 4");
  if (planes < 1 || planes > 3) return fail(INTLORA_ERR_INVALID_ARG, "planes must be 1, 2 or 3");
  if (d < 0 || n < 0 || n % 16 != 0) return fail(INTLORA_ERR_INVALID_ARG, "d >= 0, n >= 0 and n %% 16 == 0 required");
  if (n > 0 && d > kMaxElements / n) return fail(INTLORA_ERR_INVALID_ARG, "d*n exceeds 2^40");
  if (d * n == 0) return INTLORA_OK;
  if (q == nullptr || packed == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "q and packed are required");
  if (!aligned16(packed)) return fail(INTLORA_ERR_INVALID_ARG, "packed must be 16-byte aligned");
  const cudaError_t e = launch_int_pack(q, q_bytes, d, n, planes, packed, overflow, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INTLORA_OK : cuda_fail(e, "int pack launch");
}

intlora_status intlora_int_gemm_batched(const intlora_int_gemm_job* jobs, int32_t count, int32_t planes,
                                        void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  if (planes < 1 || planes > 3) return fail(INTLORA_ERR_INVALID_ARG, "planes must be 1, 2 or 3");
  std::vector<IntGemmJob> work;
  std::vector<int32_t> zero_jobs;
  for (int32_t k = 0; k < count; ++k) {
    const intlora_int_gemm_job& j = jobs[k];
    if (j.tokens < 0 || j.d < 0 || j.n < 0 || j.n % 16 != 0)
      return fail(INTLORA_ERR_INVALID_ARG, "int GEMM job %d: tokens, d, n >= 0 and n %% 16 == 0 required", k);
    if (j.tokens > (int64_t{1} << 31) || j.d * planes > (int64_t{1} << 31) || j.n > (int64_t{1} << 31))
      return fail(INTLORA_ERR_INVALID_ARG, "int GEMM job %d: tokens, d * planes, n must be <= 2^31", k);
    if (j.tokens == 0 || j.d == 0) continue;
    if (j.Y == nullptr || !aligned16(j.Y))
      return fail(INTLORA_ERR_INVALID_ARG, "int GEMM job %d: Y is required, 16-byte aligned", k);
    if (j.n == 0) {
      zero_jobs.push_back(k);
      continue;
    }
    if (j.X == nullptr || j.W == nullptr || j.x_scale == nullptr || j.w_scale == nullptr)
      return fail(INTLORA_ERR_INVALID_ARG, "int GEMM job %d: X, x_scale, W, w_scale are required", k);
    if (!aligned16(j.X) || !aligned16(j.W))
      return fail(INTLORA_ERR_INVALID_ARG, "int GEMM job %d: X and W must be 16-byte aligned", k);
    work.push_back(IntGemmJob{j.X, j.x_scale, j.W, j.w_scale, j.tokens, j.d, j.n, j.Y, j.y_bf16 != 0});
  }
  if (!work.empty() && !int_gemm_supported())
    return fail(INTLORA_ERR_UNSUPPORTED, "int GEMM: the driver's tensor-map encoder is unavailable");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t k : zero_jobs) {
    const size_t bytes = static_cast<size_t>(jobs[k].tokens * jobs[k].d) * (jobs[k].y_bf16 ? 2 : 4);
    const cudaError_t e = cudaMemsetAsync(jobs[k].Y, 0, bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "int GEMM zero fill");
  }
  if (!work.empty()) {
    const cudaError_t e = launch_int_gemm(work.data(), static_cast<int>(work.size()), planes, st);
    if (e != cudaSuccess) return cuda_fail(e, "int GEMM launch");
  }
  return INTLORA_OK;
}

intlora_status intlora_fakequant_bf16_batched(const intlora_fakequant_job* jobs, int32_t count, void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  std::vector<FakeQuantJob> work;
  for (int32_t k = 0; k < count; ++k) {
    const intlora_fakequant_job& j = jobs[k];
    if (j.q_bytes != 1 && j.q_bytes != 2 && j.q_bytes != 4)
      return fail(INTLORA_ERR_INVALID_ARG, "fake-quantization job %d: q_bytes must be 1, 2 or 4", k);
    if (j.d < 0 || j.n < 0) return fail(INTLORA_ERR_INVALID_ARG, "fake-quantization job %d: d, n must be >= 0", k);
    if (j.n > 0 && j.d > kMaxElements / j.n)
      return fail(INTLORA_ERR_INVALID_ARG, "fake-quantization job %d: d*n exceeds 2^40", k);
    if (j.d * j.n == 0) continue;
    if (j.q == nullptr || j.sbar == nullptr || j.w_out == nullptr || !aligned16(j.q) || !aligned16(j.w_out))
      return fail(INTLORA_ERR_INVALID_ARG, "fake-quantization job %d: q, sbar, w_out are required; q and "
                  "w_out 16-byte aligned", k);
    work.push_back(FakeQuantJob{j.q, j.q_bytes, j.sbar, j.d, j.n, static_cast<uint16_t*>(j.w_out)});
  }
  if (work.empty()) return INTLORA_OK;
  const cudaError_t e = launch_fakequant(work.data(), static_cast<int>(work.size()),
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? INTLORA_OK : cuda_fail(e, "fake-quantization launch");
}

intlora_status intlora_fakequant_bf16(const void* q, int32_t q_bytes, const float* sbar, int64_t d, int64_t n,
                                      void* w_out, void* stream) {
  intlora_fakequant_job j{q, q_bytes, sbar, d, n, w_out};
  return intlora_fakequant_bf16_batched(&j, 1, stream);
}

intlora_status intlora_linear_bf16_batched(const intlora_linear_job* jobs, int32_t count, void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  std::vector<IntGemmJob> work;
  std::vector<int32_t> zero_jobs;
  for (int32_t k = 0; k < count; ++k) {
    const intlora_linear_job& j = jobs[k];
    if (j.tokens < 0 || j.d < 0 || j.n < 0 || j.n % 8 != 0)
      return fail(INTLORA_ERR_INVALID_ARG, "linear job %d: tokens, d, n >= 0 and n %% 8 == 0 required", k);
    if (j.tokens > (int64_t{1} << 31) || j.d > (int64_t{1} << 31) || j.n > (int64_t{1} << 31))
      return fail(INTLORA_ERR_INVALID_ARG, "linear job %d: tokens, d, n must be <= 2^31", k);
    if (j.tokens == 0 || j.d == 0) continue;
    if (j.Y == nullptr || !aligned16(j.Y))
      return fail(INTLORA_ERR_INVALID_ARG, "linear job %d: Y is required, 16-byte aligned", k);
    if (j.n == 0) {
      zero_jobs.push_back(k);
      continue;
    }
    if (j.X == nullptr || j.W == nullptr || !aligned16(j.X) || !aligned16(j.W))
      return fail(INTLORA_ERR_INVALID_ARG, "linear job %d: X and W are required, 16-byte aligned", k);
    work.push_back(IntGemmJob{static_cast<const int8_t*>(j.X), nullptr, static_cast<const int8_t*>(j.W),
                              nullptr, j.tokens, j.d, j.n, j.Y, j.y_bf16 != 0});
  }
  if (!work.empty() && !int_gemm_supported())
    return fail(INTLORA_ERR_UNSUPPORTED, "bf16 GEMM: the driver's tensor-map encoder is unavailable");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t k : zero_jobs) {
    const size_t bytes = static_cast<size_t>(jobs[k].tokens * jobs[k].d) * (jobs[k].y_bf16 ? 2 : 4);
    const cudaError_t e = cudaMemsetAsync(jobs[k].Y, 0, bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "linear zero fill");
  }
  if (!work.empty()) {
    const cudaError_t e = launch_int_gemm(work.data(), static_cast<int>(work.size()), 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "bf16 GEMM launch");
  }
  return INTLORA_OK;
}

intlora_status intlora_int_gemm(const int8_t* X, const float* x_scale, const int8_t* W, const float* w_scale,
                                int64_t tokens, int64_t d, int64_t n, int32_t planes, float* Y, void* stream) {
  intlora_int_gemm_job j{X, x_scale, W, w_scale, tokens, d, n, Y, 0};
  return intlora_int_gemm_batched(&j, 1, planes, stream);
}

int32_t intlora_merge_out_bytes(int32_t variant, int32_t w_bits, int32_t out_bits) {
  if ((variant != 0 && variant != 1) || (w_bits != 4 && w_bits != 8)) return 0;
  return out_bytes_for(variant, w_bits, out_bits);
}

size_t intlora_gen_aux_workspace_size(const intlora_aux_job* jobs, int32_t count) {
  if (jobs == nullptr || count <= 0) return 0;
  return aux_ws_bytes(jobs, count);
}

intlora_status intlora_gen_aux_batched(const intlora_aux_job* jobs, int32_t count, void* ws,
                                       size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  for (int32_t k = 0; k < count; ++k) {
    const intlora_status s = check_aux_job(jobs[k], k);
    if (s != INTLORA_OK) return s;
  }
  const size_t need = aux_ws_bytes(jobs, count);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws)))
    return fail(INTLORA_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required", need);
  char* w = static_cast<char*>(ws);
  for (int32_t k0 = 0; k0 < count; k0 += kMaxBatch) {
    const int32_t c = std::min<int32_t>(kMaxBatch, count - k0);
    const intlora_status s = gen_aux_chunk(jobs + k0, c, w, static_cast<cudaStream_t>(stream));
    if (s != INTLORA_OK) return s;
    w += aux_ws_bytes(jobs + k0, c);
  }
  return INTLORA_OK;
}

intlora_status intlora_gen_aux(const float* W, int64_t d, int64_t n, uint64_t seed, uint32_t stream_id,
                               float alpha, int32_t w_bits, double* sigma_w_out, double* sigma_r_out,
                               float* r_star_out, void* w_round_out, int64_t ld_w_out, float* s_out,
                               int32_t* z_out, void* ws, size_t ws_bytes, void* stream) {
  intlora_aux_job j;
  j.W = W;
  j.d = d;
  j.n = n;
  j.seed = seed;
  j.stream_id = stream_id;
  j.alpha = alpha;
  j.w_bits = w_bits;
  j.sigma_w_out = sigma_w_out;
  j.sigma_r_out = sigma_r_out;
  j.r_star_out = r_star_out;
  j.w_round_out = w_round_out;
  j.ld_w_out = ld_w_out;
  j.s_out = s_out;
  j.z_out = z_out;
  j.distribution = INTLORA_DIST_LAPLACE;
  return intlora_gen_aux_batched(&j, 1, ws, ws_bytes, stream);
}

size_t intlora_merge_workspace_size(const intlora_layer* layers, int32_t count) {
  if (layers == nullptr || count <= 0) return 0;
  return merge_ws_bytes(layers, count);
}

intlora_status intlora_merge_mul_batched(const intlora_layer* layers, const intlora_merge_out* outs,
                                         int32_t count, int32_t u_bits, void* ws, size_t ws_bytes,
                                         void* stream) {
  g_last_error[0] = '\0';
  return merge_batched(kMul, layers, outs, count, u_bits, ws, ws_bytes, stream);
}

intlora_status intlora_merge_shift_batched(const intlora_layer* layers, const intlora_merge_out* outs,
                                           int32_t count, int32_t shift_bits, void* ws,
                                           size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  return merge_batched(kShift, layers, outs, count, shift_bits, ws, ws_bytes, stream);
}

intlora_status intlora_merge_mul(const intlora_layer* layer, int32_t u_bits, void* prod_out,
                                 float* sbar_out, int32_t* zbar_out, uint8_t* u_round_out, void* ws,
                                 size_t ws_bytes, void* stream) {
  intlora_merge_out o{prod_out, sbar_out, zbar_out, u_round_out};
  g_last_error[0] = '\0';
  if (layer == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "layer is NULL");
  return merge_batched(kMul, layer, &o, 1, u_bits, ws, ws_bytes, stream);
}

intlora_status intlora_merge_shift(const intlora_layer* layer, int32_t shift_bits, void* m_out,
                                   float* sbar_out, uint8_t* shift_out, void* ws, size_t ws_bytes,
                                   void* stream) {
  intlora_merge_out o{m_out, sbar_out, nullptr, shift_out};
  g_last_error[0] = '\0';
  if (layer == nullptr) return fail(INTLORA_ERR_INVALID_ARG, "layer is NULL");
  return merge_batched(kShift, layer, &o, 1, shift_bits, ws, ws_bytes, stream);
}

size_t intlora_ste_workspace_size(const intlora_ste_job* jobs, int32_t count) {
  // masked jobs: a bf16 copy of G with the masked elements zeroed
  size_t total = 0;
  for (int32_t k = 0; k < count && jobs != nullptr; ++k)
    if (jobs[k].mask_codes != nullptr) total += round256(static_cast<size_t>(jobs[k].d * jobs[k].n) * 2);
  return total;
}

intlora_status intlora_ste_backward_batched(const intlora_ste_job* jobs, int32_t count, void* ws,
                                            size_t ws_bytes, void* stream) {
  g_last_error[0] = '\0';
  if (count < 0 || (count > 0 && jobs == nullptr))
    return fail(INTLORA_ERR_INVALID_ARG, "jobs must be a non-NULL array, count >= 0");
  for (int32_t k = 0; k < count; ++k) {
    const intlora_status s = check_ste(jobs[k], k);
    if (s != INTLORA_OK) return s;
  }
  // masked and plain jobs go to separate launches (the plain ones keep the
  // tensor-core path). With the workspace of intlora_ste_workspace_size the
  // masked jobs become plain jobs on a masked copy of G; without it they run
  // on the CUDA-core kernels, which apply the mask as they read G.
  std::vector<intlora_ste_job> plain, masked;
  const size_t need = intlora_ste_workspace_size(jobs, count);
  const bool copy = need > 0 && ws != nullptr && ws_bytes >= need && aligned16(ws);
  std::vector<MaskJob> mjobs;
  char* wp = static_cast<char*>(ws);
  for (int32_t k = 0; k < count; ++k) {
    if (jobs[k].mask_codes == nullptr) {
      plain.push_back(jobs[k]);
    } else if (copy) {
      intlora_ste_job j = jobs[k];
      MaskJob m{static_cast<const uint16_t*>(j.G), reinterpret_cast<uint16_t*>(wp),
                static_cast<const uint8_t*>(j.mask_codes), j.mask_ld, j.mask_bits, j.mask_z, j.d, j.n};
      mjobs.push_back(m);
      j.G = wp;
      j.mask_codes = nullptr;
      plain.push_back(j);
      wp += round256(static_cast<size_t>(j.d * j.n) * 2);
    } else {
      masked.push_back(jobs[k]);
    }
  }
  if (!mjobs.empty()) {
    const cudaError_t e = launch_mask_g(mjobs.data(), static_cast<int>(mjobs.size()),
                                        static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "STE mask launch");
  }
  for (const auto* list : {&plain, &masked}) {
    const int32_t total = static_cast<int32_t>(list->size());
    for (int32_t k0 = 0; k0 < total; k0 += kMaxBatch) {
      const int32_t c = std::min<int32_t>(kMaxBatch, total - k0);
      const intlora_status s = ste_chunk(list->data() + k0, c, static_cast<cudaStream_t>(stream));
      if (s != INTLORA_OK) return s;
    }
  }
  return INTLORA_OK;
}

intlora_status intlora_ste_backward(const void* G, const void* A, const void* B, int64_t d, int64_t n,
                                    int32_t r, float* dA, float* dB, void* ws, size_t ws_bytes,
                                    void* stream) {
  intlora_ste_job j{G, A, B, d, n, r, dA, dB, nullptr, 0, 0, nullptr};
  return intlora_ste_backward_batched(&j, 1, ws, ws_bytes, stream);
}

}  // extern "C"
