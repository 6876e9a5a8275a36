// Internal descriptors and launchers of the IntLoRA kernels. The public C ABI
// (include/intlora.h) validates arguments, fills these descriptors and calls
// the launchers; descriptors travel to the device as kernel parameters, so a
// batched call needs no device-side table and no host-to-device copy.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace intlora {

constexpr int kMaxBatch = 128;          // descriptors per launch

// ---------------------------------------------------------------------------
// Whole-layer statistics (sigma_W and sigma_R): one partial per CTA, reduced
// in a fixed order by the finalize kernel, so sigma is bit-reproducible.
// ---------------------------------------------------------------------------
struct StatsJob {
  const float* W;            // nullptr: R statistics only
  int64_t numel;
  uint32_t stream_id;        // Philox counter word 2 (the key is batch level)
  int32_t nblocks;           // CTAs working on this job
  int64_t block_begin;       // index of the job's first CTA in the grid
  double* partial;           // [nblocks][4]: sum(w-K), sum((w-K)^2), sum R, sum R^2
  double* sigma_w_out;       // may be nullptr
  double* sigma_r_out;
};
// Elements one statistics CTA reduces (256 threads x 64 groups of 4) and the
// bytes of its fp64 partial (four sums), when a layer spans enough CTAs.
constexpr int kStatsThreadsPerCta = 256;
constexpr int kStatsGroupsPerThread = 64;
constexpr int64_t kStatsElementsPerCta = int64_t{4} * kStatsThreadsPerCta * kStatsGroupsPerThread;
constexpr size_t kStatsPartialBytes = 4 * sizeof(double);
struct StatsBatch {
  StatsJob job[kMaxBatch];
  int32_t count;
  uint32_t key0, key1;       // Philox key shared by every job of the batch (kept
                             // at batch level so the round keys stay uniform)
  int32_t dist;              // auxiliary law of every job (kDistLaplace, ...)
};

// ---------------------------------------------------------------------------
// Row-tile kernels (base quantization, MUL merge, SHIFT merge). A layer is cut
// into tiles of m rows; a cluster of C CTAs covers one tile, CTA k of the
// cluster owning the column slice [k n_c, (k+1) n_c). Row minima and maxima
// are reduced inside the CTA and then across the cluster through distributed
// shared memory, so every tile is finished in one pass.
// ---------------------------------------------------------------------------
enum Variant : int { kGen = 0, kMul = 1, kShift = 2 };

struct TileLayer {
  // inputs
  const void* src;           // kGen: fp32 W; merges: W_round codes
  int64_t ld_src;            // bytes per row of src
  const float* s;            // merges: base scales
  const int32_t* z;          // merges: base zero-points
  const float* A;            // merges: d x r
  const float* B;            // merges: r x n
  const double* sigma_w;
  const double* sigma_r;
  float alpha;
  uint32_t stream_id;        // Philox counter word 2 (the key is batch level)
  // outputs
  void* out;                 // kGen: codes; kMul: P; kShift: M
  int64_t ld_out;            // kGen: bytes per code row; merges: elements (= n)
  float* scale_out;          // kGen: s; merges: s_bar
  int32_t* zero_out;         // kGen: z; kMul: z_bar
  uint8_t* code_out;         // kMul: U_round; kShift: shift (optional)
  float* r_star_out;         // kGen only, optional
  const float* T;            // merges: precomputed A B (d x n) or nullptr (then r = 0)
  // geometry
  int64_t d, n;
  int32_t r;
  int32_t n_c;               // columns per CTA (multiple of 4)
  int32_t m;                 // rows per tile (multiple of kRowsPerItem)
  int32_t b_resident;        // B slice stays in shared memory across tiles
  int32_t kc;                // B rows per staged chunk
  int32_t aligned;           // n % 4 == 0: one Philox block per 4 columns
  int64_t tile_begin;        // global index of the layer's first tile
};
struct TileBatch {
  TileLayer layer[kMaxBatch];
  int32_t count;
  uint32_t key0, key1;       // Philox key shared by every layer of the batch
  int32_t variant;           // kGen, kMul or kShift
  int32_t cluster;           // C
  int32_t num_clusters;
  int64_t total_tiles;
  int32_t bits;              // kGen: w_bits; kMul: u_bits; kShift: shift_bits
  int32_t w_bits;            // code width of the input W_round (merges)
  int32_t out_bytes;         // merges: bytes per element of `out` (1, 2 or 4)
  int32_t smem_u;            // floats of the tile buffer (>= m n_c of every layer)
  int32_t smem_b;            // floats of the B buffer
  int32_t smem_a;            // floats of the A-rows buffer (>= r m)
  int32_t small;             // every layer below 2^34 elements (32-bit Philox block index)
  int32_t dist;              // auxiliary law (other than Laplace: the RANK = -2 kernels)
};

constexpr int kTileThreads = 256;
constexpr int kRowsPerItem = 4;                     // rows of one work item
constexpr int kMaxTileRows = 128;

// Dynamic shared memory of a tile launch with the given carve-up.
size_t tile_smem_bytes(int variant, int smem_u, int smem_b, int smem_a);

// ---------------------------------------------------------------------------
// Team kernels (same three operations, rows up to kTeamMaxCols columns with
// n % 4 == 0). A team of TW warps of one CTA owns a group of 4 rows across the
// whole row: lane l of the team takes the column quads l, l + 32 TW, ... (at
// most kTeamMaxSweeps of them), keeps its values in a lane-private stretch of
// shared memory, and the team combines its row extrema with one named barrier
// (none for TW = 1). Warps never wait on the rest of the CTA inside a layer.
// ---------------------------------------------------------------------------
constexpr int kTeamThreads = 256;
constexpr int kTeamWarps = kTeamThreads / 32;
constexpr int kTeamRows = 4;
constexpr int kTeamMaxSweeps = 6;
constexpr int64_t kTeamMaxCols = int64_t{4} * kTeamThreads * kTeamMaxSweeps;
constexpr int kTeamMaxCtas = 148 * 4;
// Base quantization of wider rows (n up to 4 x 256 x (kTeamMaxSweeps +
// kTeamTmemSweeps), a whole number of sweeps of the 8-warp team): the first
// kTeamTmemSweeps sweeps of every lane are parked in tensor memory (256
// columns per CTA, two CTAs per SM), the rest in shared memory.
constexpr int kTeamTmemSweeps = 8;
constexpr int64_t kTeamWideMaxCols = int64_t{4} * kTeamThreads * (kTeamMaxSweeps + kTeamTmemSweeps);

struct TeamLayer {
  const void* src;           // kGen: fp32 W; merges: W_round codes
  int64_t ld_src;            // bytes per row of src
  const float* s;            // merges: base scales
  const int32_t* z;          // merges: base zero-points
  const float* A;            // merges: d x r
  const float* B;            // merges: r x n (16-byte aligned)
  const double* sigma_w;
  const double* sigma_r;
  float alpha;
  uint32_t stream_id;
  void* out;
  int64_t ld_out;            // kGen: bytes per code row; merges: elements (= n)
  float* scale_out;
  int32_t* zero_out;
  uint8_t* code_out;
  float* r_star_out;
  const float* T;            // merges: precomputed A B (d x n) or nullptr
  int64_t d, n;
  int32_t r;
  int32_t team_warps;        // TW: 1, 2, 4 or 8
  int32_t sweeps;            // column quads per lane: ceil(n / (128 TW))
  int64_t tile_begin;        // a tile is the kTeamWarps / TW row groups of one CTA step
};
struct TeamBatch {
  TeamLayer layer[kMaxBatch];
  int32_t count;
  uint32_t key0, key1;
  int32_t bits;              // kGen: w_bits; kMul: u_bits; kShift: shift_bits
  int32_t w_bits;
  int32_t sweeps_max;        // shared memory is carved for this many sweeps
  int32_t tmem_sweeps;       // 0, or kTeamTmemSweeps: sweeps parked in tensor memory (kGen)
  int32_t num_ctas;
  int64_t total_tiles;
  int32_t cta_begin[kTeamMaxCtas + 1];   // tiles of CTA k: [cta_begin[k], cta_begin[k+1])
};

size_t team_smem_bytes(int variant, int sweeps_max);

// ---------------------------------------------------------------------------
// STE backward.
// ---------------------------------------------------------------------------
struct SteJob {
  const uint16_t* G;
  const uint16_t* A;
  const uint16_t* B;
  int64_t d, n;
  int32_t r;
  float* dA;
  float* dB;
  const uint8_t* mcodes;     // masked STE: W_round (nullptr: no mask), row stride mld
  int64_t mld;
  int32_t mbits;             // 4 or 8
  const int32_t* mz;         // zero-points: G is used only where code != z
  int64_t tile_begin;        // first CTA of this job in the grid
  int32_t ksplit;            // CTAs sharing one output tile (split reduction); fused
                             // pass: row ranges per column strip
};
struct SteBatch {
  SteJob job[kMaxBatch];
  int32_t count;
  int32_t transposed;        // 0: dA = G B^T; 1: dB^T = G^T A
  int32_t fused;             // 4 or 8: one fused pass (both outputs) at that rank bound
  int64_t total_tiles;
};

// Launchers: return the cudaError_t of the launch.
cudaError_t launch_stats(const StatsBatch& b, int64_t total_blocks, cudaStream_t s);
cudaError_t launch_stats_finalize(const StatsBatch& b, cudaStream_t s);
cudaError_t launch_tiles(const TileBatch& b, int rank_ct, bool aligned, cudaStream_t s);
int tile_max_active_clusters(int variant, int w_bits, int rank_ct, int out_bytes, bool aligned,
                             int cluster, size_t smem);
cudaError_t launch_team(const TeamBatch& b, int variant, int rank_ct, int out_bytes, cudaStream_t s);
int team_max_active_ctas(int variant, int w_bits, int rank_ct, int out_bytes, size_t smem, bool tmem_park = false);
cudaError_t launch_ste(const SteBatch& b, cudaStream_t s);
cudaError_t launch_ste_zero(const SteBatch& b, cudaStream_t s);   // dA and dB of every job
// Masked STE with a workspace: G' = G where W_round != z, else 0 (bf16 copy),
// after which the plain (tensor-core) path runs on G'.
struct MaskJob {
  const uint16_t* G;
  uint16_t* out;
  const uint8_t* codes;
  int64_t ld;
  int32_t bits;
  const int32_t* z;
  int64_t d, n;
};
cudaError_t launch_mask_g(const MaskJob* jobs, int count, cudaStream_t s);
// tcgen05 path of the STE backward (one pass over G, both products on the
// tensor cores); outputs must be zeroed first.
constexpr int kSteTcMaxRank = 128;
bool ste_tc_supported(const SteJob& j);
cudaError_t launch_ste_tc(const SteJob* jobs, int count, cudaStream_t s);
unsigned int ste_tc_timeouts();
// Ranks 64..128 (r % 8 == 0): two tensor-core passes over G, each product
// reduced inside one CTA (no atomics, no zeroing).
constexpr int kSteWideMinRank = 64;
bool ste_wide_supported(const SteJob& j);
cudaError_t launch_ste_wide(const SteJob* jobs, int count, cudaStream_t s);
unsigned int ste_wide_timeouts();

// T = A B on the tensor cores (tf32 three-term split) for ranks in
// [kTensorTMinRank, kTensorTMaxRank]: the row kernels then read T instead of
// forming it on the CUDA cores.
constexpr int kTensorTMinRank = 32;
constexpr int kTensorTMaxRank = 64;
struct TGemmJob {
  const float* A;            // d x r
  const float* B;            // r x n
  int64_t d, n;
  int32_t r, kp;             // kp = t_gemm_kp(r)
  float* T;                  // d x n (workspace)
  float* a_hi;               // d x kp (workspace), 16-byte aligned like the others
  float* a_lo;
  float* b_hi;               // n x kp: B transposed
  float* b_lo;
};
int64_t t_gemm_kp(int32_t r);
bool t_gemm_supported(int64_t d, int64_t n, int32_t r);
cudaError_t launch_t_gemm(const TGemmJob* jobs, int count, cudaStream_t s);
unsigned int t_gemm_timeouts();
// The split pass alone: A_hi, A_lo (d x kp) and B^T_hi, B^T_lo (n x kp) of
// every job (T and r above kp unused), one launch.
cudaError_t launch_t_split(const TGemmJob* jobs, int count, cudaStream_t s);

// Fused merge with A B on the tensor cores (merge_tc_kernels.cu): T = A B
// (tf32 three-term split) lands in tensor memory, U is formed and parked
// there, the row extrema are combined across the group of CTAs that shares a
// row (through an exchange area of the workspace), and the merged weights are
// stored; no other intermediate goes to global memory.
constexpr int32_t kMergeTcMaxRank = 128;
constexpr int kMergeTcMaxGroup = 64;        // CTAs per row: rows of up to 64 x 512 columns
constexpr int kMergeTcMaxCtas = 256;        // CTAs of one launch (one per SM)
struct MtcJob {
  const uint8_t* codes;      // W_round, row stride ld_w bytes (multiple of 16)
  int64_t ld_w;
  const float* s;
  const int32_t* z;
  const float* a_hi;         // d x kp split operands (workspace, 16-byte aligned)
  const float* a_lo;
  const float* b_hi;         // n x kp (B transposed)
  const float* b_lo;
  const double* sigma_w;
  const double* sigma_r;
  float alpha;
  uint32_t stream_id;
  void* out;                 // P or M, d x n dense
  float* scale_out;
  int32_t* zero_out;         // MUL only (may be nullptr)
  uint8_t* code_out;         // optional U_round / shift codes
  int64_t d, n;
  int32_t kp;                // merge_tc_kp(r)
};
struct MtcPlan {
  int group;                 // CTAs sharing one row (G)
  int32_t slice;             // columns per CTA (multiple of 32, <= 512)
};
int64_t merge_tc_kp(int32_t r);
// Geometry for rows of n columns at rank r, or false when the fused kernel
// does not take such a layer (n % 32 != 0, r outside [1, kMergeTcMaxRank],
// rows longer than kMergeTcMaxGroup x 512 columns).
bool merge_tc_plan(int64_t n, int32_t r, MtcPlan* plan);
// Bytes of the exchange area a launch needs (16-byte aligned, any contents).
size_t merge_tc_exchange_bytes();
cudaError_t launch_merge_tc(const MtcJob* jobs, int count, int variant, int w_bits, int out_bytes, int bits,
                            uint32_t key0, uint32_t key1, const MtcPlan& plan, void* exchange, cudaStream_t s);
unsigned int merge_tc_timeouts();
cudaError_t launch_zero(float* p, int64_t count, cudaStream_t s);

// Integer inference GEMM on merged weights (tcgen05 kind::i8): Y = diag(x_scale)
// X Q^T diag(w_scale) with Q held as base-128 int8 digit planes [d][P][n].
struct IntGemmJob {
  const int8_t* X;           // tokens x n, 16-byte aligned, n % 16 == 0
  const float* x_scale;      // [tokens]
  const int8_t* W;           // [d][planes][n] digit planes, 16-byte aligned
  const float* w_scale;      // [d]
  int64_t tokens, d, n;
  void* Y;                   // tokens x d: fp32, or bf16 when y_bf16
  int32_t y_bf16;
};
int int_gemm_chans(int planes);          // output channels per tile: 256 / 128 / 64
bool int_gemm_supported();
cudaError_t launch_int_pack(const void* w, int w_bytes, int64_t d, int64_t n, int planes, int8_t* out,
                            int32_t* overflow, cudaStream_t s);
cudaError_t launch_int_gemm(const IntGemmJob* jobs, int count, int planes, cudaStream_t s);
// planes = 0 above: the bf16 GEMM Y = X W^T (X tokens x n, W d x n bf16).
struct FakeQuantJob {
  const void* q;             // merged integer weights (q_bytes 1, 2 or 4), d x n, 16-byte aligned
  int32_t q_bytes;
  const float* sbar;
  int64_t d, n;
  uint16_t* out;             // bf16 d x n, 16-byte aligned
};
cudaError_t launch_fakequant(const FakeQuantJob* jobs, int count, cudaStream_t s);
unsigned int int_gemm_timeouts();

// Sets the calling thread's intlora_last_error() message.
void set_last_error(const char* message);

// Glue kernels of the training backward (train_backward_kernels.cu).
struct TransposeJob {        // out (cols x rows) = in (rows x cols)^T, bf16
  const uint16_t* in;
  uint16_t* out;
  int64_t rows, cols;
  int64_t block_begin;       // set by the launcher
};
struct SplitZJob {           // zs (rows x 2r bf16) = [hi | lo] of z (rows x r fp32, row stride ld)
  const float* z;
  uint16_t* zs;
  int64_t rows;
  int32_t r;
  int32_t ld;                // floats between rows of z (>= r)
};
struct CombineJob {          // out = in[0:r] + in[r:2r] (in: 2r x cols fp32); transposed: out is cols x r
  const float* in;
  float* out;
  int64_t cols;
  int32_t r;
  int32_t transposed;
};
cudaError_t launch_transpose_bf16(const TransposeJob* jobs, int count, cudaStream_t s);
cudaError_t launch_split_hilo(const SplitZJob* jobs, int count, cudaStream_t s);
cudaError_t launch_combine_halves(const CombineJob* jobs, int count, cudaStream_t s);

// Self-test of the bounded waits: one mbarrier that nothing completes, waited
// on for limit_ns (selftest_kernels.cu); *completed (device int, optional)
// receives 0 when the wait gave up.
cudaError_t launch_selftest_wait(uint64_t limit_ns, int* completed, cudaStream_t s);
unsigned int selftest_timeouts();

// Count of kernel launches this library has enqueued (all threads, since it
// was loaded); `counted` adds one when a launch returned cudaSuccess.
void note_launch();
inline cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) note_launch();
  return e;
}

}  // namespace intlora
