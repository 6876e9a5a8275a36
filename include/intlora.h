/*
 * intlora.h - C ABI of the IntLoRA integer low-rank merge library (B200, sm_100a).
 *
 * IntLoRA adapts a quantized linear layer with integer-type low-rank factors
 * so that the merged weight comes out already quantized, with no post-training
 * quantization step. This library implements the per-layer hot path of that
 * method on the GPU:
 *
 *   - intlora_gen_aux       auxiliary matrix R (seeded Philox4x32-10 Laplace
 *                           noise, never stored), its variance-matched copy
 *                           R* = (sigma_W / sigma_R)^alpha * R, and the base
 *                           quantization W_round, s, z of W - R*;
 *   - intlora_merge_mul     IntLoRA_MUL: the adaptation term
 *                           U = s + (R* + A B) / (W_round - z) quantized per row
 *                           by a uniform affine quantizer, merged by an integer
 *                           Hadamard product;
 *   - intlora_merge_shift   IntLoRA_SHIFT: U quantized by a log2 quantizer,
 *                           merged by arithmetic shifts;
 *   - intlora_ste_backward  straight-through backward dA = G B^T, dB = A^T G;
 *   - intlora_int_gemm      integer inference GEMM on the merged weights
 *                           (int8 activations x integer merged weights).
 *
 * Sources, cited by page title and section:
 *   [notes]   "IntLoRA: Integral Low-rank Adaptation of Quantized Diffusion
 *             Models", Paper-Notes page (ICML2025), section 方法详解:
 *             1. AQS (W' = Q[W - sg(R)] + sg(R) + AB; R regenerated online from
 *             a fixed seed and distribution statistics, no storage),
 *             2. MLA (W' = [s + (R + AB) / (W_round - z)] (.) (W_round - z)),
 *             3. VMC (R* = r^alpha R, r = sigma_W / sigma_R),
 *             两种实现版本 (IntLoRA_MUL: W' = s_bar (U_round - z_bar) (.)
 *             (W_round - z); IntLoRA_SHIFT: W' = sign(V) (.) [(W_round - z) >>
 *             shift]; training through the quantizers with the STE).
 *   [summary] atlas.scime.ai summary of the same paper, "Measured effects":
 *             Laplace is the auxiliary distribution.
 *   [Philox]  Salmon et al., SC'11, Philox4x32-10.
 *
 * Conventions (fixed here where the pages are silent):
 *   - Layer W is d x n, row-major: d output channels (rows i), n inputs
 *     (columns j). Flat index e = i * n + j. A is d x r, B is r x n, both
 *     dense row-major (leading dimensions r and n).
 *   - W_round codes are unsigned: 8-bit codes one per byte; 4-bit codes two per
 *     byte, even column in the low nibble. Row i starts at byte i * ld_w.
 *   - R_ij = Laplace(0,1) from word (e mod 4) of Philox4x32-10 with key
 *     (seed low 32 bits, seed high 32 bits) and counter (e/4 low, e/4 high,
 *     stream_id, 0). u = (2 (x >> 9) + 1) 2^-24, v = u - 1/2,
 *     R = -sign(v) ln(1 - 2|v|).
 *   - sigma_W, sigma_R are population standard deviations over the whole
 *     d x n layer. c = (sigma_W / sigma_R)^alpha is formed in fp64.
 *   - Affine quantizer of a row x (b bits): range [min(0, min x), max(0, max x)],
 *     scale = range / (2^b - 1) (a row whose range is {0} gets scale 1, zero 0),
 *     zero = clamp(rne(-min / scale), 0, 2^b - 1),
 *     code = clamp(rne(x / scale) + zero, 0, 2^b - 1); rne = round to nearest,
 *     ties to even.
 *   - D_ij = W_round_ij - z_i. Where D_ij = 0 the quotient term of U is 0.
 *   - SHIFT: s_bar_i = max_j |U_ij|, V = U / s_bar, shift = nearest integer
 *     of -log2|V| clamped to [0, 2^shift_bits - 1], M = sign(V) (D >> shift)
 *     with an arithmetic (floor) shift. The merged weight is s_bar_i M_ij.
 *   - MUL: the merged weight is s_bar_i P_ij with P = (U_round - z_bar) D.
 *   - GPU arithmetic is fp32 (fp64 for the sigma reductions and c). A code
 *     may differ by one from an fp64 evaluation only where the fp64 pre-round
 *     value lies within ~1e-5 relative of a rounding boundary.
 *
 * Ownership and execution:
 *   - Every data pointer is a DEVICE pointer (or managed memory) on the
 *     current device, allocated and owned by the caller. sigma scalars are
 *     device doubles. The library keeps no state between calls and allocates
 *     nothing; scratch space is the caller's workspace (ws, ws_bytes), whose
 *     required size the *_workspace_size queries return.
 *   - Every call validates its arguments on the host and returns a status
 *     before launching anything. Work is then enqueued asynchronously on
 *     `stream` (a cudaStream_t; NULL = legacy default stream). A launch
 *     failure returns INTLORA_ERR_CUDA. No call synchronizes the device,
 *     except the status queries intlora_device_status and
 *     intlora_device_timeouts, which say so.
 *   - Outputs must not alias inputs. Calls on different streams that share a
 *     workspace race.
 *   - intlora_last_error() returns a thread-local description of the most
 *     recent failure in the calling thread.
 */
#ifndef INTLORA_H
#define INTLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum intlora_status {
    INTLORA_OK = 0,
    INTLORA_ERR_INVALID_ARG = 1,  /* bad pointer, size, bit width, alignment */
    INTLORA_ERR_UNSUPPORTED = 2,  /* valid but outside what this library handles */
    INTLORA_ERR_WORKSPACE = 3,    /* ws NULL or ws_bytes below the query's value */
    INTLORA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    INTLORA_ERR_TIMEOUT = 5       /* a bounded device wait gave up */
} intlora_status;

/* Static description of a status code. */
const char* intlora_status_string(int status);
/* Thread-local message of the last failure in this thread ("" if none). */
const char* intlora_last_error(void);
/* Library version, major * 10000 + minor * 100 + patch. */
int intlora_version(void);

/* Auxiliary law of R [summary, "Measured effects": the ablation compares
 * Laplace, the method's choice, with Gaussian, Cauchy and Student-t auxiliary
 * matrices]. Every law reads element e from word e mod 4 of Philox block e / 4
 * through u = (2 (x >> 9) + 1) 2^-24:
 *   LAPLACE     -sign(u - 1/2) ln(1 - 2 |u - 1/2|)
 *   GAUSSIAN    Box-Muller on the word pair (2p, 2p + 1) of the block: word 2p
 *               gets sqrt(-2 ln u_2p) cos(2 pi u_2p+1), word 2p + 1 the sine
 *   CAUCHY      tan(pi (u - 1/2))
 *   STUDENT_T2  (2u - 1) / sqrt(2 u (1 - u)): Student-t with 2 degrees of
 *               freedom (the pages give none; 2 has a closed-form inverse CDF)
 * Layers with a law other than Laplace run on the general row-tile kernels
 * with A B on the CUDA cores. */
#define INTLORA_DIST_LAPLACE 0
#define INTLORA_DIST_GAUSSIAN 1
#define INTLORA_DIST_CAUCHY 2
#define INTLORA_DIST_STUDENT_T2 3

/* Limits of this library. */
#define INTLORA_MAX_RANK 256
#define INTLORA_MAX_BATCH 128     /* descriptors per batched call */

/* --------------------------------------------------------------------------
 * Layer preparation [notes, AQS and VMC].
 *
 * From the fp32 weight W (d x n, dense row-major) computes, for one layer:
 *   sigma_w_out  = std(W), sigma_r_out = std(R)            (device doubles)
 *   r_star_out   = R* = c R            (optional, fp32 d x n dense; may be NULL)
 *   w_round_out  = codes of W - R*     (optional; w_bits 4 or 8, row stride
 *                                       ld_w_out bytes; may be NULL)
 *   s_out, z_out = per-row scale (fp32) and zero-point (int32) of W - R*
 *                  (required when w_round_out is given, else may be NULL)
 * alpha >= 0. With alpha = 0 (c = 1) r_star_out is R itself.
 * Requirements: d, n >= 1; d * n < 2^40; w_bits in {4, 8}; n even when
 * w_bits = 4; ld_w_out >= n * w_bits / 8; W, w_round_out, r_star_out 16-byte
 * aligned; ws of at least intlora_gen_aux_workspace_size bytes, 256-byte
 * aligned.
 * ------------------------------------------------------------------------ */
typedef struct intlora_aux_job {
    const float* W;
    int64_t d, n;
    uint64_t seed;
    uint32_t stream_id;
    float alpha;
    int32_t w_bits;
    double* sigma_w_out;
    double* sigma_r_out;
    float* r_star_out;
    void* w_round_out;
    int64_t ld_w_out;
    float* s_out;
    int32_t* z_out;
    int32_t distribution;       /* INTLORA_DIST_*; intlora_gen_aux(_noalloc) use LAPLACE */
} intlora_aux_job;

size_t intlora_gen_aux_workspace_size(const intlora_aux_job* jobs, int32_t count);

intlora_status intlora_gen_aux(const float* W, int64_t d, int64_t n, uint64_t seed,
                               uint32_t stream_id, float alpha, int32_t w_bits,
                               double* sigma_w_out, double* sigma_r_out, float* r_star_out,
                               void* w_round_out, int64_t ld_w_out, float* s_out,
                               int32_t* z_out, void* ws, size_t ws_bytes, void* stream);

/* `count` jobs (a host array) in three launches in total. */
intlora_status intlora_gen_aux_batched(const intlora_aux_job* jobs, int32_t count, void* ws,
                                       size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * Layer preparation without a workspace argument. The paper has no
 * counterpart: this serves callers that cannot allocate device memory, such
 * as a host framework whose memory manager owns every device allocation, or a
 * latency-critical loop where cudaMalloc (which may synchronize the device) is
 * not allowed.
 *
 * Same arguments, results and validation as intlora_gen_aux, minus ws and
 * ws_bytes: the scratch it needs comes from a fixed array compiled into the
 * library (16 KB of device memory on every GPU that loads the library, held
 * until the process exits). Hence a size limit: d * n must not exceed
 * INTLORA_NOALLOC_MAX_ELEMENTS, else INTLORA_ERR_UNSUPPORTED with a message in
 * intlora_last_error(). Allocates nothing.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it for the life of the process; make that first
 * call before any stream capture, and do not reset the device
 * (cudaDeviceReset) between calls, since the cached address would then be
 * stale. All calls share the one array: calls whose GPU work can overlap
 * (different streams without ordering) race on it and must be serialized by
 * the caller. Nothing in the array needs clearing between calls.
 * ------------------------------------------------------------------------ */
#define INTLORA_NOALLOC_MAX_ELEMENTS 4194304

intlora_status intlora_gen_aux_noalloc(const float* W, int64_t d, int64_t n, uint64_t seed,
                                       uint32_t stream_id, float alpha, int32_t w_bits,
                                       double* sigma_w_out, double* sigma_r_out,
                                       float* r_star_out, void* w_round_out, int64_t ld_w_out,
                                       float* s_out, int32_t* z_out, void* stream);

/* --------------------------------------------------------------------------
 * Merges [notes, MLA and 两种实现版本].
 *
 * One quantized layer with its LoRA factors. All pointers are device pointers.
 * sigma_w is required (from intlora_gen_aux); sigma_r may be NULL, in which
 * case the call regenerates R once more to reduce it on the device (this
 * needs workspace). r in [1, INTLORA_MAX_RANK].
 * ------------------------------------------------------------------------ */
typedef struct intlora_layer {
    int64_t d, n;
    int32_t r;
    int32_t w_bits;             /* 4 (packed nibbles) or 8 */
    const void* w_round;        /* 16-byte aligned; row i at byte i * ld_w */
    int64_t ld_w;               /* bytes per row, >= n * w_bits / 8 */
    const float* s;             /* [d] base scales */
    const int32_t* z;           /* [d] base zero-points, in [0, 2^w_bits - 1] */
    const float* A;             /* d x r fp32 */
    const float* B;             /* r x n fp32 */
    uint64_t seed;              /* Philox key of R */
    uint32_t stream_id;         /* Philox counter word 2 */
    float alpha;                /* VMC exponent */
    const double* sigma_w;      /* device scalar */
    const double* sigma_r;      /* device scalar or NULL */
    int32_t distribution;       /* INTLORA_DIST_*: the law R was drawn from in gen_aux */
} intlora_layer;

/* Outputs of one merge.
 *   out:  MUL: P = (U_round - z_bar) D, int16 when
 *         (2^w_bits - 1)(2^u_bits - 1) <= 32767, else int32, d x n dense;
 *         SHIFT: M = sign(V) (D >> shift), int8 when w_bits <= 7, else int16.
 *   sbar: [d] fp32 per-row scale of the merged weight (W' = sbar_i * out_ij).
 *   zbar: [d] int32 MUL zero-point of U (ignored by SHIFT, may be NULL there).
 *   code: optional uint8 d x n: MUL U_round, SHIFT shift; may be NULL.
 * out and code must be 16-byte aligned. */
typedef struct intlora_merge_out {
    void* out;
    float* sbar;
    int32_t* zbar;
    uint8_t* code;
} intlora_merge_out;

/* Bytes per element of `out`: MUL (variant 0) or SHIFT (variant 1). */
int32_t intlora_merge_out_bytes(int32_t variant, int32_t w_bits, int32_t out_bits);

/* Workspace of a merge call (16-byte aligned device memory, caller-owned):
 *  - for each layer with sigma_r == NULL: the scratch of its sigma_R reduction;
 *  - for each Laplace layer the fused tensor-core merge takes (n % 32 == 0,
 *    and r >= 16 or n > 6144): the exact tf32 hi/lo splits of A and B^T that
 *    the tensor cores multiply (4 (d + n) kp x 2 bytes, kp = 32, 64 or 128),
 *    plus, once per call, the kernel's row-exchange area (512 KiB);
 *  - for each other Laplace layer with r in [32, 128] and n % 4 == 0: its
 *    product T = A B (d x n fp32) and the same splits (kp = 32 or 64); for r
 *    above 64 (two passes over the rank) also the second product (d x n
 *    fp32) and A's two column blocks (2 x d x 64 fp32)
 *  -- [IntLoRA paper notes, method section 2: U = s + (R* + A B) / D].
 * A call given at least the sigma part but less than the whole still runs: it
 * then forms A B on the CUDA cores inside the row merge kernels (same results
 * up to fp32 rounding order, slower at these ranks). Less than the sigma
 * part: INTLORA_ERR_WORKSPACE. */
size_t intlora_merge_workspace_size(const intlora_layer* layers, int32_t count);

/* IntLoRA_MUL, u_bits in [2, 8]. */
intlora_status intlora_merge_mul(const intlora_layer* layer, int32_t u_bits, void* prod_out,
                                 float* sbar_out, int32_t* zbar_out, uint8_t* u_round_out,
                                 void* ws, size_t ws_bytes, void* stream);
/* IntLoRA_SHIFT, shift_bits in [1, 5] (shift codes 0 .. 2^shift_bits - 1). */
intlora_status intlora_merge_shift(const intlora_layer* layer, int32_t shift_bits, void* m_out,
                                   float* sbar_out, uint8_t* shift_out, void* ws,
                                   size_t ws_bytes, void* stream);

/* `count` layers (host arrays `layers` and `outs`) in one grouped launch. */
intlora_status intlora_merge_mul_batched(const intlora_layer* layers,
                                         const intlora_merge_out* outs, int32_t count,
                                         int32_t u_bits, void* ws, size_t ws_bytes,
                                         void* stream);
intlora_status intlora_merge_shift_batched(const intlora_layer* layers,
                                           const intlora_merge_out* outs, int32_t count,
                                           int32_t shift_bits, void* ws, size_t ws_bytes,
                                           void* stream);

/* --------------------------------------------------------------------------
 * STE backward [notes, 两种实现版本: training through the quantizers with the
 * straight-through estimator]. With G the upstream gradient on W' (d x n),
 *   dA = G B^T   (d x r, fp32),     dB = A^T G   (r x n, fp32).
 * G, A, B are bf16 (raw 16-bit patterns), dense row-major, 16-byte aligned;
 * accumulation is fp32. dA and dB are overwritten.
 * ------------------------------------------------------------------------ */
typedef struct intlora_ste_job {
    const void* G;
    const void* A;
    const void* B;
    int64_t d, n;
    int32_t r;
    float* dA;
    float* dB;
    /* Masked STE (optional; mask_codes NULL = the plain STE above). Where
     * D_ij = W_round_ij - z_i = 0 the adaptation term is U = s_i whatever A B
     * is [notes, MLA, with the zero-divisor rule], so the exact derivative of
     * the pre-quantization weight U (.) D with respect to A B is the mask
     * [D != 0]; the masked STE uses G (.) [D != 0] in both products.
     * mask_codes: the layer's W_round (mask_bits 4: packed nibbles, low nibble
     * = even column; 8: bytes), row i at byte i * mask_ld, 16-byte aligned;
     * mask_z: [d] int32 zero-points. Given the workspace that
     * intlora_ste_workspace_size asks for (a bf16 copy of G per masked job),
     * a masked job zeroes the masked elements into that copy and takes the
     * plain path; without it the CUDA-core kernels apply the mask as they
     * read G (slower, same results up to fp32 summation order). */
    const void* mask_codes;
    int64_t mask_ld;
    int32_t mask_bits;
    const int32_t* mask_z;
} intlora_ste_job;

size_t intlora_ste_workspace_size(const intlora_ste_job* jobs, int32_t count);

intlora_status intlora_ste_backward(const void* G, const void* A, const void* B, int64_t d,
                                    int64_t n, int32_t r, float* dA, float* dB, void* ws,
                                    size_t ws_bytes, void* stream);
intlora_status intlora_ste_backward_batched(const intlora_ste_job* jobs, int32_t count,
                                            void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------------------
 * Integer inference on the merged weights [notes, 两种实现版本 and the
 * training/inference efficiency table: the merged weight is s_bar_i Q_ij with
 * Q integer (IntLoRA_MUL: Q = P = (U_round - z_bar) D; IntLoRA_SHIFT:
 * Q = M = sign(V) (D >> shift)), so the merged layer runs as an integer GEMM
 * (W8A8 / W4A8) with no post-training quantization step]:
 *
 *   Y[t][i] = x_scale[t] * w_scale[i] * sum_j X[t][j] Q[i][j]
 *
 * X: int8 activations, tokens x n row-major, with a per-token scale (the
 * activation quantizer is the caller's). w_scale: s_bar of the merged layer.
 *
 * Q reaches the tensor cores as P base-128 digit planes of int8:
 *   digit_k = (Q >> 7k) & 127 for k < P - 1, digit_{P-1} = Q >> 7(P-1)
 * (arithmetic shift), Q = sum_k 128^k digit_k. P = 1 holds |Q| <= 127 (SHIFT
 * of 4-bit codes), 2 holds |Q| <= 16383 (MUL of 4-bit codes, SHIFT of 8-bit
 * codes), 3 holds |Q| <= 2^21 - 1 (MUL of 8-bit codes); each plane costs one
 * int8 GEMM.
 * ------------------------------------------------------------------------ */

/* Digit planes needed for |Q| <= max_abs: 1, 2 or 3; 0 if above 2^21 - 1. */
int32_t intlora_int_planes(int64_t max_abs);

/* Packs Q (d x n row-major; q_bytes = 1, 2 or 4: int8, int16 or int32, the
 * merge outputs) into `packed`, laid out [d][planes][n] int8 (plane k of row i
 * at packed + (i * planes + k) * n). n % 16 == 0; packed 16-byte aligned.
 * If `overflow` (a device int32, may be NULL) is given, the number of values
 * whose top digit leaves [-128, 127] is added to it (those are stored
 * truncated). Asynchronous on `stream`. */
intlora_status intlora_int_pack(const void* q, int32_t q_bytes, int64_t d, int64_t n,
                                int32_t planes, int8_t* packed, int32_t* overflow,
                                void* stream);

typedef struct intlora_int_gemm_job {
    const int8_t* X;          /* tokens x n, 16-byte aligned */
    const float* x_scale;     /* [tokens] */
    const int8_t* W;          /* packed digit planes [d][planes][n], 16-byte aligned */
    const float* w_scale;     /* [d] */
    int64_t tokens, d, n;     /* n % 16 == 0; tokens, d * planes <= 2^31 */
    void* Y;                  /* tokens x d row-major, 16-byte aligned (overwritten) */
    int32_t y_bf16;           /* 0: Y fp32; 1: Y bf16 (nearest, ties to even) */
} intlora_int_gemm_job;

/* Every job of one call uses the same plane count. The integer sums are
 * exact (s32 per plane, planes added in 64-bit integers); the result is
 * fp32(sum) * fp32(x_scale[t] * w_scale[i]), three fp32 roundings, then
 * rounded to bf16 (nearest, ties to even) when y_bf16. Jobs with n = 0 get
 * Y = 0. Asynchronous on `stream`; no workspace. The single-layer call
 * writes fp32 Y. */
intlora_status intlora_int_gemm_batched(const intlora_int_gemm_job* jobs, int32_t count,
                                        int32_t planes, void* stream);
intlora_status intlora_int_gemm(const int8_t* X, const float* x_scale, const int8_t* W,
                                const float* w_scale, int64_t tokens, int64_t d, int64_t n,
                                int32_t planes, float* Y, void* stream);

/* --------------------------------------------------------------------------
 * Training forward on the merged weights [notes, 两种实现版本 and the
 * efficiency table: IntLoRA trains with the merged weight quantized in the
 * forward pass (fake quantization) and the STE in the backward]:
 *
 *   W'_bf16 = bf16(fp32(s_bar_i) * Q_ij)          (intlora_fakequant_bf16)
 *   Y = X W'^T,  X bf16 tokens x n, fp32 accumulation, Y fp32 tokens x d
 *                                                 (intlora_linear_bf16_batched)
 *
 * Q: the merge output (q_bytes 1, 2 or 4); the product is rounded once to
 * fp32 and then to bf16 (nearest, ties to even). The GEMM runs on the tensor
 * cores (tcgen05 kind::f16, the integer GEMM's pipeline with bf16 operands).
 * Requirements: n % 8 == 0; X, W, Y, w_out 16-byte aligned. Y is
 * overwritten (zero when n = 0). Asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
intlora_status intlora_fakequant_bf16(const void* q, int32_t q_bytes, const float* sbar, int64_t d,
                                      int64_t n, void* w_out, void* stream);

typedef struct intlora_fakequant_job {
    const void* q;            /* merged integer weights, d x n, 16-byte aligned */
    int32_t q_bytes;          /* 1, 2 or 4 */
    const float* sbar;        /* [d] */
    int64_t d, n;
    void* w_out;              /* bf16 d x n, 16-byte aligned */
} intlora_fakequant_job;

/* Many layers in one launch. */
intlora_status intlora_fakequant_bf16_batched(const intlora_fakequant_job* jobs, int32_t count,
                                              void* stream);

typedef struct intlora_linear_job {
    const void* X;            /* bf16 tokens x n */
    const void* W;            /* bf16 d x n (the fake-quantized merged weight) */
    int64_t tokens, d, n;
    void* Y;                  /* tokens x d: fp32, or bf16 when y_bf16 */
    int32_t y_bf16;
} intlora_linear_job;

intlora_status intlora_linear_bf16_batched(const intlora_linear_job* jobs, int32_t count,
                                           void* stream);

/* Number of bounded device-side waits that gave up since the library was
 * loaded: 0 in a healthy run. Every kernel that waits on an mbarrier or on
 * another CTA (the tensor-core STE kernels, the T GEMM, the integer GEMM,
 * the fused merge and its row exchange) bounds each wait (2 s); a wait that
 * gives up is counted here, the CTA drains what it started, releases its
 * tensor memory and returns, so a broken run shows up as a nonzero count and
 * wrong outputs instead of a hung device. Synchronous (reads the device
 * counters); the library has no counterpart of this on the pages. */
uint32_t intlora_device_timeouts(void);

/* --------------------------------------------------------------------------
 * Training backward of one IntLoRA linear Y = X W'^T, W' the fake-quantized
 * merged weight of the forward (intlora_fakequant_bf16), the gradient
 * reaching the low-rank factors through the straight-through estimator
 * [notes, 两种实现版本: training passes the quantizers with the STE; the
 * efficiency table times these steps]. Per job, from bf16 inputs:
 *     dX = dY W'                       (tokens x n)
 *     dA = G B^T,  dB = A^T G,  G = dY^T X  (the gradient on W', d x n)
 * G is never formed: with Z1 = X B^T and Z2 = dY A (tokens x r),
 * dA = dY^T Z1 and dB = Z2^T X, every product on the tensor cores with fp32
 * accumulation (Z enters the last products as two exact bf16 halves, so
 * they stay fp32-faithful). Besides the dX GEMM, X is streamed twice and dY
 * once (X -> Z1; dY -> Z2 and dA; X -> dB), each pass forming both of its
 * products from one read.
 *
 * X: bf16 tokens x n; dY: bf16 tokens x d; W: bf16 d x n; A: bf16 d x r;
 * B: bf16 r x n; all row-major, X, dY, W, B 16-byte aligned. Outputs (fp32,
 * row-major, 16-byte aligned): dX tokens x n, dA d x r, dB r x n; written,
 * not accumulated. Requires tokens >= 1, d and n multiples of 8, 1 <= r <= 64.
 * The workspace (intlora_train_backward_workspace_size, 256-byte aligned
 * regions per job) holds W'^T, A^T and B padded with r zero rows, Z1 and Z2
 * with their bf16 halves, and the halves' products.
 * ------------------------------------------------------------------------ */
typedef struct intlora_train_backward_job {
    const void* X;
    const void* dY;
    const void* W;
    const void* A;
    const void* B;
    int64_t tokens, d, n;
    int32_t r;
    float* dX;
    float* dA;
    float* dB;
} intlora_train_backward_job;

size_t intlora_train_backward_workspace_size(const intlora_train_backward_job* jobs, int32_t count);

intlora_status intlora_train_backward_batched(const intlora_train_backward_job* jobs, int32_t count,
                                              void* ws, size_t ws_bytes, void* stream);

/* Device health check: synchronizes the device, then returns
 * INTLORA_ERR_TIMEOUT (with the count in intlora_last_error()) when bounded
 * device-side waits gave up since the previous intlora_device_status() call
 * (the results of the calls in between are not valid), a CUDA error as
 * INTLORA_ERR_CUDA, else INTLORA_OK. Each timeout is reported once. The pages
 * have no counterpart of this; it is how the library's failure detection
 * reaches the caller without a device trap. */
intlora_status intlora_device_status(void);

/* Self-test of that failure path: enqueues on `stream` one kernel that waits,
 * through the same bounded mbarrier wait the tensor-core kernels use, on a
 * barrier nothing will complete, for limit_us microseconds (1 .. 1,000,000).
 * No copy or tensor-core product is in flight; the wait gives up, is counted,
 * and the kernel returns, leaving the context usable. A following
 * intlora_device_status() returns INTLORA_ERR_TIMEOUT. */
intlora_status intlora_selftest_bounded_wait(uint32_t limit_us, void* stream);

/* Number of kernels this library has enqueued (every entry point, every
 * thread) since it was loaded; a launch that the CUDA runtime refused is not
 * counted. Host-side counter, never synchronizes. The pages have no
 * counterpart of this; it lets a caller count the GPU launches of a region. */
uint64_t intlora_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* INTLORA_H */
