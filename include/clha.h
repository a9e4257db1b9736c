/*
 * clha.h — C ABI of the CLHA calibration library (libclha.so, CUDA, sm_100a).
 *
 * CLHA (Cross-Layer Hessian Aggregation) quantizes weights that several layers of a weight-shared
 * Mixture-of-Experts transformer reuse. Source: the technical summary "CLHA – Cross-Layer Hessian
 * Aggregation voor het kwantiseren van Weight-Shared Mixture-of-Experts Transformers" (below: the
 * CLHA page). Its section 2.2 gives three phases, which the calls below follow:
 *   (1) collection  — per layer and per active expert, a Hessian and a token count
 *                     (clha_route_topk, clha_gather, clha_expert_act, clha_collect);
 *   (2) aggregation — H_comb = sum_i alpha_i H_i with routing-frequency or equal weights (clha_aggregate);
 *   (3) quantization — standard GPTQ column-sequential updates with H_comb (clha_factor_groups_as,
 *                     clha_quantize_as; GPTQ's factor either U with H^-1 = U^T U, as the paper states
 *                     it, or the block-scaled Cholesky factor of H itself, which gives the same
 *                     updates at half the factor's work), scored by the loss of section 2.1 (clha_loss).
 * GPTQ is the algorithm of Frantar et al. (2022), "GPTQ: Accurate Post-Training Quantization for
 * Generative Pre-trained Transformers", Algorithm 1.
 *
 * Conventions for every call:
 *   - Array arguments are DEVICE pointers owned by the caller unless the comment says "host".
 *     The library owns only clha_ctx, clha_accum and its internal workspace.
 *   - Work is queued on the context's stream, in call order. Calls that return host values
 *     (alpha_out, lambda_out, loss_out, clha_accum_export, clha_check) synchronise that stream.
 *   - Row-major layouts. X is [tokens, d] (a token's d values contiguous). A weight W is
 *     [d_out, d_in] with y = W x. Hessians and factors are [d, d] float32.
 *   - Shapes: every d, d_in and d_out must be a multiple of 128, else CLHA_ERR_UNSUPPORTED_SHAPE.
 *     Token counts may be any value >= 0.
 *   - Errors are returned, never raised: no call aborts or traps. Argument errors are detected on
 *     the host before any work is queued. Errors found by a kernel (a non-finite input, a
 *     non-positive pivot) are recorded on the device and returned by the next synchronising call
 *     on the context; clha_last_error() then names the call and, for a pivot, the column.
 */
#ifndef CLHA_H
#define CLHA_H

#include <stdint.h>

#if defined(__GNUC__)
#define CLHA_API __attribute__((visibility("default")))
#else
#define CLHA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CLHA_OK = 0,
    CLHA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, k > E, bits outside 2..8, ... */
    CLHA_ERR_UNSUPPORTED_SHAPE = 2, /* d / d_in / d_out not a multiple of 128, group not 128, ... */
    CLHA_ERR_NOT_PD = 3,            /* damped Hessian has a non-positive pivot (index in last_error) */
    CLHA_ERR_NONFINITE = 4,         /* NaN or Inf in logits, activations or a Hessian */
    CLHA_ERR_EMPTY = 5,             /* aggregation over slots with no tokens in any layer */
    CLHA_ERR_OOM = 6,               /* workspace allocation failed */
    CLHA_ERR_CUDA = 7,              /* a CUDA runtime call failed (message in last_error) */
    CLHA_ERR_TIMEOUT = 8            /* a bounded device-side wait ran out (factor graph, GPTQ, Gram,
                                       activation); the kernel returned and the context stays usable */
} clha_status;

typedef enum { CLHA_BF16 = 0, CLHA_F32 = 1 } clha_dtype;

typedef enum {
    CLHA_ALPHA_ROUTING = 0,   /* alpha_i = n_i / sum_j n_j           (CLHA page §2.2 (2), "rt") */
    CLHA_ALPHA_EQUAL = 1,     /* alpha_i = 1 / n_layers              (CLHA page §2.2 (2), "eq") */
    CLHA_ALPHA_EXPLICIT = 2,  /* alpha from the caller; (1, 0) is per-layer calibration on layer 0 */
    CLHA_ALPHA_SUM = 3,       /* alpha_i = n_i / 2, so H_comb = sum_i S_i: the unnormalised Gram sum
                                 of the E-PMQ statistics (the E-PMQ page, section 2) */
    /* Flag, or'ed into one of the modes above: a slot whose weighted aggregate has no energy
     * (tr H_comb = 0: no tokens in any layer, or none in the layers with nonzero alpha) gets
     * H_comb = 0, lambda = 1 and H_damped = I instead of CLHA_ERR_EMPTY (no tokens at all) or a zero
     * H_damped that clha_factor rejects. GPTQ under H_damped = I is round to nearest: the calibration
     * data say nothing about that expert. Its loss under H_comb is 0. */
    CLHA_AGG_EMPTY_IDENTITY = 0x100
} clha_alpha_mode;

/* GPTQ parameters: bits in 2..8, group = 128 (grid per 128 input columns), block = 128 (lazy-update
 * block), damp_frac > 0 (lambda = damp_frac * mean(diag H_comb)). */
typedef struct { int bits; int group; int block; float damp_frac; } clha_quant_params;

typedef struct clha_ctx clha_ctx;
typedef struct clha_accum clha_accum;

/* ------------------------------------------------------------------------------------------ context */

/* Create a context on CUDA `device` that queues work on `cuda_stream` (a cudaStream_t; NULL = the
 * legacy default stream). The stream is borrowed, not owned. */
CLHA_API clha_status clha_create(int device, void* cuda_stream, clha_ctx** out);
/* Release the context and its workspace (synchronises its stream first). NULL is ignored. */
CLHA_API void clha_destroy(clha_ctx* ctx);
/* Message of the last failed call on this context ("" if none). Valid until the next call. */
CLHA_API const char* clha_last_error(const clha_ctx* ctx);
/* Synchronise the stream and return (and clear) any error a kernel recorded. */
CLHA_API clha_status clha_check(clha_ctx* ctx);
/* Library ABI version (major*100 + minor). */
CLHA_API int clha_version(void);
/* Number of kernels this context has launched so far (a tracing counter; 0 for NULL). */
CLHA_API int64_t clha_kernel_launches(const clha_ctx* ctx);

/* ------------------------------------------------------------------------------- phase 1: collection */

/* Top-k routing (the CLHA page §2.2 (1) accumulates statistics "for each active expert"; §2.3 names
 * the K-of-E routing). For each of n tokens, the k largest of its E router logits [n, E] float32:
 * ids [n, k] int32 in descending logit order, ties to the lower expert index; counts [E] int32 is
 * OVERWRITTEN with the number of tokens each expert receives. 1 <= k <= E <= 1024.
 * A NaN or Inf logit is recorded as CLHA_ERR_NONFINITE. */
CLHA_API clha_status clha_route_topk(clha_ctx* ctx, const float* logits, int64_t n, int E, int k,
                            int32_t* ids, int32_t* counts);

/* Upper bound of the rows clha_gather writes for (n, k, E): n*k + 128*E. */
CLHA_API int64_t clha_packed_rows(int64_t n, int k, int E);

/* Group the routed tokens by expert. X [n, d] (bf16 or f32) -> X_packed [packed_rows, d], same dtype,
 * in which expert e owns rows [seg[e], seg[e] + seg[E + 1 + e]) in ascending token order, every
 * segment starts at a multiple of 128 and the rows between segments are zero.
 * seg is int64 [2E + 1]: seg[0..E] segment starts (seg[E] = total padded rows), seg[E+1 .. 2E]
 * token counts. packed_rows must be >= clha_packed_rows(n, k, E). perm (optional, int32
 * [packed_rows]) receives each packed row's token index (-1 for padding rows). X_packed may be NULL
 * when perm is given: then only the permutation and seg are produced (nothing is copied), for
 * clha_collect_gathered and clha_expert_act_gathered, which read the rows where they are. */
CLHA_API clha_status clha_gather(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n, int d,
                        const int32_t* ids, int k, int E, void* X_packed, int64_t packed_rows,
                        int64_t* seg, int32_t* perm);

/* clha_gather without any device allocation; the paper has no counterpart (it is a service for
 * callers, not part of the method). Same arguments, layout and results as clha_gather. It exists for
 * callers that must not see the library allocate device memory: processes whose memory is handed
 * out by their own allocator (a framework's caching allocator, a fixed arena), where a cudaMalloc
 * can fail once the arena holds the memory and a cudaFree synchronises the whole device.
 * Its scratch (clha_gather's workspace) is a fixed 4 MiB array in the library's device image,
 * which every GPU that loads the library holds until the process exits. A call needs
 * ceil(n/256)*E*4 bytes there for the block histograms, plus packed_rows*4 bytes for the token
 * permutation only when perm is NULL (each part rounded up to 256 bytes). So with perm given the
 * limit is ceil(n/256)*E <= ~1M (e.g. n = 8M tokens at E = 32); with perm NULL, roughly
 * n*k + 128*E <= ~1M packed rows. A larger gather is rejected with CLHA_ERR_INVALID_ARG before
 * anything is queued. Every call looks up the array's device address (cudaGetSymbolAddress) with
 * the context's device current; the first call on a device may load the module, so make it before
 * any stream capture. All calls share the array and it keeps the last call's contents (each call
 * rewrites what it reads); calls that overlap on the GPU race on it. */
CLHA_API clha_status clha_gather_noalloc(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n, int d,
                                         const int32_t* ids, int k, int E, void* X_packed, int64_t packed_rows,
                                         int64_t* seg, int32_t* perm);

/* Expert FFN activation feeding the down projection: h = SiLU(x Wg^T) * (x Wu^T) per token of
 * each expert, SiLU product in fp64, stored as bf16 (round to nearest even). The pages do not
 * spell this out: the down projection's Hessian needs its input, and that input is this product.
 * X is bf16 [rows, d_model]; Wg, Wu are bf16 [E, d_ff, d_model] (experts stacked); h is bf16
 * [rows, d_ff]. With seg (from clha_gather) rows follow its segments and padding rows of h are
 * written as zero; with seg == NULL, E must be 1 and all `rows` rows belong to that expert.
 * Two kernels (clha_set_act_kernel): the tensor cores (bf16 products, fp32 accumulation in up to 8
 * K-chunks added in fp64), or fp32 FMA (32-term fp32 chunks added in fp64). The tensor core adds a
 * group of products after aligning them to the largest one, so inputs with outlier channels (tens of
 * times the rest) lose enough low bits there to flip bf16 roundings of h too often; by default each
 * call measures every channel's max |x| over the rows on the device and takes the tensor cores only
 * when all of them are within 4x of their mean, the FMA kernel otherwise (no host round trip). */
CLHA_API clha_status clha_expert_act(clha_ctx* ctx, const void* X, int64_t rows, int d_model,
                            const int64_t* seg, int E, const void* Wg, const void* Wu, int d_ff,
                            void* h);

/* Which activation kernel clha_expert_act uses: CLHA_ACT_AUTO (default; chosen per call from the
 * rows' channel magnitudes), CLHA_ACT_FMA or CLHA_ACT_TENSOR (always). clha_expert_act_gathered always
 * takes the FMA kernel. clha_last_act_kernel reports the kernel of the context's last
 * clha_expert_act call (synchronises; -1 on error). */
#define CLHA_ACT_AUTO 0
#define CLHA_ACT_FMA 1
#define CLHA_ACT_TENSOR 2
CLHA_API clha_status clha_set_act_kernel(clha_ctx* ctx, int kernel);
CLHA_API int clha_last_act_kernel(clha_ctx* ctx);
/* clha_expert_act with the segment rows read from the token matrix X [n, d_model] through perm (as in
 * clha_collect_gathered; -1 entries are zero rows); h is written in the packed segment layout,
 * packed_rows rows (>= seg[E]), padding rows zero. Same values as clha_expert_act on the packed X. */
CLHA_API clha_status clha_expert_act_gathered(clha_ctx* ctx, const void* X, int64_t n, int d_model,
                                              const int32_t* perm, int64_t packed_rows, const int64_t* seg, int E,
                                              const void* Wg, const void* Wu, int d_ff, void* h);

/* Largest number of layers (or source experts) one accumulator holds. */
#define CLHA_MAX_LAYERS 32

/* Accumulator of per-(layer, slot) Gram matrices S = sum x x^T (float32 [d, d], upper triangle
 * authoritative, lower triangle may hold partial values) and token counts (int64). A slot is one
 * expert (or one dense weight). Layer-aware by construction (CLHA page §2.4): every collect names
 * its layer, and layers never share an accumulator. Created zeroed. */
CLHA_API clha_status clha_accum_create(clha_ctx* ctx, int d, int n_layers, int n_slots, clha_accum** out);
CLHA_API clha_status clha_accum_destroy(clha_accum* acc);
CLHA_API clha_status clha_accum_zero(clha_ctx* ctx, clha_accum* acc);
/* Device views: S[((layer * n_slots) + slot) * d * d ...], counts[layer * n_slots + slot]. */
CLHA_API clha_status clha_accum_buffers(const clha_accum* acc, float** S, int64_t** counts);
/* Checkpoint / resume: copy all of S and counts to or from host buffers of
 * n_layers*n_slots*d*d floats and n_layers*n_slots int64. */
CLHA_API clha_status clha_accum_export(clha_ctx* ctx, const clha_accum* acc, float* host_S, int64_t* host_counts);
CLHA_API clha_status clha_accum_import(clha_ctx* ctx, clha_accum* acc, const float* host_S, const int64_t* host_counts);

/* Phase 1 accumulation for one layer (CLHA page §2.2 (1)): S[layer][slot] += X_e^T X_e and
 * counts[layer][slot] += n_e. With seg == NULL, all `rows` rows of X go to slot `slot0` (a dense
 * weight, or an always-active shared expert); with seg (clha_gather's layout), expert e goes to
 * slot slot0 + e for e < E. X is [rows, d] bf16 (tensor cores, fp32 accumulation) or f32 (fp32 FMA).
 * A NaN or Inf entry of X is recorded as CLHA_ERR_NONFINITE. */
CLHA_API clha_status clha_collect(clha_ctx* ctx, clha_accum* acc, int layer, const void* X, clha_dtype dtype,
                         int64_t rows, int d, const int64_t* seg, int E, int slot0);

/* Phase 1 straight from the token matrix, with no packed copy of the routed rows (the gather fused
 * into the Gram accumulation): X [n, d] bf16 (n < 2^31); expert e's rows are the tokens
 * perm[seg[e] .. seg[e] + seg[E + 1 + e]) in that order, perm and seg as clha_gather writes them (a
 * padding entry, -1, reads as a zero row). The tensor-core kernel fetches the operands four rows at
 * a time by TMA gather4 from X itself. Accumulates into slots slot0 .. slot0 + E - 1 of `layer` and
 * adds the token counts, exactly as clha_collect does on clha_gather's packed X (same rows in the
 * same order: the same sums). perm must be 16-byte aligned. */
CLHA_API clha_status clha_collect_gathered(clha_ctx* ctx, clha_accum* acc, int layer, const void* X, int64_t n,
                                           int d, const int32_t* perm, const int64_t* seg, int E, int slot0);

/* ------------------------------------------------------------------------------ phase 2: aggregation */

/* For each slot s in [slot0, slot0 + n_slots): alpha_i from `mode` over the accumulator's layers
 * (CLHA page §2.2 (2); alpha_in is a host [n_layers] array for CLHA_ALPHA_EXPLICIT, else ignored),
 * H_comb = sum_i alpha_i (2 / n_i) S_i (layers with n_i = 0 contribute nothing; §2.1 Proposition 1),
 * lambda = damp_frac * mean(diag H_comb) and H_damped = H_comb + lambda I.
 * H_comb and H_damped are float32 [n_slots, d, d], full symmetric. H_comb may be NULL.
 * alpha_out (host double [n_slots * n_layers]) and lambda_out (host double [n_slots]) are optional;
 * passing either synchronises. lambda_dev (device double [n_slots], optional) receives lambda without
 * synchronising, for clha_quantize's loss. A slot with no tokens in any layer gives CLHA_ERR_EMPTY. */
CLHA_API clha_status clha_aggregate(clha_ctx* ctx, const clha_accum* acc, int slot0, int n_slots,
                           clha_alpha_mode mode, const double* alpha_in, double damp_frac,
                           float* H_comb, float* H_damped, double* alpha_out, double* lambda_out,
                           double* lambda_dev);

/* ------------------------------------------------------------------------------ phase 3: quantization */

/* GPTQ's factor of the damped Hessian: U upper triangular with H_damped^-1 = U^T U (the upper
 * Cholesky factor of the inverse), for `batch` problems [batch, d, d] float32. Computed as
 * H_damped = R R^T with R upper (Cholesky in reversed index order) and U = R^-1, in float64.
 * The strict lower triangle of U is written as zero. A non-positive pivot is recorded as
 * CLHA_ERR_NOT_PD with the problem and column. */
CLHA_API clha_status clha_factor(clha_ctx* ctx, const float* H_damped, int batch, int d, float* U);

/* The same factor for up to CLHA_FACTOR_MAX_GROUPS groups of problems of different sizes in one
 * launch of the task graph (e.g. the gate/up Hessians [E, d_model, d_model] and the down Hessians
 * [E, d_ff, d_ff] of a layer group): each group is `batch` problems [batch, d, d] float32 on the
 * device, H_damped read and U written as in clha_factor. The small groups' short dependency chains
 * run alongside the large groups' bulk work. `groups` is a host array read during the call (the
 * caller keeps ownership). Errors as in clha_factor; the problem index of a CLHA_ERR_NOT_PD report
 * counts across the groups in order. */
#define CLHA_FACTOR_MAX_GROUPS 4
typedef struct clha_factor_group {
    const float* H_damped;   /* device, [batch, d, d] */
    float* U;                /* device, [batch, d, d] */
    int batch;
    int d;                   /* multiple of 128 */
} clha_factor_group;
CLHA_API clha_status clha_factor_groups(clha_ctx* ctx, int n_groups, const clha_factor_group* groups);

/* The factor in either of two forms, each written as float32 [batch, d, d], zero below the diagonal:
 *   CLHA_FACTOR_INV_CHOL    U, as clha_factor writes it (H_damped^-1 = U^T U);
 *   CLHA_FACTOR_BLOCK_CHOL  F, the Cholesky factor of H_damped scaled per 128-column block: with R
 *                           upper and H_damped = R R^T, and U = R^-1 (U_bb = R_bb^-1 on the diagonal
 *                           blocks), F_bb = U_bb and F_ab = R_ab U_bb for a < b.
 * F takes one Cholesky and no triangular inverse (half the flops of U). GPTQ with F
 * (clha_quantize_as) makes the same decisions as GPTQ with U, up to rounding: every step inside a
 * block uses U_bb, and the lazy update of block b from the earlier columns a, W_b - E_a U_ab with
 * GPTQ's scaled errors E (W - W_hat = E U), equals W_b + (W_a - W_hat_a) F_ab. F serves GPTQ only:
 * E-PMQ's target needs U. Groups, errors and limits as clha_factor_groups. */
typedef enum clha_factor_form { CLHA_FACTOR_INV_CHOL = 0, CLHA_FACTOR_BLOCK_CHOL = 1 } clha_factor_form;
CLHA_API clha_status clha_factor_groups_as(clha_ctx* ctx, clha_factor_form form, int n_groups,
                                           const clha_factor_group* groups);

/* Time limit, in nanoseconds, of each dependency wait inside clha_factor's task graph (a CTA waiting
 * for a tile that another CTA is still producing); 0 restores the default of 4 s. A wait that runs
 * out sets the graph's abort flag: every CTA stops taking tasks and returns, the call's U is
 * undefined, and the next synchronising call (clha_check) reports CLHA_ERR_TIMEOUT. The context stays
 * usable, and the next clha_factor starts a fresh graph. Nothing in the method needs another limit;
 * it exists so that a stalled graph ends with an error instead of holding the GPU, and so that this
 * path can be exercised (a limit of a microsecond or so runs out on the first real dependency). */
CLHA_API clha_status clha_set_factor_wait_limit(clha_ctx* ctx, uint64_t ns);

/* ------------------------------------------------------------------------------ deployable codes */

/* Packs GPTQ's codes (uint8 [rows, d_in], values < 2^bits) into uint32 [rows, d_in * bits / 32]:
 * each row's codes as one little-endian bit stream, code j at bits [bits*j, bits*j + bits) (a code
 * may straddle two words). bits in 2..8, d_in a multiple of 128. Device pointers are the caller's.
 * The pages give no deployable layout; this one has no padding at any bit width. */
CLHA_API clha_status clha_pack_codes(clha_ctx* ctx, const uint8_t* codes, int64_t rows, int d_in, int bits,
                                     uint32_t* packed);
/* W_hat = s (q - z) per 128-column group from packed codes (scales float32 and zeros uint8
 * [rows, d_in / 128], as written by clha_quantize): float32 [rows, d_in], bit-identical to
 * clha_quantize's W_hat. */
CLHA_API clha_status clha_dequantize(clha_ctx* ctx, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                                     int64_t rows, int d_in, int bits, float* W_hat);

/* The deployable layer: Y [n, d_out] float32 = X [n, d_in] W_hat^T, W_hat decoded from the packed
 * codes inside the product (fp32 FMA). X bf16 or f32; d_out a multiple of 64. */
CLHA_API clha_status clha_dequant_matmul(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n,
                                         const uint32_t* packed, const float* scales, const uint8_t* zeros, int d_out,
                                         int d_in, int bits, float* Y);

/* E-PMQ's quantization target (the E-PMQ page, section 2: expert-driven output targets, anchoring to
 * the merged weights, and the solver's statistics H = sum_i H_i + lambda I, R = sum_i W_i H_i +
 * lambda W_m). The K = n_layers "layers" of `acc` are the K source experts: S_i = acc's Gram of
 * layer i in slot `slot` (H_i = S_i, upper triangle read). With U the clha_factor of the damped
 * aggregate of that slot in mode CLHA_ALPHA_SUM (H_comb = sum_i S_i, H_damped = H) and lambda its
 * damping (lambda_dev as written by clha_aggregate), computes in float64
 *   W_target = (lambda W_m + sum_i W_i S_i) U^T U  =  R H^-1
 * and writes it as float32 [d_out, d]; clha_quantize of W_target with U then runs E-PMQ's GPTQ step.
 * W_src: device [K, d_out, d] (the source experts' weights), W_merged: device [d_out, d], both of
 * `dtype`; U: device float32 [d, d]; lambda_dev: device double. d = acc's d; d_out a multiple of 64.
 * Device pointers are the caller's. */
CLHA_API clha_status clha_epmq_target(clha_ctx* ctx, const clha_accum* acc, int slot, const void* W_src,
                                      const void* W_merged, clha_dtype dtype, int d_out, const float* U,
                                      const double* lambda_dev, float* W_target);

/* GPTQ (CLHA page §2.2 (3)): column-sequential quantization of `batch` weights W [batch, d_out, d_in]
 * (bf16 or f32) in natural column order, with lazy updates over 128-column blocks. U holds n_u
 * factors [n_u, d_in, d_in] and problem b uses factor b % n_u (1 <= n_u <= batch; with gate and up
 * stacked as [2E] and n_u = E they share their expert's factor).
 * At the start of each group of 128 columns a row's grid is fixed from its current values:
 * xmin = min(0, min w), xmax = max(0, max w) ([-1, 1] if both are 0), s = (xmax - xmin)/(2^b - 1),
 * z = round(-xmin/s); each column then takes q = clamp(round(w/s) + z, 0, 2^b - 1), w_hat = s (q - z),
 * and its error (w - w_hat)/U_jj is subtracted along row j of U from the later columns. The grid and
 * the code are decided in IEEE float32 (round to nearest even); the updates inside a block accumulate
 * in float32 and the lazy block updates run on the tensor cores in three tf32 products (hi*hi +
 * hi*lo + lo*hi), float32-class accuracy. The columns are taken in chunks of 512: a lazy update sums
 * at most one chunk's errors in the tensor core's accumulator, and each finished chunk's errors are
 * folded into float32 running weights of the later columns with round-to-nearest adds (workspace:
 * one more float32 copy of W when d_in > 512).
 * Outputs: codes uint8 [batch, d_out, d_in], scales float32 and zeros uint8 [batch, d_out, d_in/128],
 * W_hat float32 [batch, d_out, d_in] (may be NULL).
 * Optional loss (device double [batch], overwritten), given lambda (device double [n_u], the damping of
 * each factor, e.g. clha_aggregate's lambda_dev): the CLHA page §2.1 term tr[(W_hat - W) H_comb
 * (W_hat - W)^T] of each problem, from GPTQ's own errors e: W - W_hat = E U and U H_d U^T = I give
 * tr[D H_d D^T] = |E|^2, and H_comb = H_d - lambda I gives loss = |E|^2 - lambda |W_hat - W|^2
 * (summed in float64). Pass NULL for both to skip it; clha_loss scores any other H. */
CLHA_API clha_status clha_quantize(clha_ctx* ctx, const float* U, int n_u, const void* W, clha_dtype dtype,
                          int batch, int d_out, int d_in, const clha_quant_params* params,
                          uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                          const double* lambda, double* loss);
/* clha_quantize with the factor in the given form (CLHA_FACTOR_BLOCK_CHOL: F from
 * clha_factor_groups_as). Under F the lazy and trailing updates take W_hat - W of the earlier columns
 * in place of their scaled errors; the grid, the codes, W_hat and the loss are defined exactly as in
 * clha_quantize. Arguments, outputs and errors as clha_quantize; an unknown form is
 * CLHA_ERR_INVALID_ARG. */
CLHA_API clha_status clha_quantize_as(clha_ctx* ctx, clha_factor_form form, const float* F, int n_u, const void* W,
                                      clha_dtype dtype, int batch, int d_out, int d_in,
                                      const clha_quant_params* params, uint8_t* codes, float* scales, uint8_t* zeros,
                                      float* W_hat, const double* lambda, double* loss);

/* Loss of the CLHA page §2.1, one term: loss_out[b] = tr[(W_hat - W) H (W_hat - W)^T] for `batch`
 * problems; H holds n_h matrices and problem b uses H[b % n_h] (1 <= n_h <= batch). Tile sums are
 * added in float64.
 * loss_out is a host double [batch] array (synchronises). */
CLHA_API clha_status clha_loss(clha_ctx* ctx, const void* W, clha_dtype dtype, const float* W_hat,
                      const float* H, int n_h, int batch, int d_out, int d_in, double* loss_out);

/* ------------------------------------------------------------------------------ analysis */

#define CLHA_DIVERGENCE_MAX_LAYERS 1024

/* Cross-layer routing divergence. The CLHA page (§4, the routing-sharpness experiment, and §5)
 * relates CLHA's gains to the divergence of routing across the layers that share experts but gives
 * no formula; it is read as the total-variation distance of two layers' expert frequencies:
 *   tv[a * n_layers + b] = 1/2 sum_e |n_{a,e} / N_a - n_{b,e} / N_b|,  N_l = sum_e n_{l,e},
 * over the experts e in [slot0, slot0 + E) of `counts`, a device int64 [n_layers, ld] array (an
 * accumulator's counts from clha_accum_buffers, ld = its slot count). tv is a caller-owned device
 * double [n_layers, n_layers] array, symmetric with a zero diagonal, values in [0, 1]. The sums are
 * exact 64-bit integer arithmetic and the one division is float64: the correctly rounded value
 * while 2 N_a N_b <= 2^53. Nothing synchronises. Errors, recorded on the device and returned by the
 * next synchronising call or clha_check: a layer without tokens in the range gives CLHA_ERR_EMPTY, a
 * count outside [0, 2^31) or N_l >= 2^31 gives CLHA_ERR_INVALID_ARG; the entries of such a layer's
 * pairs are NaN. */
CLHA_API clha_status clha_routing_divergence(clha_ctx* ctx, const int64_t* counts, int n_layers, int ld, int slot0,
                                             int E, double* tv);

/* ----------------------------------------------------------------------- multi-GPU exchange */

/* Packed upper triangles of a batch of Gram sums, for the token-sharded collection's exchange
 * between GPUs (the CLHA page, §2.2 (1): the Hessians are sums over tokens, so GPUs that collect
 * disjoint token shares add their partial sums; S is symmetric and only its upper triangle is read,
 * so only d(d+1)/2 floats per matrix need to cross). The matrices are S + (o * outer_stride + i) * d * d
 * for o < n_outer, i < n_inner (outer_stride >= n_inner, in matrices; e.g. the slots [e0, e0 + n) of
 * every layer of an accumulator: S = the accumulator's S at slot e0, n_outer = its layers,
 * outer_stride = its slot count, n_inner = n). packed holds them in (o, i) order, each as rows
 * i = 0 .. d-1 of entries (i, i .. d-1): d(d+1)/2 floats per matrix. clha_unpack_upper writes the
 * upper triangles back and leaves the strict lower triangles as they were. Device pointers, the
 * caller's; nothing synchronises. */
CLHA_API clha_status clha_pack_upper(clha_ctx* ctx, const float* S, int64_t n_outer, int64_t outer_stride,
                                     int64_t n_inner, int d, float* packed);
CLHA_API clha_status clha_unpack_upper(clha_ctx* ctx, const float* packed, int64_t n_outer, int64_t outer_stride,
                                       int64_t n_inner, int d, float* S);

#ifdef __cplusplus
}
#endif

#endif /* CLHA_H */
