/*
 * compkv.h -- C ABI of the CompKV decode hot path on NVIDIA B200 (sm_100a).
 *
 * CompKV (compensation-aware KV selection; abstract of arXiv 2609.26300 and the Evolve.pub review
 * of it) cuts the KV cache into fixed-size token blocks, keeps per-block summaries (mean key,
 * grouped key variance, mean value), scores every block by the residual that block-mean ("Mean")
 * compensation would leave if it were omitted, keeps the top blocks up to a token budget and runs
 * exact attention over them, with every omitted block folded into the same softmax as its
 * block-mean logit, weighted by its token count, carrying its mean value.
 *
 * Conventions for every call below
 *   - Pointers named as device memory are CUDA device pointers owned by the caller; the library
 *     allocates no memory, keeps no per-call state on the host and never synchronises the stream.
 *     Host pointers are named as such.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every call is
 *     asynchronous on it; the outputs are ready when the stream reaches that point.
 *   - Layouts are dense, row-major, in the order given: [B, Hkv, T, d] means d fastest.
 *   - Device pointers of q, K, V and of the float summaries must be 16-byte aligned.
 *   - Return value: COMPKV_OK (0) or a negative compkv_status. Arguments are validated on the host
 *     before any launch; on failure nothing is launched and outputs are untouched. A launch failure
 *     returns COMPKV_ERR_CUDA (see compkv_last_cuda_error). Kernels never trap: a kernel that gives
 *     up an internal wait records COMPKV_DEVERR_* in the workspace status word
 *     (compkv_read_device_status) and returns.
 *
 * Notation: B batch, Hq query heads, Hkv kv-heads, G = Hq / Hkv query heads per kv-head, d head
 * dim, T context length, block size 16, N_b = ceil(T / 16) blocks, r key-variance groups,
 * K_b = min(floor(budget / 16), N_b) selected blocks, s the softmax scale.
 */
#ifndef COMPKV_H
#define COMPKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define COMPKV_VERSION 1

/* Problem shape of one attention layer. */
typedef struct compkv_shape {
  int32_t batch;      /* B >= 1                                                                */
  int32_t n_q_heads;  /* Hq >= 1                                                               */
  int32_t n_kv_heads; /* Hkv >= 1; Hq % Hkv == 0 and G = Hq / Hkv in {1, 2, 4, 8}              */
  int32_t head_dim;   /* d in {64, 128}                                                        */
  int32_t ctx_len;    /* T >= 1: tokens per sequence, or the cache capacity when ctx_lens is   */
                      /* given                                                                 */
  int32_t block_size; /* must be 16                                                            */
  int32_t n_groups;   /* r: a power of two with 1 <= r <= d (default 4)                        */
  int32_t summary_dtype; /* compkv_summary_dtype of mean_k and mean_v (0 = fp32)                */
} compkv_shape;

/* Storage type of the mean key and mean value summaries (the grouped variances stay fp32, the
 * counts int32). FP16 halves the bytes the score pass streams; values are rounded to nearest
 * even when stored and computed on in fp32. */
typedef enum compkv_summary_dtype { COMPKV_SUMMARY_FP32 = 0, COMPKV_SUMMARY_FP16 = 1 } compkv_summary_dtype;

/* Element type of q, K and V (summaries and outputs are always fp32). */
typedef enum compkv_dtype { COMPKV_BF16 = 0, COMPKV_FP32 = 1 } compkv_dtype;

/* Selection rule.
 *   COMPKV_MODE_COMPKV     compensation-aware score (mass x within-block logit variance) and
 *                          Mean compensation of the omitted blocks (the method).
 *   COMPKV_MODE_MASS       attention-mass Top-K, omitted blocks dropped: the rule that removing
 *                          compensation recovers (review, Key claims / Strengths, App. A.5).
 *   COMPKV_MODE_MASS_COMP  mass Top-K followed by Mean compensation: the decoupled
 *                          select-then-compensate design the method argues against (review,
 *                          Summary and FAQ on Quest+RESA).                                     */
typedef enum compkv_mode {
  COMPKV_MODE_COMPKV = 0,
  COMPKV_MODE_MASS = 1,
  COMPKV_MODE_MASS_COMP = 2
} compkv_mode;

typedef enum compkv_status {
  COMPKV_OK = 0,
  COMPKV_ERR_INVALID_ARG = -1,        /* null pointer, bad enum, budget, size                   */
  COMPKV_ERR_UNSUPPORTED_SHAPE = -2,  /* d, G, r, block size outside the supported set          */
  COMPKV_ERR_BAD_ALIGNMENT = -3,      /* a pointer that must be 16-byte aligned is not          */
  COMPKV_ERR_WORKSPACE_TOO_SMALL = -4,
  COMPKV_ERR_CUDA = -5                /* a CUDA runtime call or launch failed                   */
} compkv_status;

/* Device status bits recorded in the workspace status word by a kernel. */
#define COMPKV_DEVERR_WAIT_TIMEOUT 0x1 /* an mbarrier wait gave up after its iteration limit   */
#define COMPKV_DEVERR_BAD_POSITION 0x2 /* compkv_append: a position outside [0, T); skipped     */

/* ------------------------------------------------------------------------------------------ */
/* Sizes                                                                                       */

/* K_b = min(floor(budget_tokens / block_size), N_b): the number of exactly attended blocks per
 * (sequence, kv-head) (budget counts exact tokens only; compensation terms are free). Returns a
 * negative status for an invalid shape or budget < 0. */
int32_t compkv_num_selected(const compkv_shape* shape, int32_t budget_tokens);

/* Bytes of device workspace that compkv_score_select / compkv_sparse_decode / compkv_decode_step
 * need for this shape and budget. 0 on an invalid shape. The workspace carries, between
 * compkv_score_select and compkv_sparse_decode on one stream, the Mean-compensation partial sums
 * over all blocks, the split partials and the merge counters. It must be zero-filled once before
 * its first use (e.g. cudaMemsetAsync); the library keeps the counters at zero between calls. */
size_t compkv_workspace_bytes(const compkv_shape* shape, int32_t budget_tokens);

/* Bytes of device workspace for compkv_full_decode (same zero-fill rule). */
size_t compkv_full_workspace_bytes(const compkv_shape* shape);

/* ------------------------------------------------------------------------------------------ */
/* a0. Block summaries (once per prefill).
 * CompKV review, Summary ("mean key, grouped key variance (default r=4), mean value") and FAQ
 * ("2d+r+1 scalars per block"). For block j of sequence b, kv-head g, with tokens
 * [16j, min(16j+16, T_b)):
 *   count[j]      n_j, tokens in the block (0 for blocks past T_b)
 *   mean_k[j, :]  mu_j = (1/n_j) sum_t k_t
 *   var_g[j, q]   (1/|C_q|) sum_{c in C_q} (1/n_j) sum_t (k_{t,c} - mu_{j,c})^2, C_q the q-th of r
 *                 contiguous groups of d/r channels (population variances)
 *   mean_v[j, :]  nu_j = (1/n_j) sum_t v_t
 * Blocks with n_j = 0 get zeros.
 *   K, V      device, [B, Hkv, T, d] of `dtype`, read once
 *   ctx_lens  device int32 [B] (T_b, 1..T) or NULL for T_b = T
 *   mean_k, mean_v  device [B, Hkv, N_b, d] of shape->summary_dtype (fp32 or fp16);
 *                   var_g device fp32 [B, Hkv, N_b, r];
 *   count     device int32 [B, Hkv, N_b]                                                       */
int compkv_build_summaries(const compkv_shape* shape, compkv_dtype dtype, const void* K,
                           const void* V, const int32_t* ctx_lens, void* mean_k, float* var_g,
                           void* mean_v, int32_t* count, void* stream);

/* a0, incremental. One new token per sequence enters the cache: its key and value update the
 * summaries of the block that receives it (CompKV review, Frequently asked questions: the
 * per-block summaries are "updated incrementally as new tokens enter the cache"). For each
 * sequence b and kv-head g, with t = positions[b] and j = t / 16 (n = count[j] before the call):
 *   n' = n + 1;  mu' = mu + (k - mu) / n';  nu' = nu + (v - nu) / n';
 *   var_g[j, q]' = (n |C_q| var_g[j, q] + sum_{c in C_q} (k_c - mu_c)(k_c - mu'_c)) / (n' |C_q|)
 * (Welford's update of the per-channel sums of squared deviations, summed over each group; exact
 * from the stored (n, mu, var_g) because of the population-variance reading of var_g). A block
 * with n = 0 becomes the token itself with zero variance. The caller appends tokens in order:
 * t must be the sequence's current length, and every block before j must be full.
 *   k_new, v_new  device [B, Hkv, d] of `dtype`: the new token's key and value
 *   positions     device int32 [B]: t per sequence (the length before this token)
 *   K, V          device [B, Hkv, T, d] caches of capacity T = shape->ctx_len, or NULL; when
 *                 given, the token is also stored at row t
 *   mean_k, var_g, mean_v, count   summaries as for compkv_build_summaries, updated in place
 *   status        device int32 or NULL: a sequence with t outside [0, T) is skipped and
 *                 COMPKV_DEVERR_BAD_POSITION is OR-ed into *status
 * One warp per (sequence, kv-head); no workspace.                                              */
int compkv_append(const compkv_shape* shape, compkv_dtype dtype, const void* k_new,
                  const void* v_new, const int32_t* positions, void* K, void* V, void* mean_k,
                  float* var_g, void* mean_v, int32_t* count, int32_t* status, void* stream);

/* a1 + a2. Compensation-aware score and Top-K selection, per (sequence, kv-head).
 * CompKV review, Summary (Section 3, Eq. 4-7: the residual of an omitted block is governed by its
 * attention mass and within-block logit variance; scored from the summaries "with a second-order
 * mass estimate") and Key claims. For query head h of kv-head g and block j with n_j > 0:
 *   lbar = s q_h . mu_j;  V = s^2 sum_q |q_{h,C_q}|^2 var_g[j,q];
 *   m = n_j exp(lbar) (1 + V/2);  Zhat_h = sum_j m;
 *   score_h = (m / Zhat_h) (V / 2)   [MODE_COMPKV]     or   m / Zhat_h   [MODE_MASS, MASS_COMP];
 *   S_j = sum over the G heads of g of score_h.
 * sel_idx gets the K_b blocks with the largest S_j (equal S: lower j first), ascending. Blocks
 * with n_j = 0 rank below every other block. In the compensating modes the call also accumulates,
 * into the workspace, every block's Mean-compensation term (logit lbar + log n_j, value nu_j)
 * under one running max per head; compkv_sparse_decode consumes it.
 *   q          device [B, Hq, d] of `dtype`
 *   mean_k, var_g, mean_v, count   summaries from compkv_build_summaries (mean_v may be NULL in
 *              MODE_MASS)
 *   budget_tokens  >= 0 (K_b may be 0 only in the compensating modes)
 *   softmax_scale  s; <= 0 selects 1/sqrt(d)
 *   sel_idx    device int32 [B, Hkv, K_b], ascending block indices
 *   scores     device fp32 [B, Hkv, N_b] receives S_j, or NULL
 *   workspace  device, >= compkv_workspace_bytes(shape, budget_tokens)                         */
int compkv_score_select(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                        const void* q, const void* mean_k, const float* var_g,
                        const void* mean_v, const int32_t* count, int32_t budget_tokens,
                        float softmax_scale, int32_t* sel_idx, float* scores, void* workspace,
                        size_t workspace_bytes, void* stream);

/* a1, first pass alone: the streaming pass of compkv_score_select over every block's summaries,
 * without the selection. It leaves in the workspace each block's per-head log score and mean
 * logit record and the per-segment partials of Zhat and of the compensation sum; nothing else is
 * written. Exposed so that the pass that reads all the summaries (the bandwidth-bound part of the
 * step) can be timed on its own; a following compkv_score_select recomputes everything it needs.
 * Arguments as for compkv_score_select.                                                       */
int compkv_score_stream(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                        const void* q, const void* mean_k, const float* var_g,
                        const void* mean_v, const int32_t* count, int32_t budget_tokens,
                        float softmax_scale, void* workspace, size_t workspace_bytes,
                        void* stream);

/* a3. Exact attention over the selected blocks plus Mean compensation, in one softmax.
 * CompKV abstract ("computing exact attention over a selected subset", compensation of "the
 * omitted attention tail") and review, Summary ("omitted blocks contribute their block-mean
 * logit"). For query head h:
 *   out_h = [ sum_{j in Sel} sum_{t in j} e^{l_t - M} v_t + sum_{j not in Sel} n_j e^{lbar_j - M} nu_j ]
 *         / [ sum_{j in Sel} sum_{t in j} e^{l_t - M}     + sum_{j not in Sel} n_j e^{lbar_j - M} ]
 * with l_t = s q_h . k_t; the omitted terms are absent in MODE_MASS. Must follow
 * compkv_score_select on the same stream with the same workspace, shape, mode and budget; sel_idx
 * may be any ascending or unordered set of K_b distinct valid block indices (e.g. the one
 * score_select wrote).
 *   K, V      device [B, Hkv, T, d] of `dtype`; only the selected blocks are read
 *   mean_k, mean_v, count  summaries (only the selected blocks' rows are read here)
 *   out       device fp32 [B, Hq, d]                                                          */
int compkv_sparse_decode(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                         const void* q, const void* K, const void* V, const void* mean_k,
                         const void* mean_v, const int32_t* count, const int32_t* sel_idx,
                         int32_t budget_tokens, float softmax_scale, float* out, void* workspace,
                         size_t workspace_bytes, void* stream);

/* One whole decode step: the result of compkv_score_select followed by compkv_sparse_decode, in
 * two kernels: the streaming score pass, then one kernel that selects and attends (launched with
 * programmatic dependent launch so its prologue overlaps the first's tail; the selection is kept
 * on chip and also written to sel_idx). Arguments as above. */
int compkv_decode_step(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                       const void* q, const void* K, const void* V, const void* mean_k,
                       const float* var_g, const void* mean_v, const int32_t* count,
                       int32_t budget_tokens, float softmax_scale, int32_t* sel_idx,
                       float* scores, float* out, void* workspace, size_t workspace_bytes,
                       void* stream);

/* a4. Dense baseline: exact softmax attention over all T_b tokens (the full attention the
 * speedup is quoted against; review, Key claims and FAQ, Table 4).
 *   q device [B, Hq, d]; K, V device [B, Hkv, T, d]; ctx_lens device int32 [B] or NULL;
 *   out device fp32 [B, Hq, d]; workspace >= compkv_full_workspace_bytes(shape).              */
int compkv_full_decode(const compkv_shape* shape, compkv_dtype dtype, const void* q,
                       const void* K, const void* V, const int32_t* ctx_lens, float softmax_scale,
                       float* out, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Allocation-free decode step. This entry point has no counterpart in the CompKV paper or its  */
/* review; it is a deployment convenience of this library.                                      */

/* Size of the scratch array inside the library that compkv_decode_step_static uses. */
#define COMPKV_STATIC_SCRATCH_BYTES (16u << 20)

/* compkv_decode_step for callers that cannot allocate device memory: for example code that runs
 * inside a host engine which owns every device allocation and only hands out input and output
 * buffers, or a path where calling cudaMalloc (and the device synchronisation it can cause) is
 * not allowed. Instead of a caller workspace it uses a scratch array of
 * COMPKV_STATIC_SCRATCH_BYTES compiled into the library as static device memory; every GPU that
 * loads the library keeps that array until the process exits. The call itself allocates nothing:
 * no cudaMalloc, no cudaFree, no allocating library routine.
 *   - Shapes whose compkv_workspace_bytes(shape, budget_tokens) exceeds
 *     COMPKV_STATIC_SCRATCH_BYTES are rejected with COMPKV_ERR_WORKSPACE_TOO_SMALL before any
 *     launch (the 128K-context, 8-kv-head layer needs about 4 MB).
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, a host-side lookup once the library's device code is loaded; the
 *     first call on a device may load it, so make that first call before any stream capture).
 *   - Every call shares the one array, which keeps the previous call's contents. Nothing in it has
 *     to start at zero (each call overwrites what it reads). A kernel that gives up an internal
 *     wait records it in the array's status word, which compkv_static_read_device_status reads
 *     and clears. Calls that can overlap on the GPU (other streams, other host threads) race on
 *     the array: the caller must serialise them.
 * Arguments and outputs are those of compkv_decode_step without workspace and workspace_bytes. */
int compkv_decode_step_static(const compkv_shape* shape, compkv_dtype dtype, compkv_mode mode,
                              const void* q, const void* K, const void* V, const void* mean_k,
                              const float* var_g, const void* mean_v, const int32_t* count,
                              int32_t budget_tokens, float softmax_scale, int32_t* sel_idx,
                              float* scores, float* out, void* stream);

/* compkv_read_device_status for the scratch array of compkv_decode_step_static on the current
 * device: copies its status word (COMPKV_DEVERR_* bits, 0 = clean) to *status (host) and clears
 * it. Synchronises `stream`; allocates nothing. */
int compkv_static_read_device_status(void* stream, int32_t* status);

/* ------------------------------------------------------------------------------------------ */
/* Diagnostics                                                                                  */

/* Copies the workspace status word (COMPKV_DEVERR_* bits, 0 = clean) to *status (host) and
 * clears it. Synchronises `stream`. */
int compkv_read_device_status(void* workspace, void* stream, int32_t* status);

/* Static, NUL-terminated description of a compkv_status value. */
const char* compkv_status_string(int status);

/* Text of the last CUDA error seen by a call on this host thread ("" if none). */
const char* compkv_last_cuda_error(void);

/* COMPKV_VERSION of the built library. */
int compkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* COMPKV_H */
