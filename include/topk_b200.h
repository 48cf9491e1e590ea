/*
 * topk_b200.h -- C ABI of the B200 (sm_100a) bucketed approximate top-k library.
 *
 * Method: "Approximate Top-k for Increased Parallelism" (Key, Ribar, Cattaneo,
 * Hudlass-Galley, Orr; arXiv 2412.04358), pith.science review page, section
 * "What carries the argument" and Fig. 2: a row of n scores is split into b
 * interleaved buckets (element i goes to bucket i mod b, "The reading"), an
 * exact top-k_b is kept per bucket (Stage 1), and when the b*k_b candidates
 * exceed k a final exact top-k keeps the k best (Stage 2).
 *
 * Common conventions
 *   - Every pointer argument named *_dev is CUDA device memory owned by the
 *     caller; the library keeps no pointer after the call returns.
 *   - Matrices are row-major and contiguous: row r of an [rows x n] array
 *     starts at element r*n.
 *   - Total order: a larger value ranks first; equal values (IEEE equality, so
 *     -0.0 ties +0.0) rank by lower index; NaN ranks above +inf and all NaNs
 *     are equal.
 *   - Outputs out_vals[rows*k] / out_idx[rows*k] hold, per row, the selected
 *     elements best-first.  When fewer than k elements are selected (fewer
 *     candidates than k, or n < k), the remaining slots hold -inf and -1.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Argument errors are detected on the host before any
 *     work is queued; nothing throws across the ABI.
 *   - The workspace (when required) is caller-owned device memory of at least
 *     topk_workspace_bytes(...) bytes that MUST be zero-filled before its first
 *     use.  Every call leaves it zero-filled again when it completes on the GPU,
 *     so one workspace can be reused for any later call.  Calls that overlap on
 *     the GPU (different streams) must not share a workspace.
 *   - Device-side waits are bounded in time; a wait that expires records a
 *     code readable with topk_device_status() and the kernel returns early.
 */
#ifndef TOPK_B200_H
#define TOPK_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TOPK_OK = 0,          /* queued successfully */
    TOPK_EINVAL = 1,      /* bad argument: null pointer, size < 1, k_b outside [1,4], n >= 2^31 */
    TOPK_EUNSUPPORTED = 2,/* valid but outside what this build implements (see each call) */
    TOPK_ECUDA = 3,       /* a CUDA call or kernel launch failed */
    TOPK_EWORKSPACE = 4,  /* workspace missing or smaller than topk_workspace_bytes() */
    TOPK_ESCRATCH = 5     /* topk_bucketed_noalloc: the call needs more scratch than the
                             library's built-in buffer holds (TOPK_NOALLOC_SCRATCH_BYTES) */
} topk_status;

typedef enum {
    TOPK_OP_BUCKETED = 0,
    TOPK_OP_EXACT = 1,
    TOPK_OP_SCORE = 2,
    TOPK_OP_BUCKETED_BF16 = 3
} topk_op;

/* Bytes of workspace a call of `op` with these sizes needs on the current
 * device (0 when none).  Unused arguments are ignored (d for BUCKETED/EXACT,
 * b and kb for EXACT).  Returns 0 as well for invalid sizes. */
size_t topk_workspace_bytes(int op, int64_t rows, int64_t n, int k, int b, int kb, int d);

/* Two-stage bucketed approximate top-k ("What carries the argument"; Fig. 2).
 *   scores_dev  [rows x n] float32 scores.
 *   k           number of outputs per row, 1 <= k <= 16384.
 *   b           number of interleaved buckets, 1 <= b <= 1024.
 *   kb          candidates kept per bucket, 1 <= kb <= 4 (register queues).
 *   out_vals_dev[rows x k] float32: the selected scores (input bits unchanged).
 *   out_idx_dev [rows x k] int32: their column indices.
 * The result equals the CPU definition bit for bit.  Fast path: n % 4 == 0,
 * scores 16-byte aligned and b dividing 1024; other shapes take a slower
 * general path.  Returns TOPK_EUNSUPPORTED for b > 1024 or k > 16384. */
int topk_bucketed(const float *scores_dev, int64_t rows, int64_t n, int k, int b, int kb,
                  float *out_vals_dev, int32_t *out_idx_dev, void *workspace_dev,
                  size_t workspace_bytes, void *stream);

/* topk_bucketed on bfloat16 score rows: the same selection on half the bytes
 * (the page compares the two precisions in Fig. 10, "Bandwidth comparison for
 * bfloat16 values").
 *   scores_dev   [rows x n] bf16 (raw 16-bit patterns).
 *   out_vals_dev [rows x k] bf16: the selected scores, input bits unchanged
 *                (padding slots hold -inf, 0xFF80).
 * bf16 values are ordered as the floats they represent, with the same total
 * order (ties by lowest index, -0 ties +0, NaN above +inf).  Fast path: n % 8
 * == 0, 16-byte aligned rows, b dividing 1024.  Workspace:
 * topk_workspace_bytes(TOPK_OP_BUCKETED_BF16, ...); other arguments and
 * errors as topk_bucketed. */
int topk_bucketed_bf16(const uint16_t *scores_dev, int64_t rows, int64_t n, int k, int b, int kb,
                       uint16_t *out_vals_dev, int32_t *out_idx_dev, void *workspace_dev,
                       size_t workspace_bytes, void *stream);

/* Exact top-k of every row under the total order above: the baseline the
 * page compares against (Fig. 1, "exact top-k implementations") and the
 * Stage-2 primitive.  1 <= k <= 16384 (else TOPK_EUNSUPPORTED).  No workspace:
 * pass NULL / 0. */
int topk_exact(const float *scores_dev, int64_t rows, int64_t n, int k, float *out_vals_dev,
               int32_t *out_idx_dev, void *workspace_dev, size_t workspace_bytes, void *stream);

/* Bucketed top-k over candidate lists: the merge step of a row cut into
 * column slices (several CTAs, or several GPUs that each hold part of a
 * vocabulary or an entity table).  The bucket of a pair is its GLOBAL index
 * modulo b, as for a single pass over the whole row ("What carries the
 * argument"; bucket = i mod b per "The reading"); each bucket keeps its top
 * kb pairs and the final exact top-k keeps the k best, with the total order
 * above.  When part p's lists are topk_bucketed of columns
 * [part_offset[p], part_offset[p] + n_p) of the same rows (local indices),
 * the result equals topk_bucketed of the whole rows bit for bit.
 *   vals_dev [parts x rows x m] float32 and idx_dev [parts x rows x m] int32:
 *                per part and row, m (value, index) pairs; index -1 marks an
 *                empty slot (as topk_bucketed pads).  Indices of one row must
 *                be distinct after the offsets are added.
 *   parts        1 <= parts <= 64 (else TOPK_EUNSUPPORTED).
 *   part_offset  HOST array [parts] added to every index of that part; NULL
 *                means all zero.  0 <= part_offset[p] < n_total.
 *   n_total      length of the whole rows, 1 <= n_total < 2^31.  A pair whose
 *                global index is >= n_total is skipped and sets
 *                TOPK_DEV_BAD_INDEX in the device status.
 *   k, b, kb     as in topk_bucketed; out_vals_dev / out_idx_dev [rows x k]
 *                best-first with global indices and the input value bits,
 *                padded with -inf / -1.
 * No workspace.  Asynchronous on `stream`. */
int topk_bucketed_merge(const float *vals_dev, const int32_t *idx_dev, int parts, int64_t rows,
                        int m, const int64_t *part_offset, int64_t n_total, int k, int b, int kb,
                        float *out_vals_dev, int32_t *out_idx_dev, void *stream);

/* Exact re-ranking of a candidate index set ("Recall Before You Rank",
 * abstract: the supports retrieved for similar earlier queries are reused as
 * candidates and scored exactly against the current query before the top-K
 * is kept).  For row r: score_i = sum_t q[r][t] * K_r[i][t] (bf16 inputs,
 * fp32 accumulation, no 1/sqrt(d)) for every DISTINCT index 0 <= i < n among
 * cand_idx[r][0..c); the k best (score, index) pairs under the total order
 * above, best-first, padded with -inf / -1.
 *   q_dev, K_dev, d, n, k_batch_stride  as in score_topk (d 128 or 256;
 *                16-byte aligned; k_batch_stride a multiple of 8).
 *   cand_idx_dev [rows x c] int32 candidate indices: -1 marks an empty slot,
 *                repeats are scored once, an index >= n is skipped and sets
 *                TOPK_DEV_BAD_INDEX.  1 <= c <= 4096 (else TOPK_EUNSUPPORTED).
 *   out_scores_dev  nullable [rows x c] float32: the fp32 score of each slot
 *                (-inf for empty, repeated or skipped slots), for checking.
 * Values are the fp32 scores (zero as +0.0, NaN as 0x7FFFFFFF).  No
 * workspace.  Asynchronous on `stream`. */
int score_rerank(const uint16_t *q_dev, int64_t rows, int d, const uint16_t *K_dev, int64_t n,
                 int64_t k_batch_stride, const int32_t *cand_idx_dev, int c, int k,
                 float *out_vals_dev, int32_t *out_idx_dev, float *out_scores_dev, void *stream);

/* Sampling tail of top-k vocabulary sampling (the review page's "Core claim"
 * and Fig. 4, left: vocabulary sampling keeps the top k of n logits).  The
 * pages leave the tail implicit; this is plain top-k sampling.  For each row
 * of selected pairs (best-first, as the selection calls write them), index
 * idx[i] is drawn with probability w_i / sum_j w_j, w_i = exp((v_i - v_0)/T),
 * by inverse CDF with the caller's uniform u[r] in [0, 1): the first i whose
 * running sum of w exceeds u[r] * sum w (else, from rounding, the last entry
 * of positive weight).  Padding (index -1) and -inf values weigh 0.  A row
 * whose best value is NaN or +inf draws idx[0]; a row with no candidate
 * draws -1.  Weights and sums are fp32.
 *   vals_dev, idx_dev  [rows x k] selected values / indices (device).
 *   temperature        T > 0 with 1/T finite (else TOPK_EINVAL).
 *   u_dev              [rows] float32 uniforms in [0, 1), supplied by the
 *                      caller (the library draws no random numbers).
 *   token_dev          [rows] int32 output.
 * No workspace.  Asynchronous on `stream`. */
int topk_sample_rows(const float *vals_dev, const int32_t *idx_dev, int64_t rows, int k,
                     float temperature, const float *u_dev, int32_t *token_dev, void *stream);

/* topk_bucketed with the draw of topk_sample_rows fused into it: the CTA
 * that finishes a row's selection draws that row's token right away, so the
 * selection and the sampling tail of vocabulary sampling take one kernel.
 * Arguments as in those two calls (float32 logits); out_vals_dev /
 * out_idx_dev receive the selection, token_dev the draws. */
int topk_sample(const float *logits_dev, int64_t rows, int64_t n, int k, int b, int kb,
                float temperature, const float *u_dev, int32_t *token_dev, float *out_vals_dev,
                int32_t *out_idx_dev, void *workspace_dev, size_t workspace_bytes, void *stream);

/* topk_sample on bfloat16 logits (raw 16-bit patterns): the selection of
 * topk_bucketed_bf16 with the same fused draw; a bf16 logit widens to fp32
 * exactly before the softmax.  out_vals_dev receives bf16 bits. */
int topk_sample_bf16(const uint16_t *logits_dev, int64_t rows, int64_t n, int k, int b, int kb,
                     float temperature, const float *u_dev, int32_t *token_dev,
                     uint16_t *out_vals_dev, int32_t *out_idx_dev, void *workspace_dev,
                     size_t workspace_bytes, void *stream);

/* Fused selector: score[r][i] = sum_t q[r][t] * K_r[i][t] (bf16 inputs, fp32
 * accumulation; no 1/sqrt(d) scaling), then topk_bucketed on each row of
 * scores -- the sparse-attention selector that scores the current query
 * against the whole key cache before a global top-K ("Recall Before You Rank"
 * abstract; STARC page, Fig. 3: q in R^{1 x d_h}, K in R^{L x d_h}).  The
 * score matrix is not materialised.
 *   q_dev        [rows x d] bf16 (raw 16-bit patterns), 16-byte aligned.
 *   K_dev        bf16 keys; row r uses K_r = K_dev + r*k_batch_stride
 *                elements, an [n x d] row-major matrix.  k_batch_stride = 0
 *                shares one key matrix between all rows.  16-byte aligned.
 *   d            128 or 256 (else TOPK_EUNSUPPORTED).
 *   k, b, kb     as in topk_bucketed, with b dividing 1024 (else
 *                TOPK_EUNSUPPORTED).
 *   out_scores_dev  nullable [rows x n] float32: when given, receives the
 *                fp32 scores the selection ran on (for checking).
 * Output values are the fp32 scores (a zero score is returned as +0.0 and a
 * NaN score as the quiet NaN 0x7FFFFFFF). */
int score_topk(const uint16_t *q_dev, int64_t rows, int d, const uint16_t *K_dev, int64_t n,
               int64_t k_batch_stride, int k, int b, int kb, float *out_vals_dev,
               int32_t *out_idx_dev, float *out_scores_dev, void *workspace_dev,
               size_t workspace_bytes, void *stream);

/* Allocation-free form of topk_bucketed.  The paper has no counterpart: this
 * entry point exists for callers that must not allocate device memory at call
 * time -- for example a serving loop in which a cudaMalloc could synchronise
 * the device and stall every other stream, a host framework whose memory
 * accounting forbids allocations it did not make itself, or a plugin that may
 * only allocate while it is being set up.  Such callers pass inputs and
 * outputs as for topk_bucketed, but no workspace: the scratch memory the
 * kernel needs for rows split across CTAs lives in one static device buffer
 * of TOPK_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.
 *   - Nothing is allocated and no allocating routine is called: no cudaMalloc,
 *     cudaFree or library allocator.
 *   - The first call on a device looks up that device's address of the buffer
 *     (with the device current); make that first call before any stream
 *     capture begins on the device.  The address is kept per device and
 *     context: after a device reset the first call in the new context looks
 *     it up again, with the same rule on capture.
 *   - A call whose scratch need exceeds the buffer returns TOPK_ESCRATCH and
 *     queues nothing; topk_workspace_bytes(TOPK_OP_BUCKETED, ...) tells the
 *     need in advance.
 *   - Every call on a device shares the one buffer and it keeps the previous
 *     call's contents; the part that must start at zero is cleared on
 *     `stream` at the start of each call.  Calls that overlap on the GPU
 *     (different streams, no ordering between them) race on the buffer and
 *     give wrong results: order them, or use topk_bucketed with one workspace
 *     per stream.
 * Results are identical to topk_bucketed's. */
#define TOPK_NOALLOC_SCRATCH_BYTES (32u << 20)
int topk_bucketed_noalloc(const float *scores_dev, int64_t rows, int64_t n, int k, int b, int kb,
                          float *out_vals_dev, int32_t *out_idx_dev, void *stream);

/* Self-test of the bounded waits (no counterpart in the paper): one thread
 * waits, for at most limit_ns nanoseconds (1e3 .. 2e9, else TOPK_EINVAL), on
 * a barrier that nothing completes, gives up and records TOPK_DEV_WAIT_TIMEOUT
 * in the device status, exactly as an expired wait of a selection kernel does.
 * The GPU neither faults nor hangs and the context stays usable; it lets a
 * caller check its error handling for expired waits.  Asynchronous on
 * `stream`. */
int topk_selftest_wait_timeout(unsigned long long limit_ns, void *stream);

/* Human-readable name of a topk_status value (static string). */
const char *topk_status_string(int status);

/* Reads and clears the device-side status word of the current device: 0 when
 * no bounded wait has expired since the last read, else a bit set of
 * TOPK_DEV_* codes.  Synchronises the device. */
int topk_device_status(int *status_out);

#define TOPK_DEV_WAIT_TIMEOUT 1 /* a bulk-copy wait in a streaming kernel expired */
#define TOPK_DEV_BAD_INDEX 2    /* topk_bucketed_merge or score_rerank skipped an index out of range */
#define TOPK_DEV_DRAIN_TIMEOUT 4 /* after an expired wait, the kernel's wait for its own bulk copies
                                    still in flight expired too: the kernel returned while a copy
                                    may still have been writing to its shared memory, so the
                                    context must be treated as unusable (reset or exit) */

#ifdef __cplusplus
}
#endif

#endif /* TOPK_B200_H */
