/*
 * pkm.h -- C ABI of the B200 product-key memory (PKM) layer library.
 *
 * The layer (sources: "Large Memory Layers with Product Keys", method-details list
 * and abstract; "Meta AI 可扩展内存层" sections 3.2, 4.3-4.5, 5.1-5.3, 9.2):
 *
 *   F1  q = gamma * (x Wq^T - mean) / sqrt(var + eps) + beta     query network
 *   F2  per head h and half s: scores of q_half against every sub-key of the
 *       half (C for s = 0, C' for s = 1), then the top-k of each half
 *   F3  the k x k Cartesian candidates scored s1[a] + s2[b], the best k kept
 *       (the exact top-k over all C1*C2 product keys), value row i*C2 + j,
 *       w = softmax(score_scale * (s1 + s2)) over the k winners
 *   F4  y[t] = sum_h sum_j w[t][h][j] * V[idx[t][h][j]]
 *   backward: gradients of sum_t dy[t] . y[t] with the selected keys held fixed;
 *       the value gradient is a scatter-add whose duplicate rows are combined
 *       before any write (one writer per row, no atomics, deterministic).
 *
 * Ordering: per half, (score desc, index asc); candidates, (s1+s2 desc, s1 desc,
 * s2 desc, flat index asc).  Scores are fp32 on the device.
 *
 * Conventions shared by every entry point
 *   - Every pointer is a DEVICE pointer unless stated otherwise; the caller owns
 *     all memory.  The library never allocates or frees device memory and never
 *     synchronises, except pkm_check_status.
 *   - All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and is asynchronous.
 *   - Row-major layouts:
 *       x        [N][d_in]            bf16 (fp32 with PKM_F_FP32)
 *       Wq       [h*dk][d_in]         bf16 (fp32 with PKM_F_FP32)  Linear weight, out x in
 *       bn       [4][h*dk]            fp32: running mean, running var, gamma, beta
 *       subkeys  [h][C1+C2][dk/2]     bf16 (fp32 with PKM_F_FP32)  rows [0,C1) = C, [C1,C1+C2) = C'
 *       values   [C1*C2][d_v]         bf16 (fp32 with PKM_F_FP32 or PKM_F_VALUES_FP32)
 *       y, dy    [N][d_v]             fp32
 *   - Gradients of parameters ACCUMULATE (+=) into the caller's buffers; dx is
 *     overwritten.  A NULL gradient pointer skips that gradient.
 *   - Host-side validation happens before any launch and returns an error status
 *     without touching the device.  Device-side problems (a bounded wait that
 *     expired, an out-of-range index) set a status word that pkm_check_status
 *     reports; kernels never trap.
 *   - Limits: 1 <= k <= 64, k <= min(C1, C2), h <= 64, dk/2 <= 1024 (bf16) or 512 (fp32), dk % 32 == 0 (bf16) or dk % 8 == 0
 *     (fp32), d_in % 8 == 0, d_v % 8 == 0, C1*C2 < 2^31, pointers 16-byte aligned.
 *     N == 0 is a no-op returning PKM_OK.
 */
#ifndef PKM_H_
#define PKM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKM_OK = 0,
  PKM_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, bad size, k > C, ... */
  PKM_ERR_UNSUPPORTED = 2,     /* legal but outside this build's limits (k > 64, ...) */
  PKM_ERR_WORKSPACE = 3,       /* workspace pointer NULL or smaller than pkm_workspace_bytes */
  PKM_ERR_CUDA = 4,            /* a CUDA runtime call failed (launch, attribute, ...) */
  PKM_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait expired */
  PKM_ERR_DEVICE_INDEX = 6     /* a device-side index check failed */
} pkm_status;

/* flags */
#define PKM_F_FP32 0x1u  /* x, Wq, subkeys, values are fp32 (CUDA-core kernels) */
#define PKM_F_SIMT 0x2u  /* bf16 storage, but CUDA-core kernels instead of tensor cores */
#define PKM_F_VALUES_FP32 0x4u  /* values (the table) fp32; x, Wq, subkeys stay bf16 */
/* Single-pass scoring: the sub-key scores (so the selection and the weights) take q
 * rounded to bf16 instead of q = hi + lo (half the scoring MMA work; scores move by up
 * to half a bf16 ulp of q per coordinate, ~2e-4 relative).  The sub-key gradient
 * uses the same rounded q; the query gradient passes the rounding unchanged.  bf16
 * storage only (PKM_ERR_INVALID_ARG with PKM_F_FP32). */
#define PKM_F_BF16_Q 0x8u
/* Training-mode BatchNorm on the query: the forward normalises with the batch's own
 * statistics (per column of x Wq^T over the call's N tokens: mean and biased variance),
 * records them in saved->bn_batch and needs saved->qhat; the backward differentiates
 * through them (every token's gradient depends on all tokens).  bn's running mean and
 * variance are not read; pkm_bn_running_update folds a batch into them. */
#define PKM_F_BN_TRAIN 0x10u
/* The all-k^2 variant (the code snippet of "Meta AI 可扩展内存层" section 10): no second
 * top-k -- every one of the k*k candidates top-k(s1) x top-k(s2) is kept, a-major
 * (selection a*k + b pairs the a-th sub-key of the first half with the b-th of the second),
 * and the softmax runs over all of them.  idx, w and dw then hold k*k selections per head:
 * [N][h][k*k] (pkm_saved_bytes accounts for it). */
#define PKM_F_ALL_K2 0x20u
/* Inverse-distance sub-key scores ("Fast-weight Product Key Memory", section 2.2):
 * s = -1/2 log(||q_half - c||^2 + 1e-12) instead of q_half . c; selection and softmax as
 * usual, so the weights fall off as (d1 d2)^(-score_scale).  Scoring and the sub-key /
 * query-half gradients run on the CUDA-core kernels. */
#define PKM_F_IDW 0x40u

typedef struct {
  int64_t N;          /* tokens */
  int32_t d_in;       /* input width */
  int32_t h;          /* heads */
  int32_t dk;         /* query width per head; halves of dk/2 */
  int32_t C1, C2;     /* |C|, |C'| sub-keys per half */
  int32_t k;          /* top-k per half and kept product keys per head */
  int32_t d_v;        /* value width */
  float bn_eps;       /* BatchNorm epsilon (> 0) */
  float score_scale;  /* softmax temperature factor (> 0); selection ignores it */
  uint32_t flags;     /* PKM_F_* */
} pkm_dims;

/* What the forward writes and the backward reads (caller-owned device buffers).
 *   q      bf16 storage: [2][N][h*dk] bf16, the query split as q = hi + lo
 *          (hi = bf16(q), lo = bf16(q - hi)); fp32 storage: [N][h*dk] fp32.
 *   qhat   optional [N][h*dk] fp32 normalised pre-affine query (x Wq^T - mean) /
 *          sqrt(var + eps); needed only for the gamma gradient.  May be NULL.
 *   sub_s  [N][h][2][k] fp32 per-half top-k scores, best first
 *   sub_i  [N][h][2][k] int32 per-half top-k sub-key indices, best first
 *   idx    [N][h][k] int32 selected value rows i*C2 + j, best first
 *   w      [N][h][k] fp32 softmax weights
 *   bn_batch  [2][h*dk] fp32 batch mean and biased batch variance of x Wq^T: written by
 *          the forward and read by the backward with PKM_F_BN_TRAIN (with it, qhat is
 *          required too); otherwise unused and may be NULL.                     */
typedef struct {
  void* q;
  float* qhat;
  float* sub_s;
  int32_t* sub_i;
  int32_t* idx;
  float* w;
  float* bn_batch;
} pkm_saved;

#define PKM_SAVED_Q 0
#define PKM_SAVED_QHAT 1
#define PKM_SAVED_SUB_S 2
#define PKM_SAVED_SUB_I 3
#define PKM_SAVED_IDX 4
#define PKM_SAVED_W 5
#define PKM_SAVED_BN_BATCH 6

#define PKM_FWD 0
#define PKM_BWD 1
#define PKM_FWD_FUSED 2

/* Bytes of one pkm_saved field (PKM_SAVED_*) for these dims; 0 for bad input. */
size_t pkm_saved_bytes(const pkm_dims* d, int field);

/* Bytes of device workspace pkm_forward (which = PKM_FWD) or pkm_backward
 * (PKM_BWD) needs.  The workspace is scratch: its contents on entry are ignored
 * and on return are unspecified.  256-byte alignment is required.
 * which = PKM_FWD_FUSED: the optional forward workspace of few-token calls (0 when it
 * does not apply).  When pkm_forward gets at least this many bytes (N <= 16, bf16
 * storage, eval-mode BatchNorm, dot-product scores, 1 <= k <= 32, dk/2 <= 512, C1 and C2
 * <= 4096), it runs the four steps as one cooperative kernel with grid-wide barriers
 * (one launch instead of four).  Its results agree with the separate kernels' to fp32
 * rounding: the dot products are summed in another order, so keys whose scores tie to
 * within that rounding may be kept or ordered differently.  Every barrier wait is
 * bounded and reports PKM_ERR_DEVICE_TIMEOUT through pkm_check_status; after an expired
 * wait every later fused call on that device reports the timeout and computes nothing.
 * Without the workspace, or when the device cannot hold one CTA per SM, the separate
 * kernels run. */
size_t pkm_workspace_bytes(const pkm_dims* d, int which);

/* Forward F1..F4 ("Large Memory Layers with Product Keys", method details).
 *   bn: [4][h*dk] fp32 (mean, var, gamma, beta).  y: [N][d_v] fp32, overwritten.
 *   saved: every field except qhat must be non-NULL. */
pkm_status pkm_forward(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                       const void* subkeys, const void* values, float* y,
                       const pkm_saved* saved, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Backward of sum_t dy[t].y[t] with the selected keys of `saved` held fixed.
 *   dx       [N][d_in] fp32, overwritten (NULL: skip)
 *   dWq      [h*dk][d_in] fp32, += (NULL: skip)
 *   dbn      [2][h*dk] fp32, += (d gamma, d beta) (NULL: skip; needs saved->qhat)
 *   dsubkeys [h][C1+C2][dk/2] fp32, += (NULL: skip)
 *   dvalues  [C1*C2][d_v] fp32, += dense table; only selected rows are touched
 *            (NULL: skip)
 *   dw_out   optional [N][h][k] fp32: dL/dw per selected key (NULL: skip)   */
pkm_status pkm_backward(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                        const void* subkeys, const void* values, const pkm_saved* saved,
                        const float* dy, float* dx, float* dWq, float* dbn, float* dsubkeys,
                        float* dvalues, float* dw_out, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ---- the backward's two stages; pkm_backward runs both ----
 * (The gradient reaches only the selected value rows and sub-keys: "Meta AI 可扩展内存层"
 * sections 6.1 and 9.2; the query-side chain follows "Large Memory Layers with Product
 * Keys", method details.)
 * Value stage (sort of the selections by value row, then one pass per distinct row):
 *   dw [N][h][k] fp32 out (required), dvalues += (NULL: skip).
 * Query stage (softmax backward onto the selected sub-keys, query-half and sub-key
 * gradients, BatchNorm backward, dense query gradients): reads dw from the value
 * stage.  Both stages take the same workspace (pkm_workspace_bytes(d, PKM_BWD)). */
pkm_status pkm_value_grad(const pkm_dims* d, const void* values, const pkm_saved* saved,
                          const float* dy, float* dvalues, float* dw, void* workspace,
                          size_t workspace_bytes, void* stream);
/* The value stage in its two parts (pkm_value_grad runs both, with the same results):
 * pkm_value_sort sorts saved->idx by value row and leaves the sorted selections, the
 * distinct rows and the weights in row order (gathered from saved->w) in the workspace;
 * pkm_value_rows then runs the pass per distinct row from that workspace.  Between the
 * two calls the workspace belongs to them: nothing else may write it, and the dims must
 * be the same.  pkm_value_sort needs only the forward's selection, so a caller can run it
 * before the upstream gradient exists (e.g. beside the forward's bag on another stream). */
pkm_status pkm_value_sort(const pkm_dims* d, const pkm_saved* saved, void* workspace,
                          size_t workspace_bytes, void* stream);
pkm_status pkm_value_rows(const pkm_dims* d, const void* values, const float* dy,
                          float* dvalues, float* dw, void* workspace, size_t workspace_bytes,
                          void* stream);
pkm_status pkm_query_grad(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                          const void* subkeys, const pkm_saved* saved, const float* dw, float* dx,
                          float* dWq, float* dbn, float* dsubkeys, void* workspace,
                          size_t workspace_bytes, void* stream);

/* ---- the forward's steps, each callable alone (same layouts as above) ---- */

/* F1: writes saved->q (and saved->qhat when non-NULL). */
pkm_status pkm_query(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                     const pkm_saved* saved, void* stream);

/* F2 (pkm_subkey_scores): from saved->q, writes saved->sub_s and saved->sub_i. */
pkm_status pkm_subkey_scores(const pkm_dims* d, const void* subkeys, const pkm_saved* saved,
                             void* stream);

/* F3 (pkm_candidate_topk): from sub_s/sub_i, writes idx and w. */
pkm_status pkm_candidate_topk(const pkm_dims* d, const pkm_saved* saved, void* stream);

/* F4 (pkm_gather_bag): y[t] = sum_h sum_j w * V[idx]; y overwritten. */
pkm_status pkm_gather_bag(const pkm_dims* d, const void* values, const int32_t* idx,
                          const float* w, float* y, void* stream);

/* ---- training-time pieces ("Meta AI 可扩展内存层" sections 6.1, 6.3, 6.4, 11.2) ---- */

/* Running statistics after a training-mode batch (PKM_F_BN_TRAIN forward):
 *   bn[0] <- (1 - momentum) bn[0] + momentum * mean_batch,
 *   bn[1] <- (1 - momentum) bn[1] + momentum * var_batch * N / (N - 1)   (N >= 2),
 * bn [4][h*dk] updated in place (rows 2-3 untouched), bn_batch = saved->bn_batch. */
pkm_status pkm_bn_running_update(const pkm_dims* d, float* bn, const float* bn_batch,
                                 float momentum, void* stream);

/* Value-gradient stage with a compact (sparse-rows) result instead of the dense table:
 * num_rows (device int, written) = U, the number of distinct selected rows;
 * rows_out[u] (ascending) = the u-th distinct row and dvalues_rows[u][:] = its gradient
 * sum over selections (overwritten) for u < U.  Capacity: min(N*h*k, C1*C2) rows.
 * dw [N][h][k] as in pkm_value_grad (NULL: not returned).  Moves d_v*(2 or 4) bytes of
 * V and d_v*4 of result per distinct row, against d_v*(2 or 4) + 8 for the dense form.
 * Workspace: pkm_workspace_bytes(d, PKM_BWD). */
pkm_status pkm_value_grad_rows(const pkm_dims* d, const void* values, const pkm_saved* saved,
                               const float* dy, float* dw, int32_t* rows_out,
                               float* dvalues_rows, int* num_rows, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Lazy Adam on the selected rows only: with g_r = sum over the selections of row r of
 * w * dy[t] (the value gradient of sum_t dy[t] . y[t]),
 *   m_r <- beta1 m_r + (1 - beta1) g_r,   v_r <- beta2 v_r + (1 - beta2) g_r^2,
 *   V_r <- V_r - lr * (m_r / (1 - beta1^step)) / (sqrt(v_r / (1 - beta2^step)) + eps);
 * rows not selected, and their m and v, are left unchanged.  values, m, v: [C1*C2][d_v]
 * fp32, updated in place (fp32 tables required: PKM_F_FP32 or PKM_F_VALUES_FP32).
 * step >= 1 is the caller's global step count.  0 <= beta < 1, eps > 0.
 * Workspace: pkm_workspace_bytes(d, PKM_BWD). */
pkm_status pkm_value_adam(const pkm_dims* d, float lr, float beta1, float beta2, float eps,
                          int64_t step, float* values, float* m, float* v,
                          const pkm_saved* saved, const float* dy, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Hit monitoring: slot_hits[r] += number of selections of value row r ([C1*C2] int32);
 * subkey_hits[h][i] += number of winners of head h whose first-half sub-key is i, and
 * [h][C1 + j] those whose second-half sub-key is j ([h][C1+C2] int32).  Either may be
 * NULL.  Reads idx [N][h][k] (saved->idx of a forward). */
pkm_status pkm_hit_counts(const pkm_dims* d, const int32_t* idx, int32_t* slot_hits,
                          int32_t* subkey_hits, void* stream);

/* ---- fast-weight memory: chunked read-then-write ----
 * "Fast-weight Product Key Memory", sections 2.2 and 3 (test-time training): the
 * value table is a fast weight.  The N tokens of one sequence are cut into
 * consecutive chunks of `chunk` tokens (the last may be shorter).  Each chunk first
 * READS (F1..F4 with the current table, y of its tokens written), then WRITES: one
 * SGD step of rate `lr` on the value rows the chunk selected, descending
 *     L_c = sum_{t in chunk} 1/2 ||y[t] - target[t]||^2,
 * i.e. V[r] -= lr * sum_{selections (t, h, j) of r} w[t][h][j] * (y[t] - target[t]),
 * duplicates combined before the single write of each row (deterministic).  The
 * next chunk reads what this one wrote; queries, keys and BatchNorm stay fixed.
 *   d        d->N is the sequence length; the value table must be fp32 (PKM_F_FP32,
 *            or PKM_F_VALUES_FP32 beside bf16 x, Wq, subkeys), otherwise
 *            PKM_ERR_UNSUPPORTED.
 *   chunk    >= 1 tokens per chunk.   lr: finite.
 *   mode     0: target[t] = targets[t], targets [N][d_v] fp32 (required);
 *            PKM_FW_LOOKAHEAD: target[t] = x[t + 1], the next token's input, in
 *            x's storage type (needs d_in == d_v; `targets` is ignored and may be
 *            NULL); the last token of
 *            the sequence has no target and adds nothing to the loss.
 *   values   [C1*C2][d_v] fp32, updated IN PLACE.
 *   y        [N][d_v] fp32 out: every chunk's read.
 *   workspace  pkm_fastweight_workspace_bytes(d, chunk, mode) bytes, 256-byte aligned.
 * Everything is enqueued on `stream` with no host synchronisation, so the whole loop
 * can be captured into one CUDA graph. */
/* The write step alone: one sparse SGD step on the value rows `saved` selected,
 *     V[r] -= lr * sum_{selections (t, h, j) of r} w[t][h][j] * dy[t],
 * i.e. rate lr on the value gradient of sum_t dy[t] . y[t], applied only to touched
 * rows, duplicates combined before the single write of each row (deterministic).
 *   values  [C1*C2][d_v] fp32, updated IN PLACE (PKM_F_FP32 or PKM_F_VALUES_FP32
 *           required, otherwise PKM_ERR_UNSUPPORTED).   saved: idx and w are read.   dy: [N][d_v] fp32.
 *   workspace  pkm_workspace_bytes(d, PKM_BWD) bytes. */
pkm_status pkm_value_sgd(const pkm_dims* d, float lr, float* values, const pkm_saved* saved,
                         const float* dy, void* workspace, size_t workspace_bytes, void* stream);

#define PKM_FW_LOOKAHEAD 0x1u
/* Strategy overrides (results are the same; for tests and tuning).  By default every
 * chunk's writes are sorted before the loop -- in shared memory, one CTA per chunk, when a
 * chunk has at most 16384 selections, else by one global radix sort while
 * (number of chunks) * C1*C2 < 2^31 -- and otherwise each chunk selects and sorts on its
 * own.  PKM_FW_SORT_GLOBAL asks for the global sort (per-chunk steps when it does not
 * fit); PKM_FW_PER_CHUNK for the per-chunk steps. */
#define PKM_FW_SORT_GLOBAL 0x2u
#define PKM_FW_PER_CHUNK 0x4u
/* Workspace bytes of pkm_fastweight_chunks for these dims, chunk size and mode bits. */
size_t pkm_fastweight_workspace_bytes(const pkm_dims* d, int64_t chunk, uint32_t mode);
pkm_status pkm_fastweight_chunks(const pkm_dims* d, int64_t chunk, float lr, uint32_t mode,
                                 const void* x, const void* Wq, const float* bn,
                                 const void* subkeys, float* values, const float* targets,
                                 float* y, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ---------------------------------------------------------------- row-sharded table
 * "Meta AI 可扩展内存层", 9.1: the value matrix is split by rows of the product-key
 * index over G ranks, each rank reads only its own rows, and the ranks exchange the
 * candidate indices and partial weighted sums; 4.5: row i*|C'| + j, so a range of
 * leading sub-key indices is a contiguous range of rows.  Shard g holds rows
 * [g*R, min((g+1)*R, C1*C2)) (R = ceil(C1/G)*C2 splits by leading sub-key; any
 * R >= 1 with G*R >= C1*C2 is accepted), as its own [rows][d_v] table.
 *
 * The rank that owns a batch of N tokens (its source) runs pkm_query,
 * pkm_subkey_scores and pkm_candidate_topk, then pkm_shard_route; the caller's
 * collective moves, per destination g, counts[g], then the triples, to the owner of
 * shard g.  The owner runs pkm_shard_bag over what it received (triples of every
 * source, concatenated in source order) and returns partial row j of each source's
 * segments to it; the source sums them with pkm_shard_combine.  Backward: the source
 * sends dy once per segment (pkm_shard_gather_dy), the owner runs
 * pkm_shard_value_grad (its dV += and dL/dw of every received triple), the source
 * puts the returned dL/dw in place with pkm_shard_scatter_dw and continues with
 * pkm_query_grad.  The library moves no data between ranks. */
#define PKM_MAX_SHARDS 1024
typedef struct {
  int32_t seg;  /* the triple's segment: its token's run for this destination, from 0 */
  int32_t row;  /* row within the destination's shard */
  float w;      /* softmax weight */
} pkm_triple;
/* which: PKM_SHARD_ROUTE (source side; n_triples ignored) or PKM_SHARD_OWNER (owner side,
 * for up to n_triples received triples; includes the value pass's scratch). */
#define PKM_SHARD_ROUTE 1
#define PKM_SHARD_OWNER 2
size_t pkm_shard_workspace_bytes(const pkm_dims* d, int32_t G, int which, int64_t n_triples);
/* Source side.  idx, w: [N][h][k] (as pkm_forward's saved idx and w: flat rows).
 * counts: device [G][2] int32 = {triples, segments} bound for shard g.  segpos: device
 * [G][N] int32, the row of the combined receive buffer (all partial rows sent back,
 * shard 0's first) that holds token t's partial from shard g, or -1 when t sent g
 * nothing.  send: [N*h*k] triples grouped by destination (shard 0's first), within it
 * by token, within a token in selection order.  perm: [N*h*k], perm[pos] = the flat
 * selection index t*h*k + s of send[pos].  A row outside the table records
 * PKM_ERR_DEVICE_INDEX and is routed as row 0.  1 <= G <= PKM_MAX_SHARDS,
 * G*N < 2^31. */
pkm_status pkm_shard_route(const pkm_dims* d, int32_t G, int64_t rows_per_shard,
                           const int32_t* idx, const float* w, int32_t* counts, int32_t* segpos,
                           pkm_triple* send, int32_t* perm, void* workspace,
                           size_t workspace_bytes, void* stream);
/* Owner side.  recv_counts: device [G][2] int32, the counts each source sent this shard;
 * n_triples, n_segments: their sums (host).  recv: the received triples, source 0's
 * first.  values: this shard's [shard_rows][d_v] table (bf16, or fp32 with
 * PKM_F_FP32 / PKM_F_VALUES_FP32).  partial: [n_segments][d_v] fp32, row j = sum over
 * segment j's triples of w * V[row] (segments numbered across sources in source order).
 * Out-of-range segments or rows record PKM_ERR_DEVICE_INDEX and are clamped. */
pkm_status pkm_shard_bag(const pkm_dims* d, int32_t G, int64_t shard_rows,
                         const int32_t* recv_counts, int64_t n_triples, int64_t n_segments,
                         const pkm_triple* recv, const void* values, float* partial,
                         void* workspace, size_t workspace_bytes, void* stream);
/* Source side.  partial_recv: [n_rows][d_v] fp32, the partial rows every shard sent back
 * (shard 0's first); y[t] (overwritten) = their sum over shards in ascending order. */
pkm_status pkm_shard_combine(const pkm_dims* d, int32_t G, const int32_t* segpos,
                             const float* partial_recv, int64_t n_rows, float* y, void* stream);
/* Source side.  dy_send[segpos[g][t]] = dy[t] for every segment (n_rows rows). */
pkm_status pkm_shard_gather_dy(const pkm_dims* d, int32_t G, const int32_t* segpos,
                               const float* dy, float* dy_send, int64_t n_rows, void* stream);
/* Owner side, backward.  dy_recv: [n_segments][d_v] fp32 in the received segment order.
 * dvalues: this shard's dense fp32 [shard_rows][d_v] gradient (+=, one writer per row,
 * deterministic).  dw_recv: [n_triples] fp32 (overwritten), dL/dw of every received
 * triple = dy of its segment . V[row]. */
pkm_status pkm_shard_value_grad(const pkm_dims* d, int32_t G, int64_t shard_rows,
                                const int32_t* recv_counts, int64_t n_triples,
                                int64_t n_segments, const pkm_triple* recv, const void* values,
                                const float* dy_recv, float* dvalues, float* dw_recv,
                                void* workspace, size_t workspace_bytes, void* stream);
/* Source side.  dw[perm[i]] = dw_ret[i] for the N*h*k triples this rank sent (dw_ret in
 * the send order). */
pkm_status pkm_shard_scatter_dw(const pkm_dims* d, const int32_t* perm, const float* dw_ret,
                                float* dw, void* stream);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns PKM_OK, PKM_ERR_DEVICE_TIMEOUT, PKM_ERR_DEVICE_INDEX or
 * PKM_ERR_CUDA (when the synchronisation itself failed). */
pkm_status pkm_check_status(void* stream);

/* Static, human-readable name of a status code. */
const char* pkm_status_string(pkm_status s);

/* Value-gradient stage (as pkm_value_grad) for callers that cannot allocate device
 * memory, so cannot pass a workspace.  One example is a plugin inside a host framework
 * that owns all device memory through its own allocator and gives the plugin no way to
 * reserve more.  Another is a latency-bound loop that must not call cudaMalloc, which
 * can synchronise the whole device.  This entry point allocates nothing: its scratch
 * is a fixed 64 MiB device array built into the library, which every GPU that loads
 * the library holds until the process exits.
 * The pages have no counterpart to this entry point.
 *   - Limit: the scratch holds the value stage's sort and segment buffers, about 53
 *     bytes per selection (N*h*k selections; e.g. up to N = 8192 tokens at h = 4,
 *     k = 32).  A larger problem returns PKM_ERR_WORKSPACE from a host-side check,
 *     before any CUDA call.
 *   - The first call on a device fetches the array's device address
 *     (cudaGetSymbolAddress) with that device current.  A failed lookup returns
 *     PKM_ERR_CUDA and is not cached: the next call retries.
 *   - Every call shares the one array.  Each call clears or fully rewrites the parts
 *     it reads, so nothing needs clearing between calls.  Calls whose work overlaps on
 *     the GPU (other streams, other host threads) race on the array and must be
 *     serialised by the caller.
 *   - Same arguments and results as pkm_value_grad otherwise. */
pkm_status pkm_value_grad_noalloc(const pkm_dims* d, const void* values, const pkm_saved* saved,
                                  const float* dy, float* dvalues, float* dw, void* stream);

/* Self-test of the device-side bounded wait: launches one warp that waits on a
 * barrier nothing arrives on, with a budget of `budget_cycles` SM clocks (1 to 1e8).
 * The wait gives up and records PKM_ERR_DEVICE_TIMEOUT in the status word, which the
 * next pkm_check_status returns (and clears).  Faults, traps and hangs nothing. */
pkm_status pkm_selftest_wait_timeout(uint32_t budget_cycles, void* stream);

/* Number of kernels this library has launched in this process (diagnostics). */
unsigned long long pkm_launch_count(void);

/* Build identification string (static). */
const char* pkm_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* PKM_H_ */
