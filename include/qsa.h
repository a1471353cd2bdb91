/*
 * qsa.h -- C ABI of the B200 (sm_100a) exact route-set Query Sparse Attention
 * library (libqsa_b200.so).
 *
 * What it computes.  Each query token t attends to the set R_t of K/V rows named
 * by its route IDs (cuDNN-Frontend "Query Sparse Attention (QSA)" page, sections
 * "Tensors" and "Selection and components"; "flex_qsa" page, module description
 * and `_routes_to_membership`; "fa4_qsa" page, `fa4_sparse_gqa_attention`):
 *   - a route ID r is valid iff 0 <= r < T_kv; every other value (-1, negative,
 *     >= T_kv) is padding;
 *   - duplicate IDs select a key once (route membership is a set);
 *   - no causal or other mask is added: the routes alone decide visibility;
 *   - grouped-query attention, 12 query heads per KV head: query head h reads KV
 *     head h / 12 (contiguous head groups, "cudnn_qsa" page, `_CudnnQSA`);
 *   - head dimension 256, BF16 inputs and outputs, FP32 accumulation.
 * Forward:  S = scale * Q_h K_g^T over R_t, P = softmax(S), out = P V_g,
 *           lse = natural-log softmax normaliser.  A row with empty R_t gives
 *           out = 0 and lse = -inf.
 * Backward: the equations of the "Selection and components" section:
 *           P = exp(S - lse), delta = rowsum(dO * out), dP = dO V^T,
 *           dS = P * (dP - delta), dQ = scale dS K, dK = scale dS^T Q,
 *           dV = P^T dO, dK/dV summed over the 12 query heads of each group.
 *           Empty rows give dQ = 0 and contribute nothing to dK/dV.  dK/dV are
 *           bitwise reproducible run to run (no floating-point atomics).
 *
 * Conventions for every entry point.
 *   - BF16 tensors are passed as `const void*` / `void*` holding IEEE bfloat16
 *     bit patterns.  All tensors are dense, contiguous, row-major, on the device
 *     that is current when the call is made.
 *       q, out, grad_out, dq : [T, H, 256] BF16        (H = 12 * G)
 *       k, v, dk, dv         : [T_kv, G, 256] BF16
 *       routes               : [T, n_sel] int32
 *       lse                  : [T, H] float32 (natural log)
 *   - BF16 tensors must be 16-byte aligned, int32/float32 tensors 4-byte aligned,
 *     the workspace 256-byte aligned.
 *   - The caller owns every buffer, including the workspace (size from the
 *     matching *_workspace_size function).  The library allocates no device
 *     memory and keeps no state between calls.  The workspace contents are
 *     scratch: nothing needs to be initialised, nothing survives the call,
 *     except the first int32 of the workspace, a status word: once the call's
 *     work has completed on the stream it is 0, or nonzero if a kernel gave up
 *     on a bounded wait (its outputs are then invalid), and, after a forward
 *     call, the route lists that qsa_backward_saved can reuse, with their tag
 *     in int32 words 4..7.  Every wait inside the
 *     kernels is bounded, so a fault in the pipeline ends the kernel instead of
 *     hanging the GPU.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.  Route values are never
 *     read on the host.
 *   - Errors: arguments are checked on the host before anything is launched;
 *     a failed check returns its status and launches nothing.  A failed kernel
 *     launch returns QSA_ERR_CUDA.  Route values are never errors (invalid IDs
 *     are padding).
 *   - Limits: T, T_kv, n_sel >= 1; n_sel <= 16384; T * n_sel <= 2^31 - 1;
 *     T <= 2^30; T_kv <= 2^31 - 1; H = 12 * G, G >= 1; 0 < scale < inf.
 */
#ifndef QSA_B200_H
#define QSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qsa_stream_t; /* same type as cudaStream_t */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, size out of range, bad scale */
  QSA_ERR_UNSUPPORTED = 2,        /* head geometry other than 12 query heads per KV head */
  QSA_ERR_MISALIGNED = 3,         /* a pointer violates the alignment rules above */
  QSA_ERR_WORKSPACE_TOO_SMALL = 4,
  QSA_ERR_CUDA = 5                /* a CUDA runtime call or kernel launch failed */
} qsa_status_t;

/* Human-readable name of a status; never NULL, static storage. */
const char* qsa_status_string(qsa_status_t status);

/* Library version string, static storage. */
const char* qsa_version(void);

/*
 * Workspace bytes needed by qsa_forward / qsa_backward for these sizes.  Returns
 * 0 when the sizes are outside the limits above (the matching call would return
 * QSA_ERR_INVALID_ARGUMENT or QSA_ERR_UNSUPPORTED).
 */
size_t qsa_forward_workspace_size(int64_t T, int64_t T_kv, int H, int G, int n_sel);
size_t qsa_backward_workspace_size(int64_t T, int64_t T_kv, int H, int G, int n_sel);

/*
 * Forward pass.  Cites: "Query Sparse Attention (QSA)" page, "Selection and
 * components" (forward: scaled QK, softmax, PV; FP32 output cast to BF16;
 * natural-log LSE; empty rows zero output and -inf LSE).
 *   in : q, k, v, routes, sizes, scale (finite, > 0; normally 1/16)
 *   out: out [T, H, 256] BF16, lse [T, H] float32
 */
qsa_status_t qsa_forward(const void* q, const void* k, const void* v, const int32_t* routes,
                         int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                         void* out, float* lse,
                         void* workspace, size_t workspace_bytes, qsa_stream_t stream);

/*
 * Backward pass.  Cites: "Query Sparse Attention (QSA)" page, "Selection and
 * components" (the backward equations; delta from the forward output; FP32
 * accumulation, BF16 gradients; dK/dV summed over query heads).
 *   in : grad_out, q, k, v, out and lse from qsa_forward with the same q, k, v,
 *        routes and scale; routes, sizes, scale
 *   out: dq [T, H, 256], dk and dv [T_kv, G, 256] (BF16).  Every row of dk/dv is
 *        written; keys no query routes to get exact zeros.
 */
qsa_status_t qsa_backward(const void* grad_out, const void* q, const void* k, const void* v,
                          const void* out, const float* lse, const int32_t* routes,
                          int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                          void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, qsa_stream_t stream);

/*
 * Backward with FP32 dK / dV, for callers that add dK / dV contributions of
 * several calls before the one rounding to BF16 (context parallelism: each
 * rank's queries contribute to the global keys, and the partials are summed by
 * a reduce-scatter).  Cites: "Query Sparse Attention (QSA)" page, "Selection
 * and components" (FP32 accumulation; dK/dV summed over query heads).
 * Same arguments and checks as qsa_backward, except that dk and dv are FP32
 * [T_kv, G, 256] (16-byte aligned): the FP32 values that qsa_backward rounds to
 * BF16 (keys no query routes to get exact zeros).
 */
qsa_status_t qsa_backward_fp32kv(const void* grad_out, const void* q, const void* k, const void* v,
                                 const void* out, const float* lse, const int32_t* routes,
                                 int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                 void* dq, float* dk, float* dv,
                                 void* workspace, size_t workspace_bytes, qsa_stream_t stream);

/*
 * Same as qsa_forward / qsa_backward, and in addition records caller-created
 * CUDA events (cudaEvent_t, passed as qsa_event_t) on `stream` after each stage,
 * for per-kernel timing.  Stage i's event is recorded right after stage i is
 * enqueued; only the first min(n_stage_events, stage count) are recorded.
 * `stage_events` may be NULL when n_stage_events is 0.  The pages have no
 * counterpart: this is an instrumentation hook of this library.
 *   forward stages : 0 route rows (sort/dedup), 1 attention forward
 *   backward stages: 0 route rows (+ delta, tile masks), 1 tile lists (column
 *                    scans, tile-pointer scan, fill), 2 work lists, 3 dQ (+ P/dS
 *                    records), 4 dK/dV
 * A failed eventRecord returns QSA_ERR_CUDA.
 */
typedef struct CUevent_st* qsa_event_t; /* same type as cudaEvent_t */
#define QSA_FORWARD_STAGES 2
#define QSA_BACKWARD_STAGES 5

qsa_status_t qsa_forward_ex(const void* q, const void* k, const void* v, const int32_t* routes,
                            int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                            void* out, float* lse,
                            void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                            const qsa_event_t* stage_events, int n_stage_events);
qsa_status_t qsa_backward_ex(const void* grad_out, const void* q, const void* k, const void* v,
                             const void* out, const float* lse, const int32_t* routes,
                             int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                             void* dq, void* dk, void* dv,
                             void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                             const qsa_event_t* stage_events, int n_stage_events);

/*
 * Same as qsa_forward_ex / qsa_backward_ex (dk / dv FP32 as in
 * qsa_backward_fp32kv when kv_fp32 is nonzero), with K/V that may still be in
 * flight: `kv_ready` (a cudaEvent_t, or NULL for none) is an event the caller
 * records once k and v hold their values, for instance on the stream of a K/V
 * all-gather.  The call enqueues its route work (which reads neither) first,
 * then makes `stream` wait for kv_ready before the first kernel that reads k or
 * v (the forward attention; the backward's dQ), so that the gather runs under
 * the route kernels.  The wait is a cudaStreamWaitEvent on `stream`: the host
 * never blocks.  Stage events as in the _ex calls; the wait follows stage 0 of
 * the forward and stage 2 of the backward.  The context-parallel layout of the
 * "flex_qsa" and "fa4_qsa" pages (local queries against gathered global K/V)
 * is what it serves; the pages have no such call.  A failed wait returns
 * QSA_ERR_CUDA.
 */
qsa_status_t qsa_forward_kvwait(const void* q, const void* k, const void* v, const int32_t* routes,
                                int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                void* out, float* lse,
                                void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                                qsa_event_t kv_ready, const qsa_event_t* stage_events, int n_stage_events);
qsa_status_t qsa_backward_kvwait(const void* grad_out, const void* q, const void* k, const void* v,
                                 const void* out, const float* lse, const int32_t* routes,
                                 int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                 void* dq, void* dk, void* dv, int kv_fp32,
                                 void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                                 qsa_event_t kv_ready, const qsa_event_t* stage_events, int n_stage_events);

/*
 * Backward that reuses the forward's route lists instead of sorting the routes
 * again.  Every forward call (qsa_forward, _ex, _kvwait, with a workspace of at
 * least qsa_forward_workspace_size bytes) leaves the per-row ascending,
 * de-duplicated route lists it computed in its workspace, after the status
 * word; `fwd_workspace` / `fwd_workspace_bytes` name that workspace, which must
 * still hold them: the forward ran with the same routes and sizes, and nothing
 * has written the workspace since (the backward's own `workspace` may be the
 * same buffer, if it is large enough for the backward).  The backward then
 * runs only delta and the tile masks as its route work.  Results are bit for
 * bit those of qsa_backward_kvwait on the same routes; other arguments, checks
 * and stage events as there (routes are not an argument).  The forward also
 * leaves a tag of the sizes it sorted for (int32 words 4..7 of its workspace);
 * when fwd_workspace lacks the tag of rows of these sizes (no forward wrote it,
 * or one of other sizes), the status word of `workspace` reads 2 after the
 * call, no kernel reads the lists, and dq, dk and dv are invalid.  Lists of
 * other routes with the same sizes cannot be told apart on the device: they
 * give wrong gradients.  The pages have no counterpart (training keeps a
 * forward's index structures for its backward as it keeps the LSE).
 */
qsa_status_t qsa_backward_saved(const void* grad_out, const void* q, const void* k, const void* v,
                                const void* out, const float* lse,
                                const void* fwd_workspace, size_t fwd_workspace_bytes,
                                int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                void* dq, void* dk, void* dv, int kv_fp32,
                                void* workspace, size_t workspace_bytes, qsa_stream_t stream,
                                qsa_event_t kv_ready, const qsa_event_t* stage_events, int n_stage_events);

/*
 * Number of kernels one qsa_forward (backward = 0) or qsa_backward (backward = 1)
 * call enqueues for these sizes, not counting the backward's one cudaMemsetAsync
 * node (its counters and tile masks).  The forward launches 2 (route rows,
 * attention); the backward 7 (route rows with the tile masks, column scans of
 * the masks, tile-pointer scan, tile fill, work lists, dQ, dK/dV).  Returns 0
 * for sizes the calls reject.  For instrumentation and for sizing CUDA graphs;
 * the pages have no counterpart.
 */
int qsa_launch_count(int64_t T, int64_t T_kv, int H, int G, int n_sel, int backward);

/*
 * Route preprocessing on its own.  Cites: "fa4_qsa" page, `_preprocess`
 * (duplicates collapse, invalid IDs discarded; forward and reverse lists).
 * row_cnt / row_cols are the per-row lists the forward and dQ kernels consume;
 * the reverse lists here are grouped by key quad with owner masks (the dK/dV
 * pass uses the 128-key tile grouping of qsa_tile_plan instead).
 *   row_cnt  [T] int32       : |R_t|
 *   row_cols [T, n_sel] int32: R_t ascending in the first row_cnt[t] slots; the
 *                              remaining slots are left unspecified
 *   quad_ptr [ceil(T_kv/4)+1] int32 : CSR offsets of the key-quad lists
 *   quad_ent [T * n_sel] int64 : for quad b (keys 4b..4b+3), entries
 *       quad_ent[quad_ptr[b] .. quad_ptr[b+1]) in ascending query order, each
 *       (t << 32) | (i0 << 4) | mask, where t is a query whose R_t meets the
 *       quad, mask bit j is set iff key 4b+j is in R_t, and i0 is the position in
 *       row_cols[t, :] of the quad's first key in R_t.  Slots past quad_ptr[last]
 *       are left unspecified.
 *   scratch: qsa_route_plan_scratch_size(T, T_kv) bytes, 256-byte aligned.
 */
size_t qsa_route_plan_scratch_size(int64_t T, int64_t T_kv);
qsa_status_t qsa_route_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel,
                            int32_t* row_cnt, int32_t* row_cols, int32_t* quad_ptr,
                            int64_t* quad_ent, void* scratch, size_t scratch_bytes,
                            qsa_stream_t stream);

/*
 * The key->query transpose the backward's dK/dV pass walks, on its own: the
 * reverse lists of the "fa4_qsa" page's `_preprocess` grouped by aligned tiles
 * of 128 keys instead of single keys.
 *   row_cnt, row_cols : as qsa_route_plan
 *   tile_ptr [ceil(T_kv/128)+1] int32 : CSR offsets of the tile lists
 *   tile_ent [T * n_sel] int64 : for tile b (keys 128b..128b+127), entries
 *       tile_ent[tile_ptr[b] .. tile_ptr[b+1]) in ascending query order, each
 *       (t << 32) | (i0 << 8) | (n - 1), where t is a query whose R_t meets the
 *       tile, n (1..128) is the number of keys of R_t in the tile and
 *       row_cols[t, i0 .. i0 + n) are those keys.  Slots past tile_ptr[last]
 *       are left unspecified.
 *   scratch: qsa_tile_plan_scratch_size(T, T_kv) bytes, 256-byte aligned.
 * Same size limits and errors as qsa_route_plan.
 */
size_t qsa_tile_plan_scratch_size(int64_t T, int64_t T_kv);
qsa_status_t qsa_tile_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                           int32_t* row_cols, int32_t* tile_ptr, int64_t* tile_ent, void* scratch,
                           size_t scratch_bytes, qsa_stream_t stream);

/*
 * Block-selection bitmap -> route IDs, so that callers of the bitmap API can use
 * the route-set calls above.  Cites: "Query Sparse Attention (QSA)" page,
 * "Tensors" (sel_blocks, lo, hi, blk_base, tok_base) and "Selection and
 * components" (the block lookup): key token j is allowed for query t iff
 * lo[t] <= j <= hi[t], 0 <= b < NB and sel_blocks[t, b] != 0, where
 * b = blk_base[t] + floor((j - tok_base[t]) / block_size).  The allowed set is a
 * route set: qsa_forward / qsa_backward on the returned routes compute the
 * bitmap API's attention.
 *   in : sel_blocks [T, NB] uint8 (row-major; nonzero selects global block b);
 *        lo, hi, blk_base, tok_base [T] int32; T_kv key tokens (keys outside
 *        [0, T_kv) are never allowed); block_size >= 1; n_sel route width.
 *        block_first / block_last are not taken: the lookup does not read them
 *        (their agreement with the bases is a caller contract the page leaves
 *        unchecked).
 *   out: routes [T, n_sel] int32, each row the allowed keys ascending, then -1;
 *        a row with more than n_sel allowed keys keeps its n_sel smallest.
 *        row_cnt [T] int32 (may be NULL): the true size of each allowed set.
 *        max_cnt (may be NULL; one int32): set to the largest row_cnt, so a
 *        caller can size n_sel (the call zeroes it first, on the stream).
 *   Errors: NULL sel_blocks / lo / hi / blk_base / tok_base / routes, T, NB,
 *   T_kv, n_sel or block_size < 1, T_kv > INT32_MAX or T * n_sel > 2^31 - 1:
 *   QSA_ERR_INVALID_ARGUMENT; sel_blocks not 16-byte aligned (it is read with
 *   16-byte loads) or int32 pointers not 4-byte aligned: QSA_ERR_MISALIGNED;
 *   a failed launch: QSA_ERR_CUDA.  Asynchronous on
 *   `stream`; reads no device value on the host.
 */
qsa_status_t qsa_bitmap_routes(const uint8_t* sel_blocks, const int32_t* lo, const int32_t* hi,
                               const int32_t* blk_base, const int32_t* tok_base,
                               int64_t T, int64_t NB, int64_t T_kv, int block_size, int n_sel,
                               int32_t* routes, int32_t* row_cnt, int32_t* max_cnt,
                               qsa_stream_t stream);

/*
 * QSA block selector, in two calls.  Cites: "Query Sparse Attention (QSA)" page,
 * "Finding QSA attention and its indexer" (each complete compressed block is
 * scored as scale * sum_h relu(qi[t, h] . kbar[block]); ratio-causal top-k;
 * local block IDs expanded with the incomplete causal tail and the packed
 * sequence's token origin) and the "cudnn_qsa" page, _pack_indices (four-slot
 * route groups: one complete block or the tail, -1 padded).
 *
 * Query t sits at key position pos[t] of a sequence whose first token is
 * tok_base[t] and whose first compressed block is blk_base[t] (pos, blk_base,
 * tok_base [T] int32; NULL means pos[t] = t and zero bases).  Its own block is
 * o = (pos - tok_base) / 4; its candidates are the local blocks c in
 * [0, min(o, NB - blk_base)), local block c being global block blk_base + c of
 * kbar and covering tokens tok_base + 4c .. + 3.
 *
 * qsa_selector_scores: qi [T, Hi, Di] BF16, kbar [NB, Di] BF16 (both 16-byte
 * aligned, contiguous), Di == 128, Hi in {32, 64, 128, 256}, scale > 0 finite.
 * Writes scores[t * score_stride + c] (FP32) for every candidate c and leaves
 * the other entries untouched; score_stride >= NB.  Runs on the tensor cores
 * (tcgen05, operands staged by TMA).  `status` (nullable device int) is set to
 * 2 if an internal bounded wait gave up (then some scores are missing).
 * qsa_selector_topk: from those scores, blocks [T, k] int32 = the k best
 * candidates (larger score first, equal scores by the lower local ID), written
 * ascending and -1 padded (all candidates when there are fewer than k);
 * routes [T, 4 (k + 1)] int32 = their tokens as four-slot groups, then the
 * causal tail (tokens tok_base + 4o .. pos, -1 padded), then -1.
 * Errors: NULL required pointers, T, NB or k < 1, score_stride < NB, sizes
 * whose products exceed 2^31 - 1: QSA_ERR_INVALID_ARGUMENT; other Di or Hi:
 * QSA_ERR_UNSUPPORTED; misaligned pointers: QSA_ERR_MISALIGNED; a failed
 * launch (or no tensor-map encoder in the driver): QSA_ERR_CUDA.
 */
qsa_status_t qsa_selector_scores(const void* qi, const void* kbar, int64_t T, int64_t NB, int Hi, int Di,
                                 float scale, const int32_t* pos, const int32_t* blk_base,
                                 const int32_t* tok_base, float* scores, int64_t score_stride,
                                 int* status, qsa_stream_t stream);
qsa_status_t qsa_selector_topk(const float* scores, int64_t score_stride, int64_t T, int64_t NB, int k,
                               const int32_t* pos, const int32_t* blk_base, const int32_t* tok_base,
                               int32_t* blocks, int32_t* routes, qsa_stream_t stream);

/*
 * The query-union lists the forward walks, on their own: the paired-query
 * gather of the "Query Sparse Attention (QSA)" page ("Selection and
 * components": adjacent queries gather the union of their selected keys once,
 * owner bits keeping each query's own set), for groups of
 * qsa_union_group(n_sel) adjacent rows (4, or 1 for rows of more than 4096
 * slots; 0 for an n_sel outside 1..16384).
 *   row_cnt, row_cols : as qsa_route_plan
 *   ucnt [ceil(T/group)] int32 : the number of distinct keys in each group's union
 *   ukey [ceil(T/group) * group * n_sel] int32 : group i's union, ascending, in
 *       ukey[i * group * n_sel .. + ucnt[i]); the rest is left unspecified
 *   uown (same shape) uint8 : per union key, bit q set iff row group * i + q selected it
 * Same size limits and errors as qsa_route_plan (ucnt / ukey 4-byte aligned).
 */
int qsa_union_group(int n_sel);
qsa_status_t qsa_union_plan(const int32_t* routes, int64_t T, int64_t T_kv, int n_sel, int32_t* row_cnt,
                            int32_t* row_cols, int32_t* ucnt, int32_t* ukey, uint8_t* uown, qsa_stream_t stream);

/*
 * FP32 -> BF16 rounding of n contiguous values, round to nearest with ties to
 * even: the final cast of dK / dV sums that a caller adds up in FP32 across
 * several qsa_backward_fp32kv calls (context parallelism reduce-scatters each
 * rank's FP32 partials, then rounds its own slice once), with the rounding the
 * backward applies itself ("Selection and components": FP32 accumulation,
 * BF16 gradients).
 *   x [n] float32, y [n] bf16 (device, caller-owned, 16-byte aligned; they
 *   must not overlap).  Enqueued on `stream`.
 * Errors: n < 0 or a NULL pointer with n > 0: QSA_ERR_INVALID_ARGUMENT;
 * misaligned pointers: QSA_ERR_MISALIGNED; a failed launch: QSA_ERR_CUDA.
 */
qsa_status_t qsa_cast_f32_to_bf16(const float* x, void* y, int64_t n, qsa_stream_t stream);

/*
 * Allocation-free forward, for callers that cannot allocate device memory: for
 * example an extension running inside a host application that owns the device
 * allocator and offers it no allocation hook, or a latency-critical path that
 * must not call cudaMalloc (which can synchronise the device and has no bounded
 * latency).  The pages have no counterpart: this is an interface convenience of
 * this library.
 *
 * Same arguments and results as qsa_forward, minus the workspace.  The scratch
 * the forward needs (the per-row sorted route lists) lives in a fixed array of
 * QSA_NOALLOC_SCRATCH_BYTES (16 MiB) compiled into the library; every GPU on
 * which the library runs this call holds that array until the process exits.
 *   - Limit: qsa_forward_workspace_size(T, T_kv, H, G, n_sel) must not exceed
 *     QSA_NOALLOC_SCRATCH_BYTES, roughly T * (n_sel + 1) * 4 bytes <= 16 MiB
 *     (T = 4096 with n_sel = 256 fits; T = 16384 with n_sel = 512 does not).
 *     Larger sizes return QSA_ERR_WORKSPACE_TOO_SMALL and launch nothing; call
 *     qsa_forward with a workspace instead.  Other argument errors return the
 *     same statuses as qsa_forward, checked in the same order (a call that is
 *     both misaligned and too large returns QSA_ERR_MISALIGNED).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  Later calls on the device reuse the address
 *     while the CUDA context it was taken in is current; after cudaDeviceReset
 *     the next call looks it up again in the new context (so, again, make that
 *     call before any capture).
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *   - All calls on one device share the array, and it keeps the last call's
 *     contents; nothing in it has to start at zero, because each call overwrites
 *     everything it later reads.  Calls whose GPU work overlaps (unordered
 *     streams, several host threads) race on the array and produce wrong
 *     results: order them on one stream or with events.
 */
#define QSA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
qsa_status_t qsa_forward_noalloc(const void* q, const void* k, const void* v, const int32_t* routes,
                                 int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                 void* out, float* lse, qsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_B200_H */
