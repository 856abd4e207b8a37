/*
 * ssa.h -- C ABI of libssa, the B200 (sm_100a) hot path of SSA, Sparse Sparse
 * Attention: causal block-sparse attention with per-query-block top-k block
 * selection, computed in one pass together with the full causal attention,
 * the dropped attention mass delta(t), and the backward of both streams with
 * the bidirectional alignment loss folded in.
 *
 * Sources (page title, then section):
 *   [digest]  "SSA: Achieving Sparser Attention by Aligning Full and Sparse
 *             Attention Outputs in Feature Space" (blog digest of the paper).
 *   [summary] "Technische Samenvatting: SSA (Sparse Sparse Attention)".
 *   [record]  "SSA: Sparse Sparse Attention by Aligning Full and Sparse
 *             Attention Outputs in Feature Space" (arXiv 2511.20102 record).
 *
 * Notation: B batch, Hq query heads, Hkv key/value heads (g = Hq/Hkv query
 * heads share one kv head; query head h reads kv head h/g), N tokens, d head
 * dim, s = block, n = N/s blocks, k = topk budget in blocks counting the
 * diagonal block, scale = attention scale (1/sqrt(d) in the paper's models;
 * any finite positive value is accepted).
 * Query token t lies in block i = t/s.  Sel(i) is the selected block set of
 * query block i; A_t = {u <= t : u/s in Sel(i)} is attended by both streams,
 * D_t = {u <= t : u/s not in Sel(i)} only by the full stream.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  Every pointer is a DEVICE pointer the caller allocated on the
 *   current CUDA device; the caller keeps ownership.  libssa never allocates,
 *   frees or synchronises (except ssa_device_status).  All work is enqueued
 *   on `stream` (a cudaStream_t; NULL means the legacy default stream) in
 *   stream order; calls are stateless and may be issued from several host
 *   threads on different streams.
 * Tensors.  ssa_tensor_t describes a 4-D tensor [B, H, N, d] of dims->dtype
 *   elements whose last (d) dimension is contiguous; stride_b / stride_h /
 *   stride_n are in ELEMENTS.  Q, h_full, h_sparse, dQ, g_full, g_sparse use
 *   H = Hq; K, V, dK, dV use H = Hkv.  Base pointers must be 16-byte aligned
 *   and every stride times the element size a multiple of 16 bytes.
 *   Plain arrays (scores, idx, lse_*, delta) are dense row-major as stated.
 * Shapes.  B, Hq, N >= 0 and Hkv >= 1 with Hq % Hkv == 0; block in
 *   {16, 32, 64, 128}; N a multiple of block and of 64; d in {64, 128};
 *   topk >= 1 (a budget above n is clamped: k_eff = min(topk, n));
 *   n <= 2048.  When B*Hq*N == 0 the call is a no-op and returns SSA_OK.
 *   bf16 runs on tensor cores: blocks of 64 and 128 with d = 128 and
 *   per-block selection on the tcgen05 kernels; the other bf16 shapes (d =
 *   64, the small blocks 16 and 32 of the paper's models, [digest] "Model
 *   Architecture Configuration", and per-token selection) on tcgen05
 *   kernels with per-row selection masks (dual forward, dropped mass,
 *   backward; at d = 128 the backward masks single elements) and on
 *   warp-level mma.sync kernels for the sparse stream alone (block walks fed
 *   by TMA at blocks of 16 and 32, per-token selection); the decode step's
 *   attention products on mma.sync; fp32 on the CUDA-core kernels.
 * Errors.  Arguments are checked on the host before anything is enqueued;
 *   a failed check returns SSA_ERR_INVALID_ARG (bad pointer, stride,
 *   alignment or value), SSA_ERR_UNSUPPORTED (a shape outside the list above,
 *   or a device that is not sm_100) or SSA_ERR_WORKSPACE (ws_bytes below
 *   ssa_workspace_bytes) and enqueues nothing.  A failed launch returns
 *   SSA_ERR_CUDA.  Kernels that wait on hardware barriers bound every wait;
 *   a wait that runs out records SSA_ERR_TIMEOUT in a per-device status
 *   report (read and clear it with ssa_device_status) and the kernel returns;
 *   the outputs of that call are then undefined.  The report changes nothing
 *   for later calls: every call does its full work whatever the report
 *   holds, so a timed-out call on one stream leaves calls on other streams
 *   correct.  No kernel traps.
 * Precision.  dtype SSA_BF16: inputs/outputs bf16, products on tensor cores
 *   with fp32 accumulation and fp32 softmax statistics.  SSA_F32: fp32 inputs
 *   and outputs, fp32 arithmetic throughout (CUDA cores).
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSA_API __attribute__((visibility("default")))
#else
#define SSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1,
  SSA_ERR_UNSUPPORTED = 2,
  SSA_ERR_CUDA = 3,
  SSA_ERR_TIMEOUT = 4,
  SSA_ERR_WORKSPACE = 5
} ssa_status_t;

typedef enum { SSA_F32 = 0, SSA_BF16 = 1 } ssa_dtype_t;

typedef struct {
  int32_t B, Hq, Hkv, N, d, block, topk;
  float scale;
  int32_t dtype;     /* ssa_dtype_t */
  int32_t per_token; /* 0: one selection per query block (idx rows = n);
                        1: one selection per query token (idx rows = N),
                        see ssa_select_tokens */
} ssa_dims_t;

typedef struct {
  void* ptr;
  int64_t stride_b, stride_h, stride_n; /* elements; the d stride is 1 */
} ssa_tensor_t;

typedef void* ssa_stream_t; /* cudaStream_t */

/* ABI version of this header (major * 100 + minor). */
SSA_API int ssa_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
SSA_API const char* ssa_status_string(ssa_status_t status);

/* Bytes of device workspace that ssa_block_scores, ssa_bwd_dual,
 * ssa_bwd_sparse, ssa_decode_step, ssa_dropped_mass and ssa_align_mse need for these dims (one size serves
 * all of them).  Returns 0 for an invalid or empty shape.  The workspace is
 * caller-owned scratch: its contents on entry are ignored and on return
 * undefined; two calls in flight at once must not share one workspace. */
SSA_API size_t ssa_workspace_bytes(const ssa_dims_t* dims);

/* Step 1: block pooling and block scores.
 * [digest] "Practical Implementation of SSA": split the sequence into blocks,
 * represent each block by the mean of its keys, and score the query against
 * every earlier block representation; pooling keeps the ranking because the
 * mean of q K^T over a block equals q times the mean of the block's keys.
 * The query side is the mean of the query block (selection is per query
 * block and per query head).
 *   scores [B, Hq, n, n] fp32 (out): scores[b,h,i,j] = scale * qbar_i . kbar_j
 *     for j < i, with qbar / kbar the fp32 means of query block i (head h) and
 *     key block j (kv head h/g); -INFINITY for j >= i (the diagonal is kept
 *     unconditionally by ssa_select_topk and is not scored).
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes (holds qbar, kbar). */
SSA_API ssa_status_t ssa_block_scores(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                              const ssa_tensor_t* K, float* scores, void* ws,
                              size_t ws_bytes, ssa_stream_t stream);

/* Step 2: top-k block selection.
 * [digest] "Practical Implementation of SSA": keep the top-k most relevant
 * blocks.  Sel(i) = {i} plus the k_eff-1 largest scores[b,h,i,j], j < i;
 * equal scores go to the smaller j; if i + 1 <= k_eff, Sel(i) = {0..i}.
 *   scores [B, Hq, n, n] fp32 (in): only the strictly lower triangle is read.
 *     NaN scores give an unspecified (but in-range) selection.
 *   idx [B, Hq, n, k_eff] int32 (out): Sel(i) in ascending order, padded
 *     with -1 when i + 1 < k_eff.  Deterministic. */
SSA_API ssa_status_t ssa_select_topk(const ssa_dims_t* dims, const float* scores,
                             int32_t* idx, ssa_stream_t stream);

/* Step 1+2, per-token selection (dims->per_token = 1).
 * The literal reading of [digest] "Practical Implementation of SSA" ("the
 * query" is scored against every earlier block representation), as in
 * MoBA: each query token t (block i = t/s) ranks the complete earlier
 * blocks by its own query, score_j = scale * q_t . kbar_j (j < i, kbar_j the
 * mean of key block j), and keeps Sel(t) = {i} plus the k_eff-1 best (ties to
 * the smaller j; {0..i} when i + 1 <= k_eff).  Every other entry point takes
 * the resulting per-token idx when dims->per_token = 1 (the per-row-mask
 * tensor-core kernels run for bf16, the CUDA-core kernels for fp32;
 * ssa_block_scores / ssa_select_topk are per-block only and return
 * SSA_ERR_INVALID_ARG).
 *   idx [B, Hq, N, k_eff] int32 (out): Sel(t) ascending, -1 padded.
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes (pooled keys). */
SSA_API ssa_status_t ssa_select_tokens(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                               const ssa_tensor_t* K, int32_t* idx, void* ws,
                               size_t ws_bytes, ssa_stream_t stream);

/* Step 3: fused dual-stream forward.
 * One pass over every causal K/V tile keeps two disjoint online softmaxes,
 * over A_t and over D_t, and merges them at the end:
 *   h_sparse = softmax over A_t of x_tu applied to V   ([digest] "Practical
 *     Implementation of SSA"; [summary] "1. Probleemstelling": the sparse
 *     stream normalises over the selected subset only);
 *   h_full   = causal softmax over all u <= t applied to V, the counterpart
 *     output kept for alignment ([summary] "Bidirectionele Uitlijning");
 *   delta[t] = full-softmax weight on D_t, the dropped attention mass
 *     ([summary] "1. Probleemstelling"; [record] abstract); 0 when D_t is empty;
 *   lse_full[t], lse_sel[t] = natural-log normalisers of the two softmaxes.
 * x_tu = scale * q_t . k_u.
 *   idx [B, Hq, n, k_eff] int32 (in): as written by ssa_select_topk ([B, Hq,
 *     N, k_eff] from ssa_select_tokens when dims->per_token = 1).  Any
 *     other selection may be passed: entries outside [0, i] are ignored and
 *     duplicates are harmless.  A row that omits its diagonal block attends
 *     only the listed blocks; a query whose A_t is empty gets h_sparse = 0,
 *     lse_sel = -INFINITY and delta = 1.
 *   h_full, h_sparse (out): [B, Hq, N, d] strided, dims->dtype.
 *   lse_full, lse_sel, delta [B, Hq, N] fp32 (out). */
SSA_API ssa_status_t ssa_fwd_dual(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                          const ssa_tensor_t* K, const ssa_tensor_t* V,
                          const int32_t* idx, const ssa_tensor_t* h_full,
                          const ssa_tensor_t* h_sparse, float* lse_full,
                          float* lse_sel, float* delta, ssa_stream_t stream);

/* Step 4: backward of both streams with the alignment loss folded in.
 * Gradients of L = <g_full, h_full> + <g_sparse, h_sparse> + alpha * L_align
 * with L_align = L_sparsity + L_commitment, L_sparsity = MSE(h_full, sg h_sparse),
 * L_commitment = MSE(h_sparse, sg h_full), MSE = mean over all B*Hq*N*d
 * elements ([digest] "Bidirectional Attention Alignment"; [summary]
 * "Bidirectionele Uitlijning": total objective E_mode[L_ce] + alpha L_align,
 * alpha = 10 in the paper, [digest] "Alignment Weight").  g_full / g_sparse
 * carry the next stage's gradient of whichever stream is forwarded (for a
 * next-stage loss sum(h_primary) pass all-ones on the primary stream and NULL
 * on the other).  The selection is held fixed: no gradient flows through idx
 * or delta.  dK and dV are summed over the g query heads of each kv head.
 *   Q, K, V, idx, h_full, h_sparse, lse_full, lse_sel: as passed to / written
 *     by ssa_fwd_dual for the same inputs; lse_full and lse_sel must be
 *     16-byte aligned.
 *   g_full, g_sparse: [B, Hq, N, d] dims->dtype, or NULL for zero.
 *   align_loss: device fp32 scalar (out) = L_align, or NULL.
 *   dQ [B,Hq,N,d], dK, dV [B,Hkv,N,d] (out): strided, dims->dtype; fully
 *     overwritten.
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes. */
SSA_API ssa_status_t ssa_bwd_dual(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                          const ssa_tensor_t* K, const ssa_tensor_t* V,
                          const int32_t* idx, const ssa_tensor_t* h_full,
                          const ssa_tensor_t* h_sparse, const float* lse_full,
                          const float* lse_sel, const ssa_tensor_t* g_full,
                          const ssa_tensor_t* g_sparse, float alpha,
                          float* align_loss, const ssa_tensor_t* dQ,
                          const ssa_tensor_t* dK, const ssa_tensor_t* dV,
                          void* ws, size_t ws_bytes, ssa_stream_t stream);

/* Sparse stream alone, forward (inference mode).
 * [digest] "Training Efficiency Considerations": in sparse inference SSA
 * runs the same block-sparse attention operation as MoBA; [summary]
 * "4. Experimentele Resultaten" (efficiency item) reports the speed-up of
 * this mode over full attention at long context.  Computes h_sparse and lse_sel
 * exactly as ssa_fwd_dual does, but reads only the K/V blocks that a query
 * block selected; the full stream and delta are not computed.
 *   idx: as for ssa_fwd_dual (a query whose A_t is empty gets h_sparse = 0
 *     and lse_sel = -INFINITY).
 *   h_sparse [B, Hq, N, d] strided, dims->dtype (out); lse_sel [B, Hq, N] fp32
 *     (out).  Needs no workspace. */
SSA_API ssa_status_t ssa_fwd_sparse(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                            const ssa_tensor_t* K, const ssa_tensor_t* V,
                            const int32_t* idx, const ssa_tensor_t* h_sparse,
                            float* lse_sel, ssa_stream_t stream);

/* Sparse stream alone, backward.
 * Gradients of L = <g_sparse, h_sparse> for the sparse stream on its own
 * (softmax over A_t; dropped pairs get no gradient, [digest] "The Root Cause
 * Behind the Paradox"), with the selection held fixed.  dK and dV are summed
 * over the g query heads of each kv head.  Only selected (query block, key
 * block) pairs are visited.
 *   Q, K, V, idx, h_sparse, lse_sel: as passed to / written by ssa_fwd_sparse
 *     (or ssa_fwd_dual) for the same inputs; lse_sel must be 16-byte aligned.
 *   g_sparse [B, Hq, N, d] dims->dtype (in, required).
 *   dQ [B,Hq,N,d], dK, dV [B,Hkv,N,d] (out): fully overwritten; keys that no
 *     query attends get zero.
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes. */
SSA_API ssa_status_t ssa_bwd_sparse(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                            const ssa_tensor_t* K, const ssa_tensor_t* V,
                            const int32_t* idx, const ssa_tensor_t* h_sparse,
                            const float* lse_sel, const ssa_tensor_t* g_sparse,
                            const ssa_tensor_t* dQ, const ssa_tensor_t* dK,
                            const ssa_tensor_t* dV, void* ws, size_t ws_bytes,
                            ssa_stream_t stream);

/* Decode (one generated token at a time), sparse stream.
 * [digest] "Training Efficiency Considerations": at inference SSA runs its
 * sparse attention alone; [skill] "6. Inference with Sparse or Full Mode":
 * generation appends one token per step.  The token at position t (block
 * i = t/s) selects blocks by the forward's rule, with the query side read as
 * the mean of the queries of block i seen so far (positions i*s..t; at the
 * last token of a block this is exactly the forward's block mean):
 *   score_j = scale * qbar . kbar_j (j < i, kbar_j the mean of key block j),
 *   Sel = {i} + the k_eff-1 best scores (ties to the smaller j), or {0..i}
 *   when i + 1 <= k_eff;  h = softmax over A_t of scale q_t . k_u, times V.
 * Two state buffers carry the pooling between calls:
 *   qsum [B, Hq, d] fp32: sum of the queries of the current block so far;
 *   kbar [B, Hkv, n, d] fp32: means of the complete key blocks (16-byte
 *     aligned for the decode step).
 * dims->N is the capacity of the K/V caches [B, Hkv, N, d] (a multiple of
 * block); the decode step needs k_eff <= 64 and its shared memory (the g
 * heads' scores of one eighth of the pooled blocks and their candidate lists,
 * queries, partial outputs and selections, two 64-key K/V chunks) must fit a
 * CTA (SSA_ERR_UNSUPPORTED otherwise; every workload here fits).  Its copies
 * into shared memory are waited on with a bound: a wait that runs out records
 * SSA_ERR_TIMEOUT in the per-device report that ssa_device_status reads. */

/* Builds the decode state from a prompt of t0 tokens (0 <= t0 <= N): kbar of
 * the complete blocks 0 .. t0/s - 1 and qsum of the queries of the partial
 * block (rows (t0/s)*s .. t0-1; zero when t0 is a multiple of s).
 *   Q [B, Hq, N, d], K [B, Hkv, N, d] (in): the prompt's rows 0 .. t0-1. */
SSA_API ssa_status_t ssa_decode_prefill(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                                const ssa_tensor_t* K, int32_t t0, float* qsum,
                                float* kbar, ssa_stream_t stream);

/* One decode step for the token at position t (0 <= t < N).
 *   q [B, Hq, 1, d] (in): the token's queries.
 *   K, V [B, Hkv, N, d] (in): caches whose rows 0 .. t hold the keys and
 *     values so far (the caller has written row t).
 *   qsum, kbar (in/out): state as left by ssa_decode_prefill(t0 = t) or by
 *     the call for t-1; q_t is added to qsum (which restarts at a block's
 *     first token) and, when t is the last token of block i, kbar[i] is set
 *     to the mean of that block's keys.
 *   h [B, Hq, 1, d] (out), lse [B, Hq] fp32 (out, natural log of the
 *     softmax normaliser), idx [B, Hq, k_eff] int32 (out, Sel ascending,
 *     -1 padded).
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes (checked; the
 *     step keeps its scratch in the shared memory of one thread-block cluster
 *     per (batch, kv head) and does not write it).
 * Calls for consecutive tokens must be ordered (same stream). */
SSA_API ssa_status_t ssa_decode_step(const ssa_dims_t* dims, const ssa_tensor_t* q,
                             const ssa_tensor_t* K, const ssa_tensor_t* V, int32_t t,
                             float* qsum, float* kbar, const ssa_tensor_t* h, float* lse,
                             int32_t* idx, void* ws, size_t ws_bytes, ssa_stream_t stream);

/* Standalone dropped attention mass, without V.
 * delta[t] = sum over u in D_t of exp(x_tu - lse_full[t]) ([summary]
 * "1. Probleemstelling"; [digest] "Phenomenon 3" reports this quantity for
 * full-attention models).  The sum runs over D_t directly (not 1 - sum over
 * A_t) so small masses keep their relative precision.
 *   lse_full [B, Hq, N] fp32 (in) or NULL: when NULL the causal log-sum-exp is
 *     computed in the same pass.
 *   delta [B, Hq, N] fp32 (out).
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes. */
SSA_API ssa_status_t ssa_dropped_mass(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                              const ssa_tensor_t* K, const int32_t* idx,
                              const float* lse_full, float* delta, void* ws,
                              size_t ws_bytes, ssa_stream_t stream);

/* Forward value of the alignment loss on its own.
 * loss (out): device fp32[2] = {L_sparsity, L_commitment}, each the mean of
 * (h_full - h_sparse)^2 over all B*Hq*N*d elements ([digest] "Bidirectional
 * Attention Alignment").  Deterministic (fixed-order reduction).
 *   ws: workspace of at least ssa_workspace_bytes(dims) bytes. */
SSA_API ssa_status_t ssa_align_mse(const ssa_dims_t* dims, const ssa_tensor_t* h_full,
                           const ssa_tensor_t* h_sparse, float* loss, void* ws,
                           size_t ws_bytes, ssa_stream_t stream);

/* Capacity, in floats, of the fixed device scratch array used by
 * ssa_block_scores_noalloc: B * (Hq + Hkv) * n * d must not exceed it
 * (4 Mi floats = 16 MiB; the gqa_16k, long_64k and sweep_32k shapes fit). */
#define SSA_NOALLOC_SCRATCH_FLOATS (4u << 20)

/* ssa_block_scores without a caller-supplied workspace.
 * The paper has no counterpart: this exists for callers that cannot call
 * cudaMalloc -- for example code running inside a host framework that owns
 * all device memory and only hands out the tensors it allocated itself, or a
 * latency-critical loop where an allocation (and the device synchronisation
 * a cudaFree implies) is not acceptable.  It computes exactly what
 * ssa_block_scores computes, from the same kernels, but keeps the pooled
 * block means in a fixed array of SSA_NOALLOC_SCRATCH_FLOATS floats that the
 * library declares in device memory; every GPU that loads the library holds
 * those 16 MiB until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   Q, K, scores: as for ssa_block_scores (the caller still owns inputs and
 *     outputs).
 *   Returns SSA_ERR_WORKSPACE, enqueuing nothing, when
 *     B * (Hq + Hkv) * n * d > SSA_NOALLOC_SCRATCH_FLOATS.
 * The first call on a device looks up the array's device address once (with
 * that device current) and caches it; make that first call before any
 * stream capture.  After cudaDeviceReset the next call looks the address up
 * again in the device's new context (so that call, too, belongs before any
 * capture).  All calls share the one array and it keeps the last
 * call's contents; nothing in it needs to start at zero, because every value
 * the scoring kernel reads was written by the same call.  Calls whose work
 * overlaps on the GPU (different streams, or different host threads without
 * ordering) race on the array: order them on one stream. */
SSA_API ssa_status_t ssa_block_scores_noalloc(const ssa_dims_t* dims, const ssa_tensor_t* Q,
                                              const ssa_tensor_t* K, float* scores,
                                              ssa_stream_t stream);

/* Number of kernels this library has enqueued in this process so far (all
 * devices, all threads).  Lets a caller count the launches of a region. */
SSA_API uint64_t ssa_launch_count(void);

/* Failure-detection self-test.  Enqueues a one-CTA kernel that waits on a
 * barrier nothing will ever complete, using the same bounded wait as every
 * tensor-core kernel; after about 10 ms the wait gives up, the kernel records
 * SSA_ERR_TIMEOUT in the device status report and returns.  Nothing faults
 * or hangs; the report then reads as after a real timeout (read and clear it
 * with ssa_device_status).  Returns SSA_ERR_UNSUPPORTED off sm_100. */
SSA_API ssa_status_t ssa_selftest_timeout(ssa_stream_t stream);

/* Synchronises `stream`, copies the status report of the current device to
 * *status (SSA_OK, or SSA_ERR_TIMEOUT once any kernel of this library on the
 * device -- any stream, any host thread -- gave up on a wait since the last
 * clear) and, if clear != 0, resets it.  The report is only read here: no
 * kernel consults it.  Returns SSA_ERR_CUDA if the synchronisation or the
 * copy fails. */
SSA_API ssa_status_t ssa_device_status(int32_t* status, int clear, ssa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
