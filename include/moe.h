/*
 * moe.h -- C ABI of a B200 (sm_100a) MoE-layer forward library.
 *
 * One forward pass of a Switch / top-k mixture-of-experts layer, split into the
 * stages the layer is made of: router + top-k, optimal-assignment balancing,
 * capacity slots, dispatch, expert FFN, combine, load statistics. Every stage
 * runs in hand-written CUDA kernels; there is no host fallback.
 *
 * Conventions (all calls):
 *  - Every array pointer is a DEVICE pointer owned by the caller; the library
 *    never allocates device memory. Calls that need scratch take a `workspace`
 *    of at least the size returned by the matching *_workspace_size() query
 *    (which is a pure host function and may be called without a GPU).
 *  - Arrays are dense and row-major; shapes are given as [rows, cols].
 *    Integer arrays are int32, floating-point statistics fp32.
 *  - Every call is asynchronous: it validates its arguments on the host,
 *    enqueues kernels on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns. It does not synchronise, except where stated.
 *  - Return value: MOE_OK, or an error code; the message of the last error on
 *    the calling thread is available from moe_last_error(). Invalid arguments
 *    are rejected before anything is enqueued. Conditions only the device can
 *    see (an expert index out of range, more kept rows than a buffer holds)
 *    set a device error word that moe_sync_status() reports.
 *  - Notation follows the pages: m tokens, n experts, k experts per token,
 *    d model width, d_ff expert hidden width, scores s_ij, capacity C.
 *  - Limits: 1 <= k <= n <= 256; d a multiple of 8 (bf16) or 4 (fp32);
 *    d_ff a multiple of 8; m * k < 2^31.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_NOT_CONVERGED = 5,
    MOE_ERR_INTERNAL = 6
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_SOFTMAX = 0, MOE_SIGMOID = 1 } moe_score_fn;
typedef enum { MOE_QB_STEP = 0, MOE_QB_SOLVE = 1 } moe_qb_mode;
typedef enum { MOE_QB_MIDPOINT = 0, MOE_QB_BOUNDARY = 1, MOE_QB_BIP = 2 } moe_qb_threshold;

/* Copies the message of the calling thread's last error (NUL-terminated, truncated to len). */
MOE_API void moe_last_error(char* buf, size_t len);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device. Returns MOE_OK, or MOE_ERR_INTERNAL / MOE_ERR_INVALID_ARG
 * for a condition a kernel detected (the message says which), or MOE_ERR_CUDA.
 */
MOE_API moe_status moe_sync_status(moe_stream_t stream);

/*
 * Self-test of the bounded waits (no passage: an engineering check). One warp
 * waits until the int32 *flag (device memory) is at least 1, polling it the
 * way the FFN's second-GEMM tiles poll their per-expert counters, for at most
 * limit_cycles SM clock cycles (0 .. 4e9; the library's own waits use 4e9,
 * about 2 s). If nothing sets the flag the wait gives up, the device error
 * word records a pipeline timeout, and the kernel returns: the next
 * moe_sync_status reports MOE_ERR_INTERNAL ("a pipeline wait timed out") and
 * the context stays usable. Asynchronous on `stream`; the flag is only read.
 * Errors: MOE_ERR_INVALID_ARG (NULL flag, limit out of range), MOE_ERR_CUDA.
 */
MOE_API moe_status moe_selftest_wait(const int32_t* flag, int64_t limit_cycles, moe_stream_t stream);

/*
 * Router and top-k selection.
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), Switch
 * Routing Steps 1-3 (h = x W_r, p = softmax(h), i* = argmax p, gate p_i*) and
 * selective precision (router projection and softmax in fp32); the Shazeer
 * gate Softmax(TopK(x W_g)) for k >= 2; "MoE travelogue 6"
 * (kexue.fm/archives/11619), Method review eq. (1): Loss-Free ranks by
 * rho + b and weights by rho.
 *
 *  x          [m, d] activations, dtype x_dtype (MOE_F32 or MOE_BF16); upcast to fp32.
 *  w_r        [d, n] fp32 router weight.
 *  logits_in  [m, n] fp32, or NULL. When given, x and w_r are ignored and h = logits_in.
 *  fn         MOE_SOFTMAX: p = softmax(h); MOE_SIGMOID: rho = 1 / (1 + exp(-h)).
 *  renorm_topk  softmax with k >= 2 only: gate = softmax over the k selected
 *             logits (p_sel / sum of selected p); otherwise gate = p_sel.
 *  rank_bias  [n] fp32 Loss-Free bias b, or NULL. Ranking key fp32(score) + b
 *             (fp32 add); without it the key is h (softmax) or rho (sigmoid).
 *  probs_out  [m, n] fp32 scores p or rho, or NULL.
 *  topk_idx   [m, k] out: selected experts, best key first; equal keys -> lower index first.
 *  topk_gate  [m, k] out: fp32 gates (rho_sel for sigmoid).
 *  workspace  bf16 x with n <= 128: [3, n, d] bf16 split of W_r (w = w0 + w1 + w2, each
 *             bf16) so the projection runs on the tensor cores with exact products and
 *             fp32 accumulation; size from moe_router_topk_workspace_size (0 otherwise).
 *             With w_r given, every call re-makes the split. With w_r == NULL (this
 *             tensor-core path only) the call uses the split that moe_router_prepare
 *             left in the workspace: the router weight is static across forwards, so it
 *             is split once (the caller keeps the workspace unchanged in between).
 * All h, p, rho and keys are fp32. Errors: MOE_ERR_INVALID_ARG for bad shapes
 * or NULL required pointers (w_r == NULL off the tensor-core path); MOE_ERR_WORKSPACE
 * for a missing or short workspace.
 */
MOE_API size_t moe_router_topk_workspace_size(int32_t d, int32_t n, int32_t k, moe_dtype x_dtype);
MOE_API moe_status moe_router_topk(const void* x, moe_dtype x_dtype, const float* w_r, const float* logits_in, int64_t m,
                           int32_t d, int32_t n, int32_t k, moe_score_fn fn, int32_t renorm_topk,
                           const float* rank_bias, float* probs_out, int32_t* topk_idx, float* topk_gate,
                           void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Prepare the router weight once: write the [3, n, d] bf16 split of W_r into the
 * workspace of moe_router_topk, which later calls with w_r == NULL use as is.
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), selective
 * precision: the router computes in fp32; the split keeps every product exact
 * on the bf16 tensor cores (w = w0 + w1 + w2, each part bf16).
 *  w_r [d, n] fp32; k and x_dtype as in moe_router_topk (they pick the path).
 *  workspace: moe_router_topk_workspace_size(d, n, k, x_dtype) bytes, 16-byte aligned.
 * Errors: MOE_ERR_UNSUPPORTED when the shape takes the fp32 FMA router (no split:
 * pass w_r to moe_router_topk); MOE_ERR_INVALID_ARG; MOE_ERR_WORKSPACE.
 */
MOE_API moe_status moe_router_prepare(const float* w_r, int32_t d, int32_t n, int32_t k, moe_dtype x_dtype,
                                      void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Optimal-assignment balancing (Quantile Balancing) with an exact finish.
 * Passage: "MoE travelogue 6: optimal assignment promotes balance"
 * (kexue.fm/archives/11619): Linear programming eq. (3) (maximise sum x_ij s_ij
 * with sum_j x_ij = k and sum_i x_ij = C = m k / n), the dual (8)-(11), the
 * alternating QB algorithm box, and its practical one-step form under
 * "Mind the pitfall" (select with the old beta, then update beta).
 *
 *  s          [m, n] fp32 scores, row-major, finite (no NaN or infinity: the results are
 *             unspecified otherwise), any 4-byte alignment (rows that start on 16-byte
 *             boundaries take the faster bulk-copy and vector paths). (m * k) % n must be 0
 *             and k < n.
 *  beta       [n] fp32, in: previous beta (zeros for a cold start); out: new beta.
 *  mode       MOE_QB_STEP: x = topk(s - beta_old); one alpha/beta update -> beta_new.
 *             MOE_QB_SOLVE: alternate row/column passes until topk(s - beta) has
 *             every column count equal to C or max_iters beta updates are done,
 *             then move the remaining excess with successive shortest paths on
 *             the n-expert graph (at most max_repair moves), which yields the
 *             optimum of eq. (3). beta returns the last QB beta.
 *  rule       threshold between the two neighbouring order statistics:
 *             MOE_QB_MIDPOINT fp32(fp32(a + b) * 0.5) (default) or
 *             MOE_QB_BOUNDARY the (k+1)-th / (C+1)-th largest (the page's convention);
 *             MOE_QB_BIP the BIP variant ("Related work", problem (12) with inequality
 *             constraints and non-negative duals): the (k+1)-th / (C+1)-th largest
 *             clipped at zero, max(0, .).
 *  topk_idx   [m, k] out: each token's experts in ascending index order.
 *  info       [4] int32 device out: beta updates done, repair moves, excess left
 *             (0 = balanced), tokens whose k-th and (k+1)-th values of s - beta
 *             tie in the last row pass.
 * SOLVE synchronises `stream` between phases (its loop length depends on the
 * data) and returns MOE_ERR_NOT_CONVERGED if max_repair moves did not remove
 * the excess. STEP is fully asynchronous.
 * workspace: moe_balance_assign_workspace_size bytes (device, caller-owned, any
 * contents on entry; the call clears what it needs). It holds s transposed
 * (SOLVE), alpha, the column pass's per-expert windows and candidate lists, and
 * the exact finish's arc costs and membership bitmap.
 */
MOE_API size_t moe_balance_assign_workspace_size(int64_t m, int32_t n, int32_t k, moe_qb_mode mode);
MOE_API moe_status moe_balance_assign(const float* s, int64_t m, int32_t n, int32_t k, float* beta, moe_qb_mode mode,
                              moe_qb_threshold rule, int32_t max_iters, int32_t max_repair, int32_t* topk_idx,
                              int32_t* info, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * One SignSGD step on beta, in place of the quantile update.
 * Passage: "MoE travelogue 6" (kexue.fm/archives/11619), "Gradient descent",
 * eqs. (15)-(17): with alpha given, l(beta) = sum_ij max(0, s_ij - alpha_i - beta_j)
 * + (m k / n) sum_j beta_j has dl/dbeta_j = m k / n - sum_i chi(s_ij - alpha_i - beta_j > 0),
 * and beta_j <- beta_j - gamma sign(dl/dbeta_j).
 *  The row pass selects x = topk(s - beta_old) and sets alpha by `rule`, as the
 *  STEP mode of moe_balance_assign. Then count_j = #{i : fp32(s_ij - alpha_i) > beta_j}
 *  (exact integers) and beta_j moves by gamma (one fp32 add or subtract; no move
 *  when count_j = m k / n).
 *  s, beta, rule, topk_idx, info, workspace: as moe_balance_assign (STEP).
 *  The workspace of moe_balance_assign_workspace_size(m, n, k, MOE_QB_STEP) serves.
 */
MOE_API moe_status moe_balance_sign_step(const float* s, int64_t m, int32_t n, int32_t k, float* beta, float gamma,
                                 moe_qb_threshold rule, int32_t* topk_idx, int32_t* info, void* workspace,
                                 size_t ws_bytes, moe_stream_t stream);

/*
 * The practical QB step with beta averaged over mini-batches.
 * Passage: "MoE travelogue 6" (kexue.fm/archives/11619), Mind the pitfall, closing
 * paragraph: with m in the millions the exact (m k / n + 1)-th largest per expert is
 * too costly, so the batch is split into mini-batches, beta is computed on each by
 * the formula, and the results are averaged.
 *  x = topk(s - beta_old) and alpha from s - beta_old over the whole batch (as the
 *  STEP of moe_balance_assign: select with the old beta, then update). Mini-batch b
 *  holds tokens b seg_len .. (b + 1) seg_len - 1; its beta_b comes from its own
 *  column pass with C_b = seg_len k / n and the threshold `rule`. The new beta is
 *  beta_j = fp32((sum over b, in order, of (double) beta_b_j) / (m / seg_len)).
 *  seg_len = m gives moe_balance_assign's STEP, bit for bit.
 *  s, beta, rule, topk_idx, info, workspace: as moe_balance_assign (STEP; info[0] = 1).
 *  Requires seg_len | m, (seg_len k) % n == 0 and m / seg_len <= 4096.
 *  Fully asynchronous. Workspace: moe_balance_assign_workspace_size.
 */
MOE_API moe_status moe_balance_step_minibatch(const float* s, int64_t m, int32_t n, int32_t k, float* beta,
                                              moe_qb_threshold rule, int64_t seg_len, int32_t* topk_idx,
                                              int32_t* info, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Capacity slots and the expert-major row layout.
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), Expert
 * Capacity and token drop (capacity = tokens / experts x capacity factor;
 * overflow skips the expert and rides the residual connection); "Switch
 * Transformer read for implementation" (molayo1419.me), the dispatch
 * permutation and the expert capacity example.
 *
 * Within each segment of seg_len tokens (a micro-batch; seg_len = m for one
 * segment), the assignments (token i, pick r) are visited in token order; the
 * j-th assignment to expert e (j from 0) gets slot j, kept iff j < capacity.
 *  topk_idx       [m, k] expert ids (a token lists distinct experts).
 *  capacity       per expert per segment (>= seg_len * k: nothing is dropped).
 *  slot           [m, k] out: slot or -1 (dropped).
 *  dest_row       [m, k] out: row in the expert-major buffer, or -1.
 *  src_token      [m * k] out: src_token[row] = token; the first `rows` entries are
 *                 written, rows = expert_offsets[n] (rows of expert e are
 *                 expert_offsets[e] .. expert_offsets[e+1]-1, segment by segment,
 *                 token order inside).
 *  expert_offsets [n + 1] out; routed_count, kept_count [m / seg_len, n] out
 *                 (routed = before capacity, kept = min(routed, capacity)).
 * Errors: MOE_ERR_INVALID_ARG (seg_len must divide m, capacity >= 0),
 * MOE_ERR_WORKSPACE. An expert id outside [0, n) sets the device error word.
 */
MOE_API size_t moe_capacity_slots_workspace_size(int64_t m, int32_t k, int32_t n, int64_t seg_len);
MOE_API moe_status moe_capacity_slots(const int32_t* topk_idx, int64_t m, int32_t k, int32_t n, int32_t capacity,
                              int64_t seg_len, int32_t* slot, int32_t* dest_row, int32_t* src_token,
                              int32_t* expert_offsets, int32_t* routed_count, int32_t* kept_count, void* workspace,
                              size_t ws_bytes, moe_stream_t stream);

/*
 * Capacity slots with no caller-provided scratch. The pages have no
 * counterpart: this is a convenience for callers that cannot allocate device
 * memory or pass a workspace -- for example code reached through a fixed
 * foreign-function signature that carries only inputs and outputs, or a host
 * framework that owns all device memory and forbids its plugins to call
 * cudaMalloc (which may also synchronise the device).
 *  Arguments and results: exactly those of moe_capacity_slots, minus the workspace.
 *  Scratch: a fixed 1 MiB array compiled into the library (every GPU that
 *  loads the library keeps it until the process exits). A problem needing more
 *  (moe_capacity_slots_workspace_size > 1 MiB) is rejected with
 *  MOE_ERR_WORKSPACE before anything is enqueued; use moe_capacity_slots then.
 *  The first call on a device looks up the array's device address with
 *  cudaGetSymbolAddress while that device is current; make that first call
 *  before any stream capture. `stream` must belong to the current device
 *  (MOE_ERR_INVALID_ARG otherwise). Invalid arguments are rejected before the
 *  lookup, with the same checks and codes as moe_capacity_slots.
 *  All calls share the one array and it keeps the last call's contents (no
 *  word of it needs to start at zero: every word read is first written by the
 *  same call). Calls that overlap on the GPU -- on different streams, or from
 *  threads that do not order their streams -- race on it; order them.
 */
MOE_API moe_status moe_capacity_slots_static(const int32_t* topk_idx, int64_t m, int32_t k, int32_t n,
                                             int32_t capacity, int64_t seg_len, int32_t* slot, int32_t* dest_row,
                                             int32_t* src_token, int32_t* expert_offsets, int32_t* routed_count,
                                             int32_t* kept_count, moe_stream_t stream);

/*
 * Dispatch: gather tokens into expert-major order.
 * Passage: "Switch Transformer read for implementation" (molayo1419.me), the
 * forward pass changes token order twice (first: group tokens by expert).
 *  x [m, d] (dtype dt) -> xbuf [max_rows, d]: xbuf[r] = x[src_token[r]] for
 *  r < expert_offsets[n] (read on the device). max_rows is the capacity of xbuf
 *  in rows; more kept rows than that set the device error word.
 */
MOE_API moe_status moe_dispatch(const void* x, moe_dtype dt, int64_t m, int32_t d, const int32_t* src_token,
                        const int32_t* expert_offsets, int32_t n, int64_t max_rows, void* xbuf, moe_stream_t stream);

/*
 * Dispatch, token-major: the same expert-major rows as moe_dispatch, written by
 * visiting tokens instead of rows, so each token's activations are read once
 * however many of its picks are kept (with k picks per token moe_dispatch
 * reads a token once per kept pick).
 * Passage: as moe_dispatch ("Switch Transformer read for implementation",
 * molayo1419.me: the first of the two permutations groups tokens by expert).
 *  x [m, d] (dtype dt); dest_row [m, k] from moe_capacity_slots (-1 = dropped).
 *  xbuf [max_rows, d] out: xbuf[dest_row[i, r]] = x[i] for every dest_row[i, r] >= 0;
 *  a row index >= max_rows is skipped and sets the device error word.
 *  Results: bit for bit those of moe_dispatch on the same capacity outputs.
 */
MOE_API moe_status moe_dispatch_tokens(const void* x, moe_dtype dt, int64_t m, int32_t d, int32_t k,
                                       const int32_t* dest_row, int64_t max_rows, void* xbuf, moe_stream_t stream);

/*
 * Expert FFN on the expert-major rows: for the rows of expert e,
 *   ybuf = max(0, xbuf W1_e + b1_e) W2_e + b2_e.
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), Switch
 * Layer: FFN(x) = max(0, x W1 + b1) W2 + b2 replicated per expert.
 *  xbuf [max_rows, d], ybuf [max_rows, d]: dtype dt; rows per expert from
 *       expert_offsets [n+1] (device; rows = expert_offsets[n] <= max_rows).
 *  w1   [n, d_ff, d]: W1_e stored output-major (the nn.Linear weight layout, row j
 *       holds the weights of hidden unit j); b1 [n, d_ff].
 *  w2   [n, d, d_ff]: W2_e output-major; b2 [n, d]. Weights and biases have dtype dt.
 *  bf16: bf16 x bf16 products with fp32 accumulation on the tensor cores; the
 *  hidden activation is rounded to bf16 between the two GEMMs.
 *  fp32: fp32 FMA throughout.
 *  workspace holds the hidden activations [max_rows, d_ff] (dtype dt).
 */
MOE_API size_t moe_expert_ffn_workspace_size(moe_dtype dt, int64_t max_rows, int32_t d_ff);
MOE_API moe_status moe_expert_ffn(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                          const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d, int32_t d_ff,
                          int64_t max_rows, void* ybuf, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Expert FFN reading its rows straight from the token-major activations (bf16).
 * Passage: "Switch Transformer read for implementation" (molayo1419.me): the
 * dispatch permutation groups tokens by expert before the FFN; here the FFN's
 * first GEMM loads row r of the expert-major order as x[src_token[r]], so the
 * permuted copy xbuf is never formed.
 *  x [m, d] token-major; src_token [rows] from moe_capacity_slots; other
 *  arguments as moe_expert_ffn. ybuf [max_rows, d] out, expert-major.
 *  Results: bit for bit those of moe_dispatch followed by moe_expert_ffn. Measured
 *  slower than that pair on the B200 (the row gather feeds the tensor cores more slowly
 *  than tile loads of xbuf); its use is saving the xbuf buffer (max_rows x d elements).
 *  bf16 only (MOE_ERR_UNSUPPORTED for fp32). Workspace: moe_expert_ffn_workspace_size.
 */
MOE_API moe_status moe_expert_ffn_gather(const void* x, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                                 const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d, int32_t d_ff,
                                 int64_t max_rows, const int32_t* src_token, int64_t m, void* ybuf, void* workspace,
                                 size_t ws_bytes, moe_stream_t stream);

/*
 * Expert FFN and combine in one call, for one pick per token (k = 1, bf16).
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), Switch
 * Routing Step 3 (y = p_i* E_i*(x)) with "Switch Transformer read for
 * implementation" (molayo1419.me): with top-1 routing each expert-major row
 * belongs to one token, so the FFN's second GEMM writes that token's output
 * directly, gated, and ybuf is never formed.
 *  Arguments as moe_expert_ffn (without ybuf) and moe_combine with k = 1:
 *  src_token [rows] and dest_row [m] from moe_capacity_slots, topk_gate [m],
 *  residual [m, d] or NULL (must not alias y), y [m, d] out.
 *  Results: bit for bit those of moe_expert_ffn followed by moe_combine (the
 *  same roundings in the same order); dropped tokens get the residual or zeros.
 *  max_rows <= m. bf16 only: MOE_ERR_UNSUPPORTED for fp32 (call the two
 *  entry points). Workspace: moe_expert_ffn_workspace_size.
 */
MOE_API moe_status moe_expert_ffn_combine(const void* xbuf, moe_dtype dt, const void* w1, const void* b1,
                                  const void* w2, const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d,
                                  int32_t d_ff, int64_t max_rows, const int32_t* src_token, const int32_t* dest_row,
                                  const float* topk_gate, const void* residual, int64_t m, void* y, void* workspace,
                                  size_t ws_bytes, moe_stream_t stream);

/*
 * Combine: inverse permute, gate, and join the residual path.
 * Passage: "Switch Transformer read for implementation" (molayo1419.me):
 * restore token order, multiply by the gate, join the residual; overflow
 * tokens keep only the residual. "Switch Transformers paper review", Step 3.
 *  y[i] = (residual ? residual[i] : 0) + sum over r with dest_row[i,r] >= 0 of
 *         g_ir * ybuf[dest_row[i,r]]
 *  fp32 accumulation; for dt = MOE_BF16 each gate is first rounded to bf16 (the
 *  selective-precision recipe casts the gate back to bf16). y [m, d] has dtype dt.
 *  residual may be NULL; it must not alias y.
 */
MOE_API moe_status moe_combine(const void* ybuf, moe_dtype dt, const int32_t* dest_row, const float* topk_gate,
                       const void* residual, int64_t m, int32_t k, int32_t d, void* y, moe_stream_t stream);

/*
 * Expert parallelism over G ranks (one GPU each), three calls around the owner's FFN.
 * Passage: "Switch Transformer read for implementation" (molayo1419.me), Expert
 * Parallelism (experts on different devices: the dispatch and the return of the
 * outputs become exchanges between devices, kept apart from the compute); "Switch
 * Transformers paper review" (tildalice.io/?p=118), distributed training and
 * communication cost (an all-to-all before the experts and one after them).
 *
 * Rank q owns experts q E .. q E + E - 1, E = n / G (n % G == 0). Each rank routes its
 * own m tokens over all n experts and runs moe_capacity_slots on them (capacity is per
 * source rank). The caller gathers every rank's expert_offsets [n + 1] into
 * offsets_all [G, n + 1] (rank-major; one all-gather of n + 1 int32 per rank). Owner
 * q's receive buffer then holds its local experts in order, each expert's rows from
 * source rank 0 first, then rank 1, ..., each source's rows in its own expert-major
 * order: the rows the one-GPU layer gives the expert on the concatenated batch with
 * one capacity segment per rank.
 *
 * moe_ep_plan: from offsets_all (device), this rank's send_base [n] (the row of expert
 *   e's owner's buffer where this rank's rows of e start) and recv_offsets [E + 1] (the
 *   row offsets of this rank's local experts in its own receive buffer; recv_offsets[E]
 *   = its rows). recv_offsets and this rank's E experts' weights are what moe_expert_ffn
 *   takes (n = E) to run the owner's FFN on its receive buffer.
 * moe_ep_dispatch: x [m, d] -> the owners' receive buffers. peer_xrecv is a DEVICE array
 *   of G device pointers, entry q = rank q's receive buffer [max_recv_rows, d] mapped into
 *   this GPU's address space (peer access: CUDA IPC or symmetric memory; entry `rank` is
 *   this rank's own buffer). Each token is read once and stored to each kept pick's row
 *   of its owner's buffer (plain 16-byte stores, no TMA). ep_row [m, k] out: the pick's
 *   row in its owner's buffer, or -1 (dropped). topk_idx, dest_row, expert_offsets: this
 *   rank's router and capacity outputs; send_base from moe_ep_plan.
 * moe_ep_combine: y[i] = (residual[i]) + sum over kept picks r of g_ir * yrecv_q[ep_row[i, r]]
 *   with q = topk_idx[i, r] / E, read through peer_yrecv (a DEVICE array of G pointers to
 *   the ranks' expert outputs [max_recv_rows, d]); fp32 accumulation in pick order and,
 *   for bf16, gates rounded to bf16 first: the operations of moe_combine, so the result is
 *   bit for bit the one-GPU layer's.
 * Ordering across ranks is the caller's: every rank's dispatch completes before any owner
 * runs its FFN, and every FFN before any combine reads it (the kernels wait on nothing).
 * Errors: MOE_ERR_INVALID_ARG; a row outside [0, max_recv_rows) sets the device error word.
 */
MOE_API moe_status moe_ep_plan(const int32_t* offsets_all, int32_t G, int32_t n, int32_t rank, int32_t* send_base,
                               int32_t* recv_offsets, moe_stream_t stream);
MOE_API moe_status moe_ep_dispatch(const void* x, moe_dtype dt, int64_t m, int32_t d, int32_t k, int32_t n, int32_t G,
                                   const int32_t* topk_idx, const int32_t* dest_row, const int32_t* expert_offsets,
                                   const int32_t* send_base, void* const* peer_xrecv, int64_t max_recv_rows,
                                   int32_t* ep_row, moe_stream_t stream);
MOE_API moe_status moe_ep_combine(const void* const* peer_yrecv, moe_dtype dt, const int32_t* ep_row,
                                  const int32_t* topk_idx, int32_t n, int32_t G, const float* topk_gate,
                                  const void* residual, int64_t m, int32_t k, int32_t d, void* y, moe_stream_t stream);

/*
 * Load statistics, auxiliary loss and the Loss-Free bias update.
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), auxiliary
 * load balancing loss L = alpha N sum_i f_i P_i; "Qwen global-batch load
 * balance" (agentlenshq.com): per-micro-batch loss averaged vs f_i pooled over
 * the global batch; "MoE travelogue 6", Demo code (MaxVio/MinVio/AvgVio) and
 * eq. (2) (b <- b - gamma sign(F - 1/n)).
 *
 *  probs     [m, n] router scores (p or rho), or NULL (then P and aux are not written).
 *  topk_idx  [m, k] routing decision (counts are taken before capacity).
 *  seg_len   micro-batch length (divides m); nseg = m / seg_len.
 *  f, P      [nseg + 1, n] out (row nseg: whole batch). f_i = count_i / (k m_seg).
 *  aux       [nseg + 3] out: per segment, the mean over segments (micro-batch
 *            loss), the loss on pooled f and P (global-batch loss), and the hybrid
 *            loss of "Qwen global-batch load balance" (balancing efficiency and
 *            effectiveness): the global-batch loss plus 0.01 x the micro-batch loss.
 *  vio       [3] out: MaxVio, MinVio, AvgVio of the pooled counts, or NULL.
 *  bias_inout [n] Loss-Free bias updated in place with step gamma, or NULL; the
 *            sign is decided exactly from the integer counts.
 * Accumulation is fp64 in a fixed order (the results are deterministic).
 */
MOE_API size_t moe_balance_stats_workspace_size(int64_t m, int32_t n, int64_t seg_len);
MOE_API moe_status moe_balance_stats(const float* probs, const int32_t* topk_idx, int64_t m, int32_t n, int32_t k,
                             int64_t seg_len, float alpha, float* f, float* P, float* aux, float* vio,
                             float* bias_inout, float gamma, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Router gradient of the balance loss (the backward of the statistics stage).
 * Passage: "Switch Transformers paper review" (tildalice.io/?p=118), auxiliary load
 * balancing loss: f_i is set by the argmax and is not differentiable, P_i (the mean
 * score) is, so minimising f_i P_i sends the gradient through P_i; "Qwen global-batch
 * load balance" (agentlenshq.com) for the micro-batch / global-batch losses.
 *  Loss: w_global L_global + w_micro L_micro (L_global = alpha n sum_i f^G_i P^G_i,
 *  L_micro = mean over segments of alpha n sum_i f^s_i P^s_i; w_global = 1, w_micro =
 *  0.01 is the hybrid loss aux[nseg + 2] of moe_balance_stats).
 *  probs   [m, n] router scores of moe_router_topk (p for MOE_SOFTMAX, rho for MOE_SIGMOID).
 *  f       [nseg + 1, n] of moe_balance_stats with the same seg_len (held fixed).
 *  dlogits [m, n] out: dL/dh, h the router logits: softmax p_j (g_j - sum_i p_i g_i),
 *          sigmoid g_j p_j (1 - p_j), with g_i = w_global alpha n f^G_i / m +
 *          w_micro alpha n f^s_i / (nseg seg_len) for a token of segment s. fp32.
 */
MOE_API moe_status moe_balance_loss_grad(const float* probs, moe_score_fn fn, const float* f, int64_t m, int32_t n,
                                         int64_t seg_len, float alpha, float w_micro, float w_global, float* dlogits,
                                         moe_stream_t stream);

/*
 * Global-batch statistics across data-parallel ranks, step 1 of 3: this rank's totals.
 * Passage: "Qwen global-batch load balance for MoE LLM training" (agentlenshq.com):
 * the global batch spans every data-parallel rank, so f_i is synchronised across the
 * ranks (the counts are summed) before the loss is computed on the pooled values.
 *
 *  probs     [m, n] router scores of this rank's m tokens, or NULL (then row 1 is 0).
 *  topk_idx  [m, k] routing decision of this rank's tokens.
 *  totals    [2, n] fp64 out: row 0 = routed copies per expert (exact integers),
 *            row 1 = sum over the m tokens of probs[:, e] (fixed-order fp64).
 *  workspace moe_balance_totals_workspace_size(m, n) bytes.
 * Step 2 (the caller's): sum `totals` element-wise over the ranks (one all-reduce of
 * 2 n doubles, e.g. NCCL on the device buffer). Step 3: moe_balance_global.
 * Errors: MOE_ERR_INVALID_ARG, MOE_ERR_WORKSPACE.
 */
MOE_API size_t moe_balance_totals_workspace_size(int64_t m, int32_t n);
MOE_API moe_status moe_balance_totals(const float* probs, const int32_t* topk_idx, int64_t m, int32_t n, int32_t k,
                              double* totals, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Global-batch statistics across data-parallel ranks, step 3 of 3.
 * Passage: as moe_balance_totals; the loss L = alpha N sum_i f_i P_i of
 * "Switch Transformers paper review" (tildalice.io/?p=118) and the Loss-Free
 * update b <- b - gamma sign(F - 1/n) of "MoE travelogue 6" eq. (2), taken on the
 * pooled counts so every rank applies the same update.
 *
 *  totals    [2, n] fp64: the element-wise sum of every rank's moe_balance_totals.
 *  m_total   tokens over all ranks.  has_probs: row 1 holds probability sums.
 *  f, P      [n] out: f_i = count_i / (k m_total), P_i = psum_i / m_total (P only with has_probs).
 *  aux       [1] out (with has_probs): alpha n sum_i f_i P_i.
 *  vio       [3] out or NULL: MaxVio, MinVio, AvgVio of the pooled counts.
 *  bias_inout [n] Loss-Free bias updated in place, or NULL.
 * A count that is not a non-negative integer sets the device error word.
 */
MOE_API moe_status moe_balance_global(const double* totals, int64_t m_total, int32_t n, int32_t k, int32_t has_probs,
                              float alpha, float* f, float* P, float* aux, float* vio, float* bias_inout, float gamma,
                              moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
