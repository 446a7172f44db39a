// api.cu -- the extern "C" entry points declared in include/moe.h: argument
// validation, workspace checks, error reporting, and the kernel launches.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace moe {

cudaError_t launch_router(const void* x, moe_dtype dt, const float* w_r, const float* logits_in, int64_t m, int d,
                          int n, int k, int fn, int renorm, const float* rank_bias, float* probs_out,
                          int32_t* topk_idx, float* topk_gate, void* workspace, cudaStream_t stream);
size_t router_workspace_bytes(int32_t d, int32_t n, moe_dtype dt);
cudaError_t launch_router_split(const float* w_r, int d, int n, void* workspace, cudaStream_t stream);
bool router_uses_tc(moe_dtype dt, const float* logits_in, int n, int k);
cudaError_t launch_capacity(const int32_t* topk_idx, int64_t m, int k, int n, int32_t capacity, int64_t seg_len,
                            int32_t* slot, int32_t* dest_row, int32_t* src_token, int32_t* expert_offsets,
                            int32_t* routed_count, int32_t* kept_count, void* workspace, cudaStream_t stream);
size_t capacity_workspace_bytes(int64_t m, int32_t k, int32_t n, int64_t seg_len);
cudaError_t launch_dispatch(const void* x, moe_dtype dt, int64_t m, int d, const int32_t* src_token,
                            const int32_t* expert_offsets, int n, int64_t max_rows, void* xbuf, cudaStream_t stream);
cudaError_t launch_dispatch_tokens(const void* x, moe_dtype dt, int64_t m, int d, int k, const int32_t* dest_row,
                                   int64_t max_rows, void* xbuf, cudaStream_t stream);
cudaError_t launch_combine(const void* ybuf, moe_dtype dt, const int32_t* dest_row, const float* topk_gate,
                           const void* residual, int64_t m, int k, int d, void* y, cudaStream_t stream);
cudaError_t launch_ffn(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2, const void* b2,
                       const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                       cudaStream_t stream);
cudaError_t launch_ffn_tc_gather(const void* x, const int32_t* src_token, int64_t m, const void* w1, const void* b1,
                                 const void* w2, const void* b2, const int32_t* offsets, int n, int d, int d_ff,
                                 int64_t max_rows, void* ybuf, void* hbuf, cudaStream_t stream);
cudaError_t launch_ffn_tc_combine(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                                  const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* hbuf,
                                  const int32_t* src_token, const int32_t* dest_row, const float* gate,
                                  const void* residual, int64_t m, void* y, cudaStream_t stream);
size_t stats_workspace_bytes(int64_t m, int32_t n, int64_t seg_len);
cudaError_t launch_stats(const float* probs, const int32_t* topk_idx, int64_t m, int n, int k, int64_t seg_len,
                         float alpha, float* f, float* P, float* aux, float* vio, float* bias, float gamma,
                         void* workspace, cudaStream_t stream, double* totals);
cudaError_t launch_stats_global(const double* totals, int64_t m_total, int n, int k, int has_probs, float alpha,
                                float* f, float* P, float* aux, float* vio, float* bias, float gamma,
                                cudaStream_t stream);
size_t balance_workspace_bytes(int64_t m, int32_t n, int32_t k);
cudaError_t launch_loss_grad(const float* probs, int fn, const float* f, int64_t m, int n, int64_t seg_len, float alpha,
                             float w_micro, float w_global, float* dlogits, cudaStream_t stream);
cudaError_t launch_ep_plan(const int32_t* offsets_all, int G, int n, int rank, int32_t* send_base,
                           int32_t* recv_offsets, cudaStream_t stream);
cudaError_t launch_ep_dispatch(const void* x, moe_dtype dt, int64_t m, int d, int k, int n, int G,
                               const int32_t* topk_idx, const int32_t* dest_row, const int32_t* offsets,
                               const int32_t* send_base, void* const* peers, int64_t max_recv_rows, int32_t* ep_row,
                               cudaStream_t stream);
cudaError_t launch_ep_combine(const void* const* peers, moe_dtype dt, const int32_t* ep_row, const int32_t* topk_idx,
                              int n, int G, const float* gate, const void* residual, int64_t m, int k, int d, void* y,
                              cudaStream_t stream);
cudaError_t launch_selftest_wait(const int32_t* flag, int64_t limit_cycles, cudaStream_t stream);
int run_balance_sign_step(const float* s, int64_t m, int n, int k, float* beta, float gamma, int rule,
                          int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream, const char** err);
int run_balance_step_minibatch(const float* s, int64_t m, int n, int k, float* beta, int rule, int64_t seg_len,
                               int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                               const char** err);
int run_balance_assign(const float* s, int64_t m, int n, int k, float* beta, int mode, int rule, int max_iters,
                       int max_repair, int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                       const char** err);
}  // namespace moe

using namespace moe;

static thread_local char g_last_error[512] = "";

static moe_status fail(moe_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

static moe_status check_launch(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    g_last_error[0] = 0;
    return MOE_OK;
}

#define REQUIRE(cond, ...) \
    do { if (!(cond)) return fail(MOE_ERR_INVALID_ARG, __VA_ARGS__); } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

extern "C" {

void moe_last_error(char* buf, size_t len) {
    if (!buf || len == 0) return;
    strncpy(buf, g_last_error, len - 1);
    buf[len - 1] = 0;
}

moe_status moe_sync_status(moe_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
    int code = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&code, g_error, sizeof(int));
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "read device error word: %s", cudaGetErrorString(e));
    if (code != 0) {
        cudaMemcpyToSymbol(g_error, &zero, sizeof(int));
        switch (code) {
            case kErrExpertIndex: return fail(MOE_ERR_INVALID_ARG, "device: expert index outside [0, n)");
            case kErrRowOverflow: return fail(MOE_ERR_INVALID_ARG, "device: more kept rows than max_rows");
            case kErrTokenIndex: return fail(MOE_ERR_INVALID_ARG, "device: src_token outside [0, m)");
            case kErrPipelineTimeout: return fail(MOE_ERR_INTERNAL, "device: a pipeline wait timed out");
            case kErrRepair: return fail(MOE_ERR_INTERNAL, "device: balanced-assignment repair failed");
            case kErrTotals: return fail(MOE_ERR_INVALID_ARG, "device: a routed-count total is not a non-negative integer");
            default: return fail(MOE_ERR_INTERNAL, "device error code %d", code);
        }
    }
    g_last_error[0] = 0;
    return MOE_OK;
}

moe_status moe_selftest_wait(const int32_t* flag, int64_t limit_cycles, moe_stream_t stream) {
    REQUIRE(flag, "flag is required");
    REQUIRE(limit_cycles >= 0 && limit_cycles <= 4000000000LL, "limit_cycles must be in [0, 4e9]");
    return check_launch(launch_selftest_wait(flag, limit_cycles, stream), "moe_selftest_wait");
}

size_t moe_router_topk_workspace_size(int32_t d, int32_t n, int32_t k, moe_dtype x_dtype) {
    return router_uses_tc(x_dtype, nullptr, n, k) ? router_workspace_bytes(d, n, x_dtype) : 0;
}

moe_status moe_router_topk(const void* x, moe_dtype x_dtype, const float* w_r, const float* logits_in, int64_t m,
                           int32_t d, int32_t n, int32_t k, moe_score_fn fn, int32_t renorm_topk,
                           const float* rank_bias, float* probs_out, int32_t* topk_idx, float* topk_gate,
                           void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 0, "m must be >= 0");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31) && m * (int64_t)n < ((int64_t)1 << 40), "m too large");
    REQUIRE(fn == MOE_SOFTMAX || fn == MOE_SIGMOID, "unknown score function");
    REQUIRE(x_dtype == MOE_F32 || x_dtype == MOE_BF16, "unknown dtype");
    REQUIRE(m == 0 || (topk_idx && topk_gate), "topk_idx and topk_gate are required");
    if (!logits_in) {
        REQUIRE(m == 0 || x, "x is required when logits_in is NULL");
        REQUIRE(m == 0 || w_r || router_uses_tc(x_dtype, logits_in, n, k),
                "w_r may be NULL only on the tensor-core path (bf16 x, n <= 128), with a workspace prepared by "
                "moe_router_prepare");
        REQUIRE(d >= 1, "d must be >= 1");
        REQUIRE(x_dtype != MOE_BF16 || d % 8 == 0, "d must be a multiple of 8 for bf16 x");
        REQUIRE(x_dtype != MOE_BF16 || m == 0 || aligned16(x), "bf16 x must be 16-byte aligned");
    }
    REQUIRE(!probs_out || aligned16(probs_out), "probs_out must be 16-byte aligned");
    if (router_uses_tc(x_dtype, logits_in, n, k) && m > 0) {
        const size_t need = router_workspace_bytes(d, n, x_dtype);
        if (ws_bytes < need || !workspace || !aligned16(workspace))
            return fail(MOE_ERR_WORKSPACE, "moe_router_topk: 16-byte aligned workspace of %zu bytes required", need);
    }
    return check_launch(launch_router(x, x_dtype, w_r, logits_in, m, d, n, k, (int)fn, renorm_topk, rank_bias,
                                      probs_out, topk_idx, topk_gate, workspace, stream),
                        "moe_router_topk");
}

moe_status moe_router_prepare(const float* w_r, int32_t d, int32_t n, int32_t k, moe_dtype x_dtype, void* workspace,
                              size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(d >= 1, "d must be >= 1");
    REQUIRE(x_dtype == MOE_F32 || x_dtype == MOE_BF16, "unknown dtype");
    REQUIRE(w_r, "w_r is required");
    if (!router_uses_tc(x_dtype, nullptr, n, k))
        return fail(MOE_ERR_UNSUPPORTED, "moe_router_prepare: this shape takes the fp32 FMA router, which reads w_r "
                                         "directly; pass w_r to moe_router_topk");
    REQUIRE(d % 8 == 0, "d must be a multiple of 8 for bf16 x");
    const size_t need = router_workspace_bytes(d, n, x_dtype);
    if (ws_bytes < need || !workspace || !aligned16(workspace))
        return fail(MOE_ERR_WORKSPACE, "moe_router_prepare: 16-byte aligned workspace of %zu bytes required", need);
    return check_launch(launch_router_split(w_r, d, n, workspace, stream), "moe_router_prepare");
}

size_t moe_capacity_slots_workspace_size(int64_t m, int32_t k, int32_t n, int64_t seg_len) {
    return capacity_workspace_bytes(m, k, n, seg_len);
}

}  // extern "C"

// Argument checks of the capacity stage, shared by moe_capacity_slots and moe_capacity_slots_static.
static moe_status capacity_args_ok(const int32_t* topk_idx, int64_t m, int32_t k, int32_t n, int32_t capacity,
                                   int64_t seg_len, const int32_t* slot, const int32_t* dest_row,
                                   const int32_t* src_token, const int32_t* expert_offsets,
                                   const int32_t* routed_count, const int32_t* kept_count) {
    REQUIRE(m >= 0, "m must be >= 0");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31), "m * k must be < 2^31");
    REQUIRE(capacity >= 0, "capacity must be >= 0");
    REQUIRE(seg_len >= 1 && m % seg_len == 0, "seg_len must be >= 1 and divide m");
    REQUIRE(expert_offsets && routed_count && kept_count, "output pointers are required");
    REQUIRE(m == 0 || (topk_idx && slot && dest_row && src_token), "array pointers are required");
    return MOE_OK;
}

extern "C" {

moe_status moe_capacity_slots(const int32_t* topk_idx, int64_t m, int32_t k, int32_t n, int32_t capacity,
                              int64_t seg_len, int32_t* slot, int32_t* dest_row, int32_t* src_token,
                              int32_t* expert_offsets, int32_t* routed_count, int32_t* kept_count, void* workspace,
                              size_t ws_bytes, moe_stream_t stream) {
    const moe_status st = capacity_args_ok(topk_idx, m, k, n, capacity, seg_len, slot, dest_row, src_token,
                                           expert_offsets, routed_count, kept_count);
    if (st != MOE_OK) return st;
    const size_t need = capacity_workspace_bytes(m, k, n, seg_len);
    if (ws_bytes < need || (need && !workspace))
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    return check_launch(launch_capacity(topk_idx, m, k, n, capacity, seg_len, slot, dest_row, src_token,
                                        expert_offsets, routed_count, kept_count, workspace, stream),
                        "moe_capacity_slots");
}

moe_status moe_dispatch(const void* x, moe_dtype dt, int64_t m, int32_t d, const int32_t* src_token,
                        const int32_t* expert_offsets, int32_t n, int64_t max_rows, void* xbuf, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(m >= 0 && max_rows >= 0 && max_rows < ((int64_t)1 << 31), "bad m or max_rows");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(d >= 1 && (d * (dt == MOE_BF16 ? 2 : 4)) % 16 == 0, "d must be a multiple of %d", dt == MOE_BF16 ? 8 : 4);
    REQUIRE(expert_offsets, "expert_offsets is required");
    REQUIRE(max_rows == 0 || (x && src_token && xbuf), "array pointers are required");
    REQUIRE(max_rows == 0 || (aligned16(x) && aligned16(xbuf)), "x and xbuf must be 16-byte aligned");
    return check_launch(launch_dispatch(x, dt, m, d, src_token, expert_offsets, n, max_rows, xbuf, stream),
                        "moe_dispatch");
}

moe_status moe_dispatch_tokens(const void* x, moe_dtype dt, int64_t m, int32_t d, int32_t k, const int32_t* dest_row,
                               int64_t max_rows, void* xbuf, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(m >= 0 && max_rows >= 0 && max_rows < ((int64_t)1 << 31), "bad m or max_rows");
    REQUIRE(k >= 1 && k <= kMaxExperts && m * (int64_t)k < ((int64_t)1 << 31), "bad k");
    REQUIRE(d >= 1 && (d * (dt == MOE_BF16 ? 2 : 4)) % 16 == 0, "d must be a multiple of %d", dt == MOE_BF16 ? 8 : 4);
    REQUIRE(m == 0 || (x && dest_row && xbuf), "array pointers are required");
    REQUIRE(m == 0 || (aligned16(x) && aligned16(xbuf)), "x and xbuf must be 16-byte aligned");
    return check_launch(launch_dispatch_tokens(x, dt, m, d, k, dest_row, max_rows, xbuf, stream),
                        "moe_dispatch_tokens");
}

size_t moe_expert_ffn_workspace_size(moe_dtype dt, int64_t max_rows, int32_t d_ff) {
    // hidden activations [max_rows, d_ff], then (bf16) one int32 completion counter per expert
    const size_t esz = dt == MOE_BF16 ? 2 : 4;
    return esz * (size_t)(max_rows < 0 ? 0 : max_rows) * (size_t)(d_ff < 0 ? 0 : d_ff) + 2048;
}

moe_status moe_expert_ffn(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                          const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d, int32_t d_ff,
                          int64_t max_rows, void* ybuf, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(max_rows >= 0 && max_rows < ((int64_t)1 << 31), "bad max_rows");
    REQUIRE(d >= 8 && d % 8 == 0, "d must be a positive multiple of 8");
    REQUIRE(d_ff >= 8 && d_ff % 8 == 0, "d_ff must be a positive multiple of 8");
    REQUIRE(expert_offsets && w1 && b1 && w2 && b2, "weights, biases and expert_offsets are required");
    REQUIRE(max_rows == 0 || (xbuf && ybuf), "xbuf and ybuf are required");
    REQUIRE(aligned16(xbuf) && aligned16(ybuf) && aligned16(w1) && aligned16(w2) && aligned16(workspace),
            "xbuf, ybuf, w1, w2 and the workspace must be 16-byte aligned");
    const size_t need = moe_expert_ffn_workspace_size(dt, max_rows, d_ff);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    if (max_rows == 0) return MOE_OK;
    return check_launch(launch_ffn(xbuf, dt, w1, b1, w2, b2, expert_offsets, n, d, d_ff, max_rows, ybuf, workspace,
                                   stream),
                        "moe_expert_ffn");
}

moe_status moe_expert_ffn_gather(const void* x, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                                 const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d, int32_t d_ff,
                                 int64_t max_rows, const int32_t* src_token, int64_t m, void* ybuf, void* workspace,
                                 size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    if (dt != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_expert_ffn_gather: bf16 only (use moe_dispatch + moe_expert_ffn)");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(max_rows >= 0 && max_rows < ((int64_t)1 << 31), "bad max_rows");
    REQUIRE(m >= 0 && m < ((int64_t)1 << 31), "bad m");
    REQUIRE(d >= 8 && d % 8 == 0, "d must be a positive multiple of 8");
    REQUIRE(d_ff >= 8 && d_ff % 8 == 0, "d_ff must be a positive multiple of 8");
    REQUIRE(expert_offsets && w1 && b1 && w2 && b2, "weights, biases and expert_offsets are required");
    REQUIRE(max_rows == 0 || (x && ybuf && src_token && m > 0), "x, src_token and ybuf are required");
    REQUIRE(aligned16(x) && aligned16(ybuf) && aligned16(w1) && aligned16(w2) && aligned16(workspace),
            "x, ybuf, w1, w2 and the workspace must be 16-byte aligned");
    const size_t need = moe_expert_ffn_workspace_size(dt, max_rows, d_ff);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    if (max_rows == 0) return MOE_OK;
    return check_launch(launch_ffn_tc_gather(x, src_token, m, w1, b1, w2, b2, expert_offsets, n, d, d_ff, max_rows,
                                             ybuf, workspace, stream),
                        "moe_expert_ffn_gather");
}

moe_status moe_expert_ffn_combine(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                                  const void* b2, const int32_t* expert_offsets, int32_t n, int32_t d, int32_t d_ff,
                                  int64_t max_rows, const int32_t* src_token, const int32_t* dest_row,
                                  const float* topk_gate, const void* residual, int64_t m, void* y, void* workspace,
                                  size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    if (dt != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_expert_ffn_combine: bf16 only (use moe_expert_ffn + moe_combine)");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(max_rows >= 0 && max_rows < ((int64_t)1 << 31), "bad max_rows");
    REQUIRE(m >= 0 && max_rows <= m, "one pick per token: max_rows must be <= m");
    REQUIRE(d >= 8 && d % 8 == 0, "d must be a positive multiple of 8");
    REQUIRE(d_ff >= 8 && d_ff % 8 == 0, "d_ff must be a positive multiple of 8");
    REQUIRE(expert_offsets && w1 && b1 && w2 && b2, "weights, biases and expert_offsets are required");
    REQUIRE(m == 0 || (y && dest_row && topk_gate && src_token), "y, src_token, dest_row and topk_gate are required");
    REQUIRE(max_rows == 0 || xbuf, "xbuf is required");
    REQUIRE(aligned16(xbuf) && aligned16(y) && aligned16(residual) && aligned16(w1) && aligned16(w2) &&
                aligned16(workspace),
            "xbuf, y, residual, w1, w2 and the workspace must be 16-byte aligned");
    REQUIRE(residual == nullptr || residual != y, "residual must not alias y");
    const size_t need = moe_expert_ffn_workspace_size(dt, max_rows, d_ff);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    if (m == 0) return MOE_OK;
    return check_launch(launch_ffn_tc_combine(xbuf, w1, b1, w2, b2, expert_offsets, n, d, d_ff, max_rows, workspace,
                                              src_token, dest_row, topk_gate, residual, m, y, stream),
                        "moe_expert_ffn_combine");
}

moe_status moe_combine(const void* ybuf, moe_dtype dt, const int32_t* dest_row, const float* topk_gate,
                       const void* residual, int64_t m, int32_t k, int32_t d, void* y, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(m >= 0 && k >= 1 && k <= kMaxExperts, "bad m or k");
    REQUIRE(d >= 1 && (d * (dt == MOE_BF16 ? 2 : 4)) % 16 == 0, "d must be a multiple of %d", dt == MOE_BF16 ? 8 : 4);
    REQUIRE(m == 0 || (ybuf && dest_row && topk_gate && y), "array pointers are required");
    REQUIRE(aligned16(ybuf) && aligned16(y) && aligned16(residual), "ybuf, y and residual must be 16-byte aligned");
    REQUIRE(residual == nullptr || residual != y, "residual must not alias y");
    return check_launch(launch_combine(ybuf, dt, dest_row, topk_gate, residual, m, k, d, y, stream), "moe_combine");
}

size_t moe_balance_stats_workspace_size(int64_t m, int32_t n, int64_t seg_len) {
    return stats_workspace_bytes(m, n, seg_len);
}

moe_status moe_balance_stats(const float* probs, const int32_t* topk_idx, int64_t m, int32_t n, int32_t k,
                             int64_t seg_len, float alpha, float* f, float* P, float* aux, float* vio,
                             float* bias_inout, float gamma, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 1, "m must be >= 1");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31), "m * k must be < 2^31");
    REQUIRE(seg_len >= 1 && m % seg_len == 0, "seg_len must be >= 1 and divide m");
    REQUIRE(topk_idx && f, "topk_idx and f are required");
    REQUIRE(!probs || (P && aux), "P and aux are required when probs is given");
    const size_t need = stats_workspace_bytes(m, n, seg_len);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    return check_launch(launch_stats(probs, topk_idx, m, n, k, seg_len, alpha, f, P, aux, vio, bias_inout, gamma,
                                     workspace, stream, nullptr),
                        "moe_balance_stats");
}

moe_status moe_balance_loss_grad(const float* probs, moe_score_fn fn, const float* f, int64_t m, int32_t n,
                                 int64_t seg_len, float alpha, float w_micro, float w_global, float* dlogits,
                                 moe_stream_t stream) {
    REQUIRE(m >= 0, "m must be >= 0");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(fn == MOE_SOFTMAX || fn == MOE_SIGMOID, "unknown score function");
    REQUIRE(seg_len >= 1 && m % seg_len == 0, "seg_len must be >= 1 and divide m");
    REQUIRE(m == 0 || (probs && f && dlogits), "probs, f and dlogits are required");
    return check_launch(launch_loss_grad(probs, (int)fn, f, m, n, seg_len, alpha, w_micro, w_global, dlogits, stream),
                        "moe_balance_loss_grad");
}

size_t moe_balance_totals_workspace_size(int64_t m, int32_t n) { return stats_workspace_bytes(m, n, m); }

moe_status moe_balance_totals(const float* probs, const int32_t* topk_idx, int64_t m, int32_t n, int32_t k,
                              double* totals, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 1, "m must be >= 1");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31), "m * k must be < 2^31");
    REQUIRE(topk_idx && totals, "topk_idx and totals are required");
    const size_t need = stats_workspace_bytes(m, n, m);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    return check_launch(launch_stats(probs, topk_idx, m, n, k, m, 0.f, nullptr, nullptr, nullptr, nullptr, nullptr,
                                     0.f, workspace, stream, totals),
                        "moe_balance_totals");
}

moe_status moe_balance_global(const double* totals, int64_t m_total, int32_t n, int32_t k, int32_t has_probs,
                              float alpha, float* f, float* P, float* aux, float* vio, float* bias_inout, float gamma,
                              moe_stream_t stream) {
    REQUIRE(m_total >= 1, "m_total must be >= 1");
    REQUIRE(n >= 1 && n <= kMaxExperts, "n must be in [1, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k <= n, "k must be in [1, n]");
    REQUIRE(totals && f, "totals and f are required");
    REQUIRE(!has_probs || (P && aux), "P and aux are required when has_probs is set");
    return check_launch(launch_stats_global(totals, m_total, n, k, has_probs ? 1 : 0, alpha, f, P, aux, vio,
                                            bias_inout, gamma, stream),
                        "moe_balance_global");
}

moe_status moe_balance_sign_step(const float* s, int64_t m, int32_t n, int32_t k, float* beta, float gamma,
                                 moe_qb_threshold rule, int32_t* topk_idx, int32_t* info, void* workspace,
                                 size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 1, "m must be >= 1");
    REQUIRE(n >= 2 && n <= kMaxExperts, "n must be in [2, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k < n, "k must be in [1, n - 1]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31) && m * (int64_t)n < ((int64_t)1 << 34), "m too large");
    REQUIRE((m * k) % n == 0, "m * k must be divisible by n (every expert gets exactly m k / n tokens)");
    REQUIRE(rule == MOE_QB_MIDPOINT || rule == MOE_QB_BOUNDARY || rule == MOE_QB_BIP, "unknown threshold rule");
    REQUIRE(gamma >= 0.f && gamma == gamma, "gamma must be a non-negative number");
    REQUIRE(s && beta && topk_idx && info, "s, beta, topk_idx and info are required");
    const size_t need = balance_workspace_bytes(m, n, k);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    const char* err = "";
    const int rc = run_balance_sign_step(s, m, n, k, beta, gamma, rule, topk_idx, info, workspace, stream, &err);
    if (rc != MOE_OK) return fail((moe_status)rc, "moe_balance_sign_step: %s", err);
    return MOE_OK;
}

moe_status moe_balance_step_minibatch(const float* s, int64_t m, int32_t n, int32_t k, float* beta,
                                      moe_qb_threshold rule, int64_t seg_len, int32_t* topk_idx, int32_t* info,
                                      void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 1, "m must be >= 1");
    REQUIRE(n >= 2 && n <= kMaxExperts, "n must be in [2, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k < n, "k must be in [1, n - 1]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31) && m * (int64_t)n < ((int64_t)1 << 34), "m too large");
    REQUIRE(seg_len >= 1 && m % seg_len == 0, "seg_len must be >= 1 and divide m");
    REQUIRE((seg_len * k) % n == 0, "seg_len * k must be divisible by n (each mini-batch's column count)");
    REQUIRE(m / seg_len <= 4096, "at most 4096 mini-batches");
    REQUIRE(rule == MOE_QB_MIDPOINT || rule == MOE_QB_BOUNDARY || rule == MOE_QB_BIP, "unknown threshold rule");
    REQUIRE(s && beta && topk_idx && info, "s, beta, topk_idx and info are required");
    const size_t need = balance_workspace_bytes(m, n, k);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    const char* err = "";
    const int rc = run_balance_step_minibatch(s, m, n, k, beta, rule, seg_len, topk_idx, info, workspace, stream, &err);
    if (rc != MOE_OK) return fail((moe_status)rc, "moe_balance_step_minibatch: %s", err);
    g_last_error[0] = 0;
    return MOE_OK;
}

moe_status moe_ep_plan(const int32_t* offsets_all, int32_t G, int32_t n, int32_t rank, int32_t* send_base,
                       int32_t* recv_offsets, moe_stream_t stream) {
    REQUIRE(G >= 1 && n >= 1 && n <= kMaxExperts && n % G == 0, "n must be in [1, %d] and divisible by G",
            kMaxExperts);
    REQUIRE(rank >= 0 && rank < G, "rank must be in [0, G)");
    REQUIRE(offsets_all && send_base && recv_offsets, "offsets_all, send_base and recv_offsets are required");
    return check_launch(launch_ep_plan(offsets_all, G, n, rank, send_base, recv_offsets, stream), "moe_ep_plan");
}

moe_status moe_ep_dispatch(const void* x, moe_dtype dt, int64_t m, int32_t d, int32_t k, int32_t n, int32_t G,
                           const int32_t* topk_idx, const int32_t* dest_row, const int32_t* expert_offsets,
                           const int32_t* send_base, void* const* peer_xrecv, int64_t max_recv_rows, int32_t* ep_row,
                           moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(m >= 0 && max_recv_rows >= 0 && max_recv_rows < ((int64_t)1 << 31), "bad m or max_recv_rows");
    REQUIRE(G >= 1 && n >= 1 && n <= kMaxExperts && n % G == 0, "n must be in [1, %d] and divisible by G",
            kMaxExperts);
    REQUIRE(k >= 1 && k <= n && m * (int64_t)k < ((int64_t)1 << 31), "bad k");
    REQUIRE(d >= 1 && (d * (dt == MOE_BF16 ? 2 : 4)) % 16 == 0, "d must be a multiple of %d", dt == MOE_BF16 ? 8 : 4);
    REQUIRE(m == 0 || (x && topk_idx && dest_row && expert_offsets && send_base && peer_xrecv && ep_row),
            "array pointers are required");
    REQUIRE(m == 0 || aligned16(x), "x must be 16-byte aligned");
    return check_launch(launch_ep_dispatch(x, dt, m, d, k, n, G, topk_idx, dest_row, expert_offsets, send_base,
                                           peer_xrecv, max_recv_rows, ep_row, stream),
                        "moe_ep_dispatch");
}

moe_status moe_ep_combine(const void* const* peer_yrecv, moe_dtype dt, const int32_t* ep_row, const int32_t* topk_idx,
                          int32_t n, int32_t G, const float* topk_gate, const void* residual, int64_t m, int32_t k,
                          int32_t d, void* y, moe_stream_t stream) {
    REQUIRE(dt == MOE_F32 || dt == MOE_BF16, "unknown dtype");
    REQUIRE(m >= 0 && k >= 1 && k <= kMaxExperts, "bad m or k");
    REQUIRE(G >= 1 && n >= 1 && n <= kMaxExperts && n % G == 0, "n must be in [1, %d] and divisible by G",
            kMaxExperts);
    REQUIRE(d >= 1 && (d * (dt == MOE_BF16 ? 2 : 4)) % 16 == 0, "d must be a multiple of %d", dt == MOE_BF16 ? 8 : 4);
    REQUIRE(m == 0 || (peer_yrecv && ep_row && topk_idx && topk_gate && y), "array pointers are required");
    REQUIRE(aligned16(y) && aligned16(residual), "y and residual must be 16-byte aligned");
    REQUIRE(residual == nullptr || residual != y, "residual must not alias y");
    return check_launch(launch_ep_combine(peer_yrecv, dt, ep_row, topk_idx, n, G, topk_gate, residual, m, k, d, y,
                                          stream),
                        "moe_ep_combine");
}

size_t moe_balance_assign_workspace_size(int64_t m, int32_t n, int32_t k, moe_qb_mode mode) {
    (void)mode;
    if (m < 1 || n < 1 || n > kMaxExperts || k < 1) return 0;
    return balance_workspace_bytes(m, n, k);
}

moe_status moe_balance_assign(const float* s, int64_t m, int32_t n, int32_t k, float* beta, moe_qb_mode mode,
                              moe_qb_threshold rule, int32_t max_iters, int32_t max_repair, int32_t* topk_idx,
                              int32_t* info, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    REQUIRE(m >= 1, "m must be >= 1");
    REQUIRE(n >= 2 && n <= kMaxExperts, "n must be in [2, %d]", kMaxExperts);
    REQUIRE(k >= 1 && k < n, "k must be in [1, n - 1]");
    REQUIRE(m * (int64_t)k < ((int64_t)1 << 31) && m * (int64_t)n < ((int64_t)1 << 34), "m too large");
    REQUIRE((m * k) % n == 0, "m * k must be divisible by n (every expert gets exactly m k / n tokens)");
    REQUIRE(mode == MOE_QB_STEP || mode == MOE_QB_SOLVE, "unknown mode");
    REQUIRE(rule == MOE_QB_MIDPOINT || rule == MOE_QB_BOUNDARY || rule == MOE_QB_BIP, "unknown threshold rule");
    REQUIRE(max_iters >= 0 && max_repair >= 0, "max_iters and max_repair must be >= 0");
    REQUIRE(s && beta && topk_idx && info, "s, beta, topk_idx and info are required");
    const size_t need = balance_workspace_bytes(m, n, k);
    if (ws_bytes < need || !workspace) return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes required", need);
    const char* err = nullptr;
    const int st = run_balance_assign(s, m, n, k, beta, (int)mode, (int)rule, max_iters, max_repair, topk_idx, info,
                                      workspace, stream, &err);
    if (st != MOE_OK) return fail((moe_status)st, "moe_balance_assign: %s", err ? err : "failed");
    g_last_error[0] = 0;
    return MOE_OK;
}

}  // extern "C"
