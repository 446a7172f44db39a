// balance.cu -- optimal-assignment balancing (Quantile Balancing) and its exact finish.
//
// MoE travelogue 6: optimal assignment promotes balance (kexue.fm/archives/11619):
// the balance LP (3)/(4), its dual (8), the alternating updates
//   alpha_i = threshold between the k-th and (k+1)-th largest of s_i - beta,
//   beta_j  = threshold between the C-th and (C+1)-th largest of s_:j - alpha,
// the QB algorithm box and its one-step practical form (select with the old
// beta, then update). Both thresholds are computed in fp32 exactly as defined
// (v = fp32(s - beta), u = fp32(s - alpha), midpoint fp32(fp32(a + b) * 0.5)),
// so every decision is reproducible bit for bit.
//
// Kernels:
//   qb_row     one warp per token: v = s_i - beta in registers (n/32 values per
//              lane), k + 1 rounds of a warp arg-max give the top-k set, the
//              k-th and (k+1)-th values (alpha) and a tie flag; the set is
//              written in ascending expert order and counted per expert.
//   transpose  s [m, n] -> sT [n, m] once per call, so each column is contiguous.
//   qb_col     one CTA per expert column: exact radix select (four 8-bit
//              digit passes over order-preserving uint32 keys of u) for the
//              C-th largest, then the (C+1)-th from the tie count or one max
//              pass.
//   repair     successive shortest paths on the n-expert graph (exact finish
//              when the QB iterate is not yet balanced): arc a -> b costs
//              W[a][b] = min over tokens i holding a but not b of s_ia - s_ib
//              (fp64, lowest token on ties); one CTA runs Jacobi Bellman-Ford
//              rounds from the over-full experts, picks the nearest under-full
//              expert (lowest index on ties) and moves each arc's argmin
//              token. The number of moves equals the excess, so the host
//              enqueues exactly that many rounds without waiting in between.
#include "common.cuh"

namespace moe {

cudaError_t launch_capacity(const int32_t* topk_idx, int64_t m, int k, int n, int32_t capacity, int64_t seg_len,
                            int32_t* slot, int32_t* dest_row, int32_t* src_token, int32_t* expert_offsets,
                            int32_t* routed_count, int32_t* kept_count, void* workspace, cudaStream_t stream);
size_t capacity_workspace_bytes(int64_t m, int32_t k, int32_t n, int64_t seg_len);

namespace qb {
constexpr int kRowThreads = 256;
constexpr int kColThreads = 512;
constexpr int kRepairThreads = 256;
// status words kept in the workspace
enum { kStDone = 0, kStAugments = 1, kStError = 2, kStTies = 3, kStWords = 8 };
}  // namespace qb

__device__ __forceinline__ float qb_threshold(float a, float b, int rule) {
    return rule == MOE_QB_BOUNDARY ? b : __fmul_rn(__fadd_rn(a, b), 0.5f);
}

// order-preserving key: larger float -> larger key; -0 is folded onto +0
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t b = __float_as_uint(f);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int NT>
__global__ void __launch_bounds__(qb::kRowThreads)
qb_row_kernel(const float* __restrict__ s, int64_t m, int n, int k, const float* __restrict__ beta, int rule,
              float* __restrict__ alpha, int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts,
              int32_t* __restrict__ status) {
    __shared__ float sb[kMaxExperts];
    __shared__ int cnt[kMaxExperts];
    __shared__ int nties;
    const int tid = threadIdx.x, lane = tid & 31;
    for (int j = tid; j < n; j += blockDim.x) { sb[j] = beta[j]; cnt[j] = 0; }
    if (tid == 0) nties = 0;
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    const int64_t warps = (int64_t)gridDim.x * (qb::kRowThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (qb::kRowThreads / 32) + (tid >> 5); i < m; i += warps) {
        float v[NT];
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const int j = lane + 32 * q;
            v[q] = j < n ? __fsub_rn(s[i * n + j], sb[j]) : -INFINITY;
        }
        uint32_t taken = 0;
        float vk = 0.f, vk1 = 0.f;
        for (int r = 0; r <= k; ++r) {
            float bk = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const int j = lane + 32 * q;
                if (j < n && !(taken & (1u << q)) && ranks_before(v[q], j, bk, bi)) { bk = v[q]; bi = j; }
            }
            warp_best(bk, bi);
            if (r < k && bi < n && lane == (bi & 31)) taken |= 1u << (bi >> 5);
            if (r == k - 1) vk = bk;
            if (r == k) vk1 = bk;
        }
        if (lane == 0) {
            alpha[i] = qb_threshold(vk, vk1, rule);
            if (vk == vk1) atomicAdd(&nties, 1);
        }
        int pos = 0;
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const bool bit = (taken >> q) & 1u;
            const uint32_t mask = __ballot_sync(0xffffffffu, bit);
            if (bit) {
                topk_idx[i * k + pos + __popc(mask & lt)] = lane + 32 * q;
                atomicAdd(&cnt[lane + 32 * q], 1);
            }
            pos += __popc(mask);
        }
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
    if (tid == 0 && nties) atomicAdd(&status[qb::kStTies], nties);
}

__global__ void transpose_kernel(const float* __restrict__ s, int64_t m, int n, float* __restrict__ sT) {
    __shared__ float tile[32][33];
    const int64_t i0 = (int64_t)blockIdx.x * 32;
    const int j0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int64_t i = i0 + r;
        const int j = j0 + tx;
        tile[r][tx] = (i < m && j < n) ? s[i * n + j] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int j = j0 + r;
        const int64_t i = i0 + tx;
        if (j < n && i < m) sT[(int64_t)j * m + i] = tile[tx][r];
    }
}

__global__ void __launch_bounds__(qb::kColThreads)
qb_col_kernel(const float* __restrict__ sT, int64_t m, int n, int64_t C, const float* __restrict__ alpha, int rule,
              float* __restrict__ beta) {
    __shared__ unsigned hist[256];
    __shared__ uint32_t s_prefix, s_mask;
    __shared__ int64_t s_want, s_eq;
    __shared__ uint32_t s_max;
    const int tid = threadIdx.x;
    const int j = blockIdx.x;
    const float* col = sT + (int64_t)j * m;
    if (tid == 0) { s_prefix = 0; s_mask = 0; s_want = C; s_eq = 0; s_max = 0; }
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int b = tid; b < 256; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        const uint32_t prefix = s_prefix, mask = s_mask;
        for (int64_t i = tid; i < m; i += blockDim.x) {
            const uint32_t key = float_key(__fsub_rn(col[i], alpha[i]));
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            int64_t cum = 0, want = s_want;
            int sel = 0;
            for (int dg = 255; dg >= 0; --dg) {
                const int64_t h = hist[dg];
                if (cum + h >= want) { sel = dg; break; }
                cum += h;
            }
            s_want = want - cum;
            s_prefix = prefix | ((uint32_t)sel << shift);
            s_mask = mask | (255u << shift);
            s_eq = hist[sel];
        }
        __syncthreads();
    }
    const uint32_t akey = s_prefix;
    const int64_t greater = C - s_want;
    float b;
    if (greater + s_eq >= C + 1) {
        b = key_float(akey);
    } else {
        uint32_t best = 0;
        for (int64_t i = tid; i < m; i += blockDim.x) {
            const uint32_t key = float_key(__fsub_rn(col[i], alpha[i]));
            if (key < akey && key > best) best = key;
        }
        atomicMax(&s_max, best);
        __syncthreads();
        b = key_float(s_max);
    }
    if (tid == 0) beta[j] = qb_threshold(key_float(akey), b, rule);
}

// Arc costs of the expert graph: CTA a scans the tokens holding expert a (token order).
__global__ void __launch_bounds__(qb::kRepairThreads)
qb_arc_kernel(const float* __restrict__ s, int n, int k, const int32_t* __restrict__ topk_idx,
              const int32_t* __restrict__ src_token, const int32_t* __restrict__ offsets, double* __restrict__ W,
              int32_t* __restrict__ A, const int32_t* __restrict__ status) {
    if (status[qb::kStError] || status[qb::kStDone]) return;
    const int a = blockIdx.x, b = threadIdx.x;
    double best = INFINITY;
    int32_t arg = -1;
    for (int32_t p = offsets[a]; p < offsets[a + 1]; ++p) {
        const int64_t i = src_token[p];
        bool in = false;
        for (int r = 0; r < k; ++r) in |= (topk_idx[i * k + r] == b);
        if (b < n && !in) {
            const double c = (double)s[i * n + a] - (double)s[i * n + b];
            if (c < best) { best = c; arg = (int32_t)i; }
        }
    }
    if (b < n) { W[(int64_t)a * n + b] = best; A[(int64_t)a * n + b] = arg; }
}

// One augmentation: shortest path from the over-full experts to the nearest under-full one.
__global__ void __launch_bounds__(qb::kRepairThreads)
qb_repair_step_kernel(int n, int64_t C, int k, const double* __restrict__ W, const int32_t* __restrict__ A,
                      int32_t* __restrict__ counts, int32_t* __restrict__ topk_idx, int32_t* __restrict__ status) {
    __shared__ double dist[kMaxExperts], nd[kMaxExperts];
    __shared__ int pred[kMaxExperts];
    __shared__ int any_over, changed;
    const int b = threadIdx.x;
    if (status[qb::kStError] || status[qb::kStDone]) return;
    if (b == 0) any_over = 0;
    __syncthreads();
    if (b < n) {
        const bool over = counts[b] > C;
        dist[b] = over ? 0.0 : INFINITY;
        if (over) atomicOr(&any_over, 1);
    }
    __syncthreads();
    if (!any_over) {
        if (b == 0) status[qb::kStDone] = 1;
        return;
    }
    bool settled = false;
    for (int round = 0; round <= n; ++round) {
        if (b == 0) changed = 0;
        __syncthreads();
        if (b < n) {
            double best = dist[b];
            for (int a = 0; a < n; ++a) {
                const double w = W[(int64_t)a * n + b];
                if (a == b || dist[a] == INFINITY || w == INFINITY) continue;
                const double c = dist[a] + w;
                if (c < best) best = c;
            }
            nd[b] = best;
            if (best != dist[b]) changed = 1;
        }
        __syncthreads();
        if (b < n) dist[b] = nd[b];
        const int ch = changed;
        __syncthreads();
        if (!ch) { settled = true; break; }
    }
    if (!settled) {
        if (b == 0) { status[qb::kStError] = 1; record_error(kErrRepair); }
        return;
    }
    if (b < n) {
        int p = -1;
        if (dist[b] != INFINITY) {
            for (int a = 0; a < n; ++a) {
                const double w = W[(int64_t)a * n + b];
                if (a == b || dist[a] == INFINITY || w == INFINITY) continue;
                if (dist[a] + w == dist[b]) { p = a; break; }
            }
        }
        pred[b] = p;
    }
    __syncthreads();
    if (b == 0) {
        int t = -1;
        for (int e = 0; e < n; ++e)
            if (counts[e] < C && dist[e] != INFINITY && (t < 0 || dist[e] < dist[t])) t = e;
        bool ok = t >= 0;
        int node = t, len = 0;
        int path[kMaxExperts + 1];
        if (ok) {
            path[len++] = node;
            while (pred[node] >= 0 && len <= n) { node = pred[node]; path[len++] = node; }
            ok = len <= n && counts[node] > C;
        }
        for (int p = len - 1; ok && p > 0; --p) {
            const int a = path[p], bb = path[p - 1];
            const int32_t i = A[(int64_t)a * n + bb];
            if (i < 0) { ok = false; break; }
            int32_t* row = topk_idx + (int64_t)i * k;
            int pa = -1;
            bool hasb = false;
            for (int r = 0; r < k; ++r) { if (row[r] == a) pa = r; if (row[r] == bb) hasb = true; }
            if (pa < 0 || hasb) { ok = false; break; }
            // replace a by bb and restore ascending order
            int r = pa;
            row[r] = bb;
            while (r > 0 && row[r - 1] > row[r]) { const int t2 = row[r - 1]; row[r - 1] = row[r]; row[r] = t2; --r; }
            while (r + 1 < k && row[r + 1] < row[r]) { const int t2 = row[r + 1]; row[r + 1] = row[r]; row[r] = t2; ++r; }
        }
        if (!ok) {
            status[qb::kStError] = 1;
            record_error(kErrRepair);
        } else {
            counts[node] -= 1;
            counts[t] += 1;
            status[qb::kStAugments] += 1;
        }
    }
}

__global__ void qb_info_kernel(const int32_t* __restrict__ counts, int n, int64_t C, const int32_t* __restrict__ status,
                               int32_t iters, int32_t* __restrict__ info) {
    if (threadIdx.x != 0) return;
    int64_t excess = 0;
    for (int e = 0; e < n; ++e) if (counts[e] > C) excess += counts[e] - C;
    info[0] = iters;
    info[1] = status[qb::kStAugments];
    info[2] = (int32_t)excess;
    info[3] = status[qb::kStTies];
}

struct QBWorkspace {
    float* sT;
    float* alpha;
    int32_t* counts;
    int32_t* status;
    double* W;
    int32_t* A;
    int32_t *slot, *dest, *src, *offsets, *routed, *kept;
    void* cap_ws;
};

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

static size_t qb_layout(int64_t m, int n, int k, QBWorkspace* w, char* base) {
    size_t off = 0;
    auto take = [&](size_t bytes) { char* p = base ? base + off : nullptr; off += align256(bytes); return p; };
    char* p;
    p = take(sizeof(float) * (size_t)m * n);            if (w) w->sT = (float*)p;
    p = take(sizeof(float) * (size_t)m);                if (w) w->alpha = (float*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->counts = (int32_t*)p;
    p = take(sizeof(int32_t) * qb::kStWords);           if (w) w->status = (int32_t*)p;
    p = take(sizeof(double) * (size_t)n * n);           if (w) w->W = (double*)p;
    p = take(sizeof(int32_t) * (size_t)n * n);          if (w) w->A = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)m * k);          if (w) w->slot = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)m * k);          if (w) w->dest = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)m * k);          if (w) w->src = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)(n + 1));        if (w) w->offsets = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->routed = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->kept = (int32_t*)p;
    p = take(capacity_workspace_bytes(m, k, n, m));     if (w) w->cap_ws = p;
    return off;
}

size_t balance_workspace_bytes(int64_t m, int32_t n, int32_t k) { return qb_layout(m, n, k, nullptr, nullptr); }

template <int NT>
static void launch_row_t(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                         int32_t* topk_idx, int32_t* counts, int32_t* status, cudaStream_t stream) {
    int64_t blocks = (m + qb::kRowThreads / 32 - 1) / (qb::kRowThreads / 32);
    if (blocks > (int64_t)kNumSMs * 8) blocks = (int64_t)kNumSMs * 8;
    if (blocks < 1) blocks = 1;
    qb_row_kernel<NT><<<(unsigned)blocks, qb::kRowThreads, 0, stream>>>(s, m, n, k, beta, rule, alpha, topk_idx,
                                                                        counts, status);
}

static void launch_row(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                       int32_t* topk_idx, int32_t* counts, int32_t* status, cudaStream_t stream) {
    if (n <= 32) launch_row_t<1>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, stream);
    else if (n <= 64) launch_row_t<2>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, stream);
    else if (n <= 128) launch_row_t<4>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, stream);
    else launch_row_t<8>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, stream);
}

// Returns a moe_status; SOLVE synchronises the stream between phases.
int run_balance_assign(const float* s, int64_t m, int n, int k, float* beta, int mode, int rule, int max_iters,
                       int max_repair, int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                       const char** err) {
    QBWorkspace w;
    qb_layout(m, n, k, &w, static_cast<char*>(workspace));
    const int64_t C = m * k / n;
    cudaError_t ce;
    if ((ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * qb::kStWords, stream)) != cudaSuccess) goto cuda_fail;
    {
        dim3 tb(32, 8), tg((unsigned)((m + 31) / 32), (unsigned)((n + 31) / 32));
        transpose_kernel<<<tg, tb, 0, stream>>>(s, m, n, w.sT);
    }
    if (mode == MOE_QB_STEP) {
        if ((ce = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * n, stream)) != cudaSuccess) goto cuda_fail;
        launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status, stream);
        qb_col_kernel<<<n, qb::kColThreads, 0, stream>>>(w.sT, m, n, C, w.alpha, rule, beta);
        qb_info_kernel<<<1, 32, 0, stream>>>(w.counts, n, C, w.status, 1, info);
        if ((ce = cudaGetLastError()) != cudaSuccess) goto cuda_fail;
        return MOE_OK;
    }
    {
        int iters = 0;
        int32_t hcounts[kMaxExperts];
        int64_t excess = 0;
        for (;;) {
            if ((ce = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * n, stream)) != cudaSuccess) goto cuda_fail;
            if ((ce = cudaMemsetAsync(w.status + qb::kStTies, 0, sizeof(int32_t), stream)) != cudaSuccess)
                goto cuda_fail;
            launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status, stream);
            if ((ce = cudaMemcpyAsync(hcounts, w.counts, sizeof(int32_t) * n, cudaMemcpyDeviceToHost, stream)) !=
                cudaSuccess)
                goto cuda_fail;
            if ((ce = cudaStreamSynchronize(stream)) != cudaSuccess) goto cuda_fail;
            excess = 0;
            for (int e = 0; e < n; ++e) if (hcounts[e] > C) excess += hcounts[e] - C;
            if (excess == 0 || iters >= max_iters) break;
            qb_col_kernel<<<n, qb::kColThreads, 0, stream>>>(w.sT, m, n, C, w.alpha, rule, beta);
            ++iters;
        }
        const int64_t moves = excess < max_repair ? excess : max_repair;
        for (int64_t a = 0; a < moves; ++a) {
            launch_capacity(topk_idx, m, k, n, (int32_t)(m * k), m, w.slot, w.dest, w.src, w.offsets, w.routed,
                            w.kept, w.cap_ws, stream);
            qb_arc_kernel<<<n, qb::kRepairThreads, 0, stream>>>(s, n, k, topk_idx, w.src, w.offsets, w.W, w.A,
                                                                w.status);
            qb_repair_step_kernel<<<1, qb::kRepairThreads, 0, stream>>>(n, C, k, w.W, w.A, w.counts, topk_idx,
                                                                        w.status);
        }
        qb_info_kernel<<<1, 32, 0, stream>>>(w.counts, n, C, w.status, iters, info);
        if ((ce = cudaGetLastError()) != cudaSuccess) goto cuda_fail;
        int32_t hinfo[4], hstatus[qb::kStWords];
        if ((ce = cudaMemcpyAsync(hinfo, info, sizeof(hinfo), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
            goto cuda_fail;
        if ((ce = cudaMemcpyAsync(hstatus, w.status, sizeof(hstatus), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
            goto cuda_fail;
        if ((ce = cudaStreamSynchronize(stream)) != cudaSuccess) goto cuda_fail;
        if (hstatus[qb::kStError]) { *err = "balanced-assignment repair found no valid augmenting path"; return MOE_ERR_INTERNAL; }
        if (hinfo[2] != 0) { *err = "max_repair moves did not remove the excess"; return MOE_ERR_NOT_CONVERGED; }
        return MOE_OK;
    }
cuda_fail:
    *err = cudaGetErrorString(ce);
    return MOE_ERR_CUDA;
}

}  // namespace moe
