// stats.cu -- load statistics f_i, P_i, the auxiliary loss (per micro-batch and
// global batch), MaxVio/MinVio/AvgVio and the Loss-Free bias update.
//
// Switch Transformers paper review (tildalice.io/?p=118), auxiliary load
// balancing loss L = alpha N sum_i f_i P_i (f_i routed fraction, P_i mean
// router probability); Qwen global-batch load balance (agentlenshq.com): the
// loss per micro-batch averaged over micro-batches vs f_i pooled over the
// whole batch; MoE travelogue 6 (kexue.fm/archives/11619), Demo code
// (MaxVio/MinVio/AvgVio) and eq. (2) b <- b - gamma sign(F - 1/n).
//
// One launch. Each CTA (256 threads) takes kRows consecutive rows of one
// segment: thread (four experts, row group g) sums its rows' probabilities in
// fp64 from 16-byte loads, eight in flight, the groups are folded in order,
// and the routed picks are counted. The CTA publishes its partial sums, fences, and
// takes a ticket; the last CTA of a segment folds that segment's chunks in
// chunk order (f, P and the loss of the segment), and the last segment to
// finish folds the segments in order (the whole batch, the micro-batch mean
// and global loss, the violations, the bias update). The fold order never
// depends on which CTA finishes last, and there are no floating-point atomics,
// so the results are bit-reproducible.
#include "common.cuh"

namespace moe {

namespace stats {
constexpr int kRows = 256;      // rows per CTA
constexpr int kThreads = 256;
constexpr int kBatch = 8;       // loads in flight per thread
}  // namespace stats

struct StatsGeometry {
    int64_t nseg, cps, nchunks;
};
static StatsGeometry stats_geometry(int64_t m, int64_t seg_len) {
    StatsGeometry g;
    g.nseg = m / seg_len;
    g.cps = (seg_len + stats::kRows - 1) / stats::kRows;
    g.nchunks = g.nseg * g.cps;
    return g;
}

struct StatsWs {
    double *psum, *segps, *segaux;
    int32_t *pcnt, *segcnt, *tickets;  // tickets: one per segment, then one for the batch
};

static size_t stats_layout(int64_t m, int32_t n, int64_t seg_len, StatsWs* w, char* base) {
    StatsGeometry g = stats_geometry(m, seg_len);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* p = base ? base + off : nullptr;
        off += (bytes + 255) & ~(size_t)255;
        return p;
    };
    char* p;
    p = take(sizeof(double) * (size_t)n * g.nchunks);   if (w) w->psum = (double*)p;
    p = take(sizeof(double) * (size_t)n * g.nseg);      if (w) w->segps = (double*)p;
    p = take(sizeof(double) * (size_t)g.nseg);          if (w) w->segaux = (double*)p;
    p = take(sizeof(int32_t) * (size_t)n * g.nchunks);  if (w) w->pcnt = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n * g.nseg);     if (w) w->segcnt = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)(g.nseg + 1));   if (w) w->tickets = (int32_t*)p;
    return off;
}

size_t stats_workspace_bytes(int64_t m, int32_t n, int64_t seg_len) {
    if (seg_len <= 0) return 0;
    return stats_layout(m, n, seg_len, nullptr, nullptr);
}

// Fixed-order block reductions of one double per thread.
__device__ __forceinline__ double block_sum_d(double v, double* sh) {
    const int tid = threadIdx.x;
    v = warp_sum_d(v);
    __syncthreads();
    if ((tid & 31) == 0) sh[tid >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
    __syncthreads();
    return t;
}
__device__ __forceinline__ double block_max_d(double v, double* sh) {
    const int tid = threadIdx.x;
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((tid & 31) == 0) sh[tid >> 5] = v;
    __syncthreads();
    double t = -INFINITY;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = fmax(t, sh[w]);
    __syncthreads();
    return t;
}

// Fold `cnt` [nblk][n] and `ps` [nblk][n] over the blocks in a fixed order, all threads taking part:
// thread (e, p) sums blocks p, p + P, ... (P = threads / padded n), then thread e adds the P partial
// sums in p order. Thread e < n gets the totals; barriers inside.
// The blocks were written by other CTAs of this launch: read them through L2 (__ldcg), never the
// read-only path.
__device__ __forceinline__ void fold_blocks(const int32_t* cnt, const double* ps,
                                            int64_t nblk, int n, bool has_ps, long long* pc, double* pp,
                                            int64_t* cnt_out, double* ps_out) {
    const int tid = threadIdx.x;
    const int npad = (n + 31) & ~31;
    const int P = stats::kThreads / npad;
    const int e = tid % npad, p = tid / npad;
    long long cs = 0;
    double s = 0.0;
    if (p < P && e < n) {
        for (int64_t b0 = p; b0 < nblk; b0 += (int64_t)P * stats::kBatch) {
            int32_t cv[stats::kBatch];
            double pv[stats::kBatch];
#pragma unroll
            for (int u = 0; u < stats::kBatch; ++u) {
                const int64_t b = b0 + (int64_t)u * P;
                cv[u] = b < nblk ? __ldcg(cnt + b * n + e) : 0;
                pv[u] = (has_ps && b < nblk) ? __ldcg(ps + b * n + e) : 0.0;
            }
#pragma unroll
            for (int u = 0; u < stats::kBatch; ++u) { cs += cv[u]; s += pv[u]; }
        }
    }
    pc[tid] = cs;
    pp[tid] = s;
    __syncthreads();
    if (tid < n) {
        long long c = 0;
        double t = 0.0;
        for (int q = 0; q < P; ++q) { c += pc[q * npad + tid]; t += pp[q * npad + tid]; }
        *cnt_out = c;
        *ps_out = t;
    }
    __syncthreads();
}

// Whole-batch results from the batch totals held by thread e < n (routed copies `tot`, probability
// sum `pall`) over m tokens: f and P rows, the loss on them, the violations and the Loss-Free
// update. Every thread of the block calls it (block reductions inside). Optional outputs may be NULL.
// Weight of the micro-batch loss in the hybrid loss ("Qwen global-batch load balance", balancing
// efficiency and effectiveness: the micro-batch loss added to the global-batch loss with 0.01).
constexpr double kHybridMicroWeight = 0.01;

// Whole-batch f, P, loss, violations and bias update; returns the loss (0 without scores).
__device__ double finish_batch(int64_t tot, double pall, int64_t m, int n, int k, bool has_probs, float alpha,
                             float* __restrict__ f_row, float* __restrict__ P_row, float* __restrict__ aux_out,
                             float* __restrict__ vio, float* __restrict__ bias, float gamma, double* sh) {
    const int tid = threadIdx.x;
    const bool valid = tid < n;
    double gprod = 0.0;
    if (valid) {
        const double fg = (double)tot / ((double)k * (double)m);
        if (f_row) f_row[tid] = (float)fg;
        if (has_probs) {
            const double pg = pall / (double)m;
            if (P_row) P_row[tid] = (float)pg;
            gprod = fg * pg;
        }
    }
    double g = 0.0;
    if (has_probs) {
        g = (double)alpha * (double)n * block_sum_d(gprod, sh);
        if (tid == 0 && aux_out) *aux_out = (float)g;
    }
    const double F = valid ? (double)tot / ((double)m * (double)k) * (double)n - 1.0 : 0.0;
    if (vio) {
        const double av = block_sum_d(valid ? fabs(F) : 0.0, sh);
        const double mx = block_max_d(valid ? F : -INFINITY, sh);
        const double mn = -block_max_d(valid ? -F : -INFINITY, sh);
        if (tid == 0) { vio[0] = (float)mx; vio[1] = (float)mn; vio[2] = (float)(av / (double)n); }
    }
    if (bias && valid) {
        const int64_t lhs = tot * (int64_t)n, rhs = m * (int64_t)k;
        float b = bias[tid];
        if (lhs > rhs) b = __fsub_rn(b, gamma);
        else if (lhs < rhs) b = __fadd_rn(b, gamma);
        bias[tid] = b;
    }
    return g;
}

__global__ void __launch_bounds__(stats::kThreads, 2)
stats_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx, int64_t m, int n, int k,
             int64_t seg_len, int64_t cps, int64_t nseg, float alpha, float* __restrict__ f, float* __restrict__ P,
             float* __restrict__ aux, float* __restrict__ vio, float* __restrict__ bias, float gamma, StatsWs w,
             double* __restrict__ totals) {
    __shared__ int cnt[kMaxExperts];
    __shared__ double part[stats::kThreads * 4];
    __shared__ long long pc[stats::kThreads];
    __shared__ double sh[stats::kThreads / 32];
    __shared__ int s_last;
    const int tid = threadIdx.x;
    pdl_trigger();
    pdl_wait();
    const int64_t chunk = blockIdx.x;
    const int64_t seg = chunk / cps, c = chunk - seg * cps;
    const int64_t r0 = seg * seg_len + c * stats::kRows;
    const int64_t r1 = min(r0 + (int64_t)stats::kRows, (seg + 1) * seg_len);
    const bool has_probs = probs != nullptr;

    // ---- this chunk: counts and per-expert probability sums
    for (int e = tid; e < n; e += stats::kThreads) cnt[e] = 0;
    __syncthreads();
    for (int64_t q = r0 * k + tid; q < r1 * k; q += stats::kThreads) {
        const int e = idx[q];
        if (e < 0 || e >= n) record_error(kErrExpertIndex);
        else atomicAdd(&cnt[e], 1);
    }
    if (has_probs) {
        if ((n & 3) == 0) {
            // 16-byte loads: thread (column quad c4, row group g); rows g, g + G, ... of the chunk
            const int c4n = n >> 2, G = stats::kThreads / c4n;
            const int c4 = tid % c4n, g = tid / c4n;
            const float4* p4 = reinterpret_cast<const float4*>(probs);
            double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
            if (g < G) {
                for (int64_t r = r0 + g; r < r1; r += (int64_t)G * stats::kBatch) {
                    float4 v[stats::kBatch];
#pragma unroll
                    for (int u = 0; u < stats::kBatch; ++u) {
                        const int64_t rr = r + (int64_t)u * G;
                        v[u] = rr < r1 ? p4[rr * c4n + c4] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < stats::kBatch; ++u) {
                        s0 += (double)v[u].x; s1 += (double)v[u].y; s2 += (double)v[u].z; s3 += (double)v[u].w;
                    }
                }
            }
            part[tid * 4 + 0] = s0; part[tid * 4 + 1] = s1; part[tid * 4 + 2] = s2; part[tid * 4 + 3] = s3;
            __syncthreads();
            if (tid < n) {
                const int cq = tid >> 2, q = tid & 3;
                double t = 0.0;
                for (int gg = 0; gg < G; ++gg) t += part[(gg * c4n + cq) * 4 + q];
                w.psum[chunk * n + tid] = t;
            }
        } else {
            const int npad = (n + 31) & ~31;
            const int G = stats::kThreads / npad;
            const int e = tid % npad, g = tid / npad;
            double s = 0.0;
            if (g < G && e < n) {
                for (int64_t r = r0 + g; r < r1; r += (int64_t)G * stats::kBatch) {
                    float v[stats::kBatch];
#pragma unroll
                    for (int u = 0; u < stats::kBatch; ++u) {
                        const int64_t rr = r + (int64_t)u * G;
                        v[u] = rr < r1 ? probs[rr * n + e] : 0.f;
                    }
#pragma unroll
                    for (int u = 0; u < stats::kBatch; ++u) s += (double)v[u];
                }
            }
            part[tid] = s;
            __syncthreads();
            if (tid < n) {
                double t = 0.0;
                for (int gg = 0; gg < G; ++gg) t += part[gg * npad + tid];
                w.psum[chunk * n + tid] = t;
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < n; e += stats::kThreads) w.pcnt[chunk * n + e] = cnt[e];
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&w.tickets[seg], 1) == (int)cps - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- last CTA of the segment: fold its chunks
    int64_t cs = 0;
    double ps = 0.0;
    fold_blocks(w.pcnt + seg * cps * n, w.psum + seg * cps * n, cps, n, has_probs, pc, part, &cs, &ps);
    double prod = 0.0;
    if (tid < n) {
        const int e = tid;
        w.segcnt[seg * n + e] = (int32_t)cs;
        const double fv = (double)cs / ((double)k * (double)seg_len);
        if (f) f[seg * n + e] = (float)fv;
        if (has_probs) {
            w.segps[seg * n + e] = ps;
            const double pv = ps / (double)seg_len;
            if (P) P[seg * n + e] = (float)pv;
            prod = fv * pv;
        }
    }
    if (has_probs) {
        const double a = (double)alpha * (double)n * block_sum_d(prod, sh);
        if (tid == 0) { if (aux) aux[seg] = (float)a; w.segaux[seg] = a; }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&w.tickets[nseg], 1) == (int)nseg - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- last segment: the whole batch, in segment order
    int64_t tot = 0;
    double pall = 0.0;
    fold_blocks(w.segcnt, w.segps, nseg, n, has_probs, pc, part, &tot, &pall);
    if (totals && tid < n) { totals[tid] = (double)tot; totals[n + tid] = has_probs ? pall : 0.0; }
    double micro = 0.0;
    if (has_probs && aux && tid == 0) {
        for (int64_t s = 0; s < nseg; ++s) micro += __ldcg(w.segaux + s);
        micro /= (double)nseg;
        aux[nseg] = (float)micro;
    }
    const double g = finish_batch(tot, pall, m, n, k, has_probs, alpha, f ? f + nseg * n : nullptr,
                                  P ? P + nseg * n : nullptr, aux ? aux + nseg + 1 : nullptr, vio, bias, gamma, sh);
    // the hybrid loss: the global-batch loss plus the weighted micro-batch loss
    if (has_probs && aux && tid == 0) aux[nseg + 2] = (float)(g + kHybridMicroWeight * micro);
}

// Global-batch results from totals [2, n] summed over data-parallel ranks (m_total tokens).
__global__ void __launch_bounds__(stats::kThreads)
stats_global_kernel(const double* __restrict__ totals, int64_t m_total, int n, int k, int has_probs, float alpha,
                    float* __restrict__ f, float* __restrict__ P, float* __restrict__ aux, float* __restrict__ vio,
                    float* __restrict__ bias, float gamma) {
    __shared__ double sh[stats::kThreads / 32];
    const int tid = threadIdx.x;
    int64_t tot = 0;
    double pall = 0.0;
    if (tid < n) {
        const double c = totals[tid];
        tot = (c >= 0.0 && c < 9.0e15) ? (int64_t)c : 0;
        if (c < 0.0 || c >= 9.0e15 || c != (double)tot) record_error(kErrExpertIndex);
        pall = totals[n + tid];
    }
    finish_batch(tot, pall, m_total, n, k, has_probs != 0, alpha, f, P, aux, vio, bias, gamma, sh);
}

cudaError_t launch_stats(const float* probs, const int32_t* topk_idx, int64_t m, int n, int k, int64_t seg_len,
                         float alpha, float* f, float* P, float* aux, float* vio, float* bias, float gamma,
                         void* workspace, cudaStream_t stream, double* totals) {
    StatsGeometry g = stats_geometry(m, seg_len);
    StatsWs w;
    stats_layout(m, n, seg_len, &w, static_cast<char*>(workspace));
    cudaError_t e = cudaMemsetAsync(w.tickets, 0, sizeof(int32_t) * (size_t)(g.nseg + 1), stream);
    if (e != cudaSuccess) return e;
    return launch_pdl(stats_kernel, dim3((unsigned)g.nchunks), dim3(stats::kThreads), 0, stream, probs, topk_idx, m,
                      n, k, seg_len, g.cps, g.nseg, alpha, f, P, aux, vio, bias, gamma, w, totals);
}

cudaError_t launch_stats_global(const double* totals, int64_t m_total, int n, int k, int has_probs, float alpha,
                                float* f, float* P, float* aux, float* vio, float* bias, float gamma,
                                cudaStream_t stream) {
    stats_global_kernel<<<1, stats::kThreads, 0, stream>>>(totals, m_total, n, k, has_probs, alpha, f, P, aux, vio,
                                                           bias, gamma);
    return cudaGetLastError();
}

// Router gradient of w_global L_global + w_micro L_micro ("Switch Transformers paper review",
// auxiliary loss: f_i is fixed by the routing decision, the gradient flows through P_i, the mean
// score). For token t of segment s: dL/dp_i = g_i = w_global alpha n f^G_i / m
// + w_micro alpha n f^s_i / (nseg seg_len); softmax: dL/dh_j = p_j (g_j - sum_i p_i g_i);
// sigmoid: dL/dh_j = g_j p_j (1 - p_j). One warp per token, lane j holds experts lane + 32 q;
// reads the scores once and writes the gradient once (HBM-bound).
template <int NT>
__global__ void __launch_bounds__(256)
loss_grad_kernel(const float* __restrict__ probs, int fn, const float* __restrict__ f, int64_t m, int n,
                 int64_t seg_len, int64_t nseg, float alpha, float w_micro, float w_global,
                 float* __restrict__ dlogits) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    const float cg = w_global * alpha * (float)n / (float)m;
    const float cm = w_micro * alpha * (float)n / ((float)nseg * (float)seg_len);
    for (int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); t < m; t += warps) {
        const int64_t seg = t / seg_len;
        float p[NT], g[NT];
        float c = 0.f;
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const int j = lane + 32 * q;
            p[q] = 0.f;
            g[q] = 0.f;
            if (j < n) {
                p[q] = probs[t * n + j];
                g[q] = fmaf(cg, f[nseg * n + j], cm * f[seg * n + j]);
                c = fmaf(p[q], g[q], c);
            }
        }
        c = warp_sum(c);
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const int j = lane + 32 * q;
            if (j < n)
                dlogits[t * n + j] = fn == MOE_SOFTMAX ? p[q] * (g[q] - c) : g[q] * p[q] * (1.f - p[q]);
        }
    }
}

cudaError_t launch_loss_grad(const float* probs, int fn, const float* f, int64_t m, int n, int64_t seg_len, float alpha,
                             float w_micro, float w_global, float* dlogits, cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    int64_t blocks = (m + 7) / 8;
    if (blocks > (int64_t)kNumSMs * 8) blocks = (int64_t)kNumSMs * 8;
    const int64_t nseg = m / seg_len;
    if (n <= 32)
        return launch_pdl(loss_grad_kernel<1>, dim3((unsigned)blocks), dim3(256), 0, stream, probs, fn, f, m, n,
                          seg_len, nseg, alpha, w_micro, w_global, dlogits);
    if (n <= 64)
        return launch_pdl(loss_grad_kernel<2>, dim3((unsigned)blocks), dim3(256), 0, stream, probs, fn, f, m, n,
                          seg_len, nseg, alpha, w_micro, w_global, dlogits);
    if (n <= 128)
        return launch_pdl(loss_grad_kernel<4>, dim3((unsigned)blocks), dim3(256), 0, stream, probs, fn, f, m, n,
                          seg_len, nseg, alpha, w_micro, w_global, dlogits);
    return launch_pdl(loss_grad_kernel<8>, dim3((unsigned)blocks), dim3(256), 0, stream, probs, fn, f, m, n, seg_len,
                      nseg, alpha, w_micro, w_global, dlogits);
}

}  // namespace moe
