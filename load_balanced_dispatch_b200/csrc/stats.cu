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
// Two launches. `partial`: each CTA takes kRows consecutive rows of one
// segment, sums the probabilities per expert in fp64 (column-parallel,
// coalesced row reads, 8 loads in flight per thread, fixed order) and counts
// the routed picks. `final`: one CTA; every thread folds the chunks of one
// (segment, expert) pair in order, then one expert per thread folds the
// segments for the whole batch, then warps reduce the loss terms in a fixed
// tree order. No floating-point atomics anywhere, so the results are
// bit-reproducible.
#include "common.cuh"

namespace moe {

namespace stats {
constexpr int kRows = 128;      // rows per partial CTA
constexpr int kThreads = 256;
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

size_t stats_workspace_bytes(int64_t m, int32_t n, int64_t seg_len) {
    if (seg_len <= 0) return 0;
    StatsGeometry g = stats_geometry(m, seg_len);
    // psum [nchunks][n] f64, prod [nseg + 1][n] f64, segps [nseg][n] f64, pcnt [nchunks][n] i32, segcnt [nseg][n] i32
    return sizeof(double) * (size_t)n * (size_t)(g.nchunks + 2 * g.nseg + 1) +
           sizeof(int32_t) * (size_t)n * (size_t)(g.nchunks + g.nseg);
}

__global__ void __launch_bounds__(stats::kThreads)
stats_partial_kernel(const float* __restrict__ probs, const int32_t* __restrict__ idx, int n, int k, int64_t seg_len,
                     int64_t cps, double* __restrict__ psum, int32_t* __restrict__ pcnt) {
    __shared__ int cnt[kMaxExperts];
    __shared__ double part[stats::kThreads];
    const int tid = threadIdx.x;
    const int64_t chunk = blockIdx.x;
    const int64_t seg = chunk / cps, c = chunk - seg * cps;
    const int64_t r0 = seg * seg_len + c * stats::kRows;
    const int64_t r1 = min(r0 + (int64_t)stats::kRows, (seg + 1) * seg_len);
    for (int e = tid; e < n; e += stats::kThreads) cnt[e] = 0;
    __syncthreads();
    for (int64_t q = r0 * k + tid; q < r1 * k; q += stats::kThreads) {
        const int e = idx[q];
        if (e < 0 || e >= n) record_error(kErrExpertIndex);
        else atomicAdd(&cnt[e], 1);
    }
    if (probs) {
        const int npad = (n + 31) & ~31;
        const int groups = stats::kThreads / npad > 0 ? stats::kThreads / npad : 1;
        const int e = tid % npad, gid = tid / npad;
        double s = 0.0;
        if (gid < groups && e < n) {
            for (int64_t r = r0 + gid; r < r1; r += 8 * (int64_t)groups) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int64_t rr = r + (int64_t)u * groups;
                    v[u] = rr < r1 ? probs[rr * n + e] : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) s += (double)v[u];
            }
        }
        part[tid] = s;
        __syncthreads();
        if (tid < n) {
            double t = 0.0;
            for (int g = 0; g < groups; ++g) t += part[g * npad + tid];
            psum[chunk * n + tid] = t;
        }
    }
    __syncthreads();
    for (int e = tid; e < n; e += stats::kThreads) pcnt[chunk * n + e] = cnt[e];
}

// Fixed-order block reduction of one double per thread (256 threads).
__device__ __forceinline__ double block_sum_d(double v, double* sh) {
    const int tid = threadIdx.x;
    v = warp_sum_d(v);
    __syncthreads();
    if ((tid & 31) == 0) sh[tid >> 5] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < stats::kThreads / 32; ++w) t += sh[w];
    __syncthreads();
    return t;
}

__global__ void __launch_bounds__(stats::kThreads)
stats_final_kernel(const double* __restrict__ psum, const int32_t* __restrict__ pcnt, int has_probs, int64_t m, int n,
                   int k, int64_t seg_len, int64_t nseg, int64_t cps, float alpha, float* __restrict__ f,
                   float* __restrict__ P, float* __restrict__ aux, float* __restrict__ vio,
                   float* __restrict__ bias, float gamma, double* __restrict__ prod, double* __restrict__ segps,
                   int32_t* __restrict__ segcnt) {
    __shared__ double sh[stats::kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // phase A: one (segment, expert) pair per thread folds its chunks in order, 8 loads in flight
    for (int64_t pr = tid; pr < nseg * n; pr += stats::kThreads) {
        const int64_t s = pr / n;
        const int e = (int)(pr - s * n);
        int64_t cs = 0;
        double ps = 0.0;
        for (int64_t c0 = 0; c0 < cps; c0 += 8) {
            int32_t cv[8];
            double pv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t c = c0 + u;
                cv[u] = c < cps ? pcnt[(s * cps + c) * n + e] : 0;
                pv[u] = (has_probs && c < cps) ? psum[(s * cps + c) * n + e] : 0.0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) { cs += cv[u]; ps += pv[u]; }
        }
        segcnt[s * n + e] = (int32_t)cs;
        const double fv = (double)cs / ((double)k * (double)seg_len);
        f[s * n + e] = (float)fv;
        if (has_probs) {
            segps[s * n + e] = ps;
            const double pv = ps / (double)seg_len;
            P[s * n + e] = (float)pv;
            prod[s * n + e] = fv * pv;
        }
    }
    __syncthreads();
    // phase B: the whole batch, one expert per thread, segments in order
    const int e = tid;
    int64_t tot = 0;
    double pall = 0.0;
    if (e < n) {
        for (int64_t s0 = 0; s0 < nseg; s0 += 8) {
            int32_t cv[8];
            double pv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t s = s0 + u;
                cv[u] = s < nseg ? segcnt[s * n + e] : 0;
                pv[u] = (has_probs && s < nseg) ? segps[s * n + e] : 0.0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) { tot += cv[u]; pall += pv[u]; }
        }
        const double fg = (double)tot / ((double)k * (double)m);
        f[nseg * n + e] = (float)fg;
        if (has_probs) {
            const double pg = pall / (double)m;
            P[nseg * n + e] = (float)pg;
            prod[nseg * n + e] = fg * pg;
        }
    }
    __syncthreads();
    if (has_probs) {
        // per-segment losses: warp w folds segments w, w+8, ... ; its running sum of losses in order
        double wsum = 0.0;
        for (int64_t s = warp; s < nseg + 1; s += stats::kThreads / 32) {
            double t = 0.0;
            for (int j = lane; j < n; j += 32) t += prod[s * n + j];
            t = warp_sum_d(t);
            const double a = (double)alpha * (double)n * t;
            if (lane == 0) aux[s < nseg ? s : nseg + 1] = (float)a;
            if (s < nseg) wsum += a;
        }
        if (lane != 0) wsum = 0.0;
        const double micro = block_sum_d(wsum, sh);
        if (tid == 0) aux[nseg] = (float)(micro / (double)nseg);
    }
    // MaxVio / MinVio / AvgVio of the pooled counts
    const double F = (e < n) ? (double)tot / ((double)m * (double)k) * (double)n - 1.0 : 0.0;
    if (vio) {
        const double av = block_sum_d(e < n ? fabs(F) : 0.0, sh);
        double mx = (e < n) ? F : -INFINITY, mn = (e < n) ? F : INFINITY;
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        __shared__ double smx[stats::kThreads / 32], smn[stats::kThreads / 32];
        if (lane == 0) { smx[warp] = mx; smn[warp] = mn; }
        __syncthreads();
        if (tid == 0) {
            double a = -INFINITY, b = INFINITY;
            for (int w = 0; w < stats::kThreads / 32; ++w) { a = fmax(a, smx[w]); b = fmin(b, smn[w]); }
            vio[0] = (float)a; vio[1] = (float)b; vio[2] = (float)(av / (double)n);
        }
    }
    if (bias && e < n) {
        const int64_t lhs = tot * (int64_t)n, rhs = m * (int64_t)k;
        float b = bias[e];
        if (lhs > rhs) b = __fsub_rn(b, gamma);
        else if (lhs < rhs) b = __fadd_rn(b, gamma);
        bias[e] = b;
    }
}

cudaError_t launch_stats(const float* probs, const int32_t* topk_idx, int64_t m, int n, int k, int64_t seg_len,
                         float alpha, float* f, float* P, float* aux, float* vio, float* bias, float gamma,
                         void* workspace, cudaStream_t stream) {
    StatsGeometry g = stats_geometry(m, seg_len);
    double* psum = static_cast<double*>(workspace);
    double* prod = psum + g.nchunks * n;
    double* segps = prod + (g.nseg + 1) * n;
    int32_t* pcnt = reinterpret_cast<int32_t*>(segps + g.nseg * n);
    int32_t* segcnt = pcnt + g.nchunks * n;
    if (g.nchunks > 0)
        stats_partial_kernel<<<(unsigned)g.nchunks, stats::kThreads, 0, stream>>>(probs, topk_idx, n, k, seg_len,
                                                                                  g.cps, psum, pcnt);
    stats_final_kernel<<<1, stats::kThreads, 0, stream>>>(psum, pcnt, probs != nullptr, m, n, k, seg_len, g.nseg,
                                                          g.cps, alpha, f, P, aux, vio, bias, gamma, prod, segps,
                                                          segcnt);
    return cudaGetLastError();
}

}  // namespace moe
