// capacity.cu -- capacity slots and the expert-major row layout.
//
// Switch Transformers paper review (tildalice.io/?p=118), Expert Capacity and
// token drop; Switch Transformer read for implementation (molayo1419.me), the
// dispatch permutation and the capacity example: within a micro-batch, the
// j-th assignment (in token order) to expert e gets slot j and is kept iff
// j < capacity; overflow rides the residual path.
//
// Two launches over chunks of kChunk tokens (a chunk never straddles a
// segment):
//   count+scan -- per-chunk expert histogram (shared-memory integer atomics);
//             the last CTA to finish (ticket after a fence) runs the scan:
//             chunk prefixes within each segment, routed/kept counts, the
//             expert offsets (block exclusive scan over e) and each (segment,
//             expert) base row -- a thread per (segment, expert) pair when
//             they fit, else groups of threads walking the segments in order;
//   assign -- per chunk, a stable in-order rank for every assignment
//             (warp __match_any_sync groups + per-warp running counters in
//             shared memory, warps owning consecutive sub-ranges), then
//             slot / dest_row / src_token.
// Everything is integer arithmetic: the result is exact and deterministic.
#include "common.cuh"

namespace moe {

namespace cap {
constexpr int kChunk = 256;   // tokens per chunk
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
}  // namespace cap

struct CapGeometry {
    int64_t nseg, cps, nchunks;
};

static CapGeometry cap_geometry(int64_t m, int64_t seg_len) {
    CapGeometry g;
    g.nseg = m / seg_len;
    g.cps = (seg_len + cap::kChunk - 1) / cap::kChunk;
    g.nchunks = g.nseg * g.cps;
    return g;
}

// Workspace: hist [nchunks][n], prefix [nchunks][n], seg_base [nseg][n], then one ticket word.
size_t capacity_workspace_bytes(int64_t m, int32_t k, int32_t n, int64_t seg_len) {
    (void)k;
    if (seg_len <= 0) return 0;
    CapGeometry g = cap_geometry(m, seg_len);
    return sizeof(int32_t) * ((size_t)n * (size_t)(2 * g.nchunks + g.nseg) + 1);
}

__device__ __forceinline__ void chunk_range(int64_t chunk, int64_t cps, int64_t seg_len, int64_t& seg, int64_t& t0,
                                            int64_t& t1) {
    seg = chunk / cps;
    const int64_t c = chunk - seg * cps;
    t0 = seg * seg_len + c * cap::kChunk;
    t1 = min(t0 + (int64_t)cap::kChunk, (seg + 1) * seg_len);
}

// Block-wide exclusive scan of one value per thread (blockDim.x == 256), in a fixed order.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* sh, int64_t& total) {
    const int tid = threadIdx.x;
    sh[tid] = v;
    __syncthreads();
    for (int o = 1; o < cap::kThreads; o <<= 1) {
        int64_t add = tid >= o ? sh[tid - o] : 0;
        __syncthreads();
        sh[tid] += add;
        __syncthreads();
    }
    total = sh[cap::kThreads - 1];
    return sh[tid] - v;
}

// The scan, run by the last CTA of the count phase. Thread (e, g): expert e = tid % npad, group
// g = tid / npad of P = blockDim / npad groups; group g takes the g-th contiguous range of each
// segment's chunks, holding up to kRun histogram entries in registers. The groups' sums are
// added in group order, so each chunk's prefix (the earlier chunks of its segment, in chunk
// order) is exact. hist was written by other CTAs of this launch, so it is read through L2
// (__ldcg). Ranges longer than kRun (more chunks per segment than P kRun) re-read hist.
namespace cap {
constexpr int kRun = 16;
}
__device__ __forceinline__ void cap_scan_body(const int32_t* hist, int n, int64_t nseg, int64_t cps, int32_t capacity,
                                              int32_t* __restrict__ prefix, int32_t* __restrict__ seg_base,
                                              int32_t* __restrict__ expert_offsets, int32_t* __restrict__ routed_count,
                                              int32_t* __restrict__ kept_count) {
    __shared__ int64_t sh[cap::kThreads];
    __shared__ int64_t part[cap::kThreads];
    const int tid = threadIdx.x;
    const int npad = (n + 31) & ~31;
    const int P = cap::kThreads / npad;
    const int e = tid % npad, g = tid / npad;
    const bool act = g < P && e < n;
    const int64_t per = (cps + P - 1) / P;
    const int64_t c0 = min(cps, (int64_t)g * per), c1 = min(cps, c0 + per);
    int64_t kept_total = 0;
    for (int64_t s = 0; s < nseg; ++s) {
        const int32_t* hs = hist + s * cps * n;
        int32_t h[cap::kRun];
        int64_t sum = 0;
        if (act) {
#pragma unroll
            for (int u = 0; u < cap::kRun; ++u) {
                h[u] = (c0 + u < c1) ? __ldcg(hs + (c0 + u) * n + e) : 0;
                sum += h[u];
            }
            for (int64_t c = c0 + cap::kRun; c < c1; ++c) sum += __ldcg(hs + c * n + e);
        }
        part[tid] = sum;
        __syncthreads();
        int64_t run = 0, total = 0;
        if (act) {
            for (int q = 0; q < P; ++q) {
                const int64_t v = part[q * npad + e];
                if (q < g) run += v;
                total += v;
            }
#pragma unroll
            for (int u = 0; u < cap::kRun; ++u) {
                if (c0 + u < c1) {
                    prefix[(s * cps + c0 + u) * n + e] = (int32_t)run;
                    run += h[u];
                }
            }
            for (int64_t c = c0 + cap::kRun; c < c1; ++c) {
                prefix[(s * cps + c) * n + e] = (int32_t)run;
                run += __ldcg(hs + c * n + e);
            }
            if (g == 0) {
                const int64_t kept = total < capacity ? total : (int64_t)capacity;
                routed_count[s * n + e] = (int32_t)total;
                kept_count[s * n + e] = (int32_t)kept;
                kept_total += kept;
            }
        }
        __syncthreads();
    }
    // expert offsets: exclusive scan over the experts of their kept totals (held by group 0)
    int64_t total;
    const int64_t off = block_exclusive_scan((g == 0 && e < n) ? kept_total : 0, sh, total);
    // thread tid's scan slot is tid; the expert of group 0 is e = tid there
    if (g == 0 && e < n) {
        expert_offsets[e] = (int32_t)off;
        int64_t base = off;
        for (int64_t s = 0; s < nseg; ++s) {
            seg_base[s * n + e] = (int32_t)base;
            base += kept_count[s * n + e];
        }
    }
    if (tid == 0) expert_offsets[n] = (int32_t)total;
}

// The same scan with one thread per (segment, expert) pair, when the pairs fit in shared memory
// and a segment has at most kPairChunks chunks: each thread loads all of its pair's chunk counts
// at once and writes the pair's prefixes in chunk order (one round of L2 latency instead of one
// per segment), then thread e adds expert e's kept totals over the segments in segment order.
namespace cap {
constexpr int kPairCap = 4096;
constexpr int kPairChunks = 32;
}
__device__ __forceinline__ void cap_scan_pairs(const int32_t* hist, int n, int64_t nseg, int64_t cps,
                                               int32_t capacity, int32_t* __restrict__ prefix,
                                               int32_t* __restrict__ seg_base, int32_t* __restrict__ expert_offsets,
                                               int32_t* __restrict__ routed_count, int32_t* __restrict__ kept_count) {
    __shared__ int32_t kept_sh[cap::kPairCap];
    __shared__ int64_t sh[cap::kThreads];
    const int tid = threadIdx.x;
    const int64_t npairs = nseg * n;
    for (int64_t pr = tid; pr < npairs; pr += blockDim.x) {
        const int64_t s = pr / n;
        const int e = (int)(pr - s * n);
        const int32_t* hs = hist + s * cps * n + e;
        int32_t h[cap::kPairChunks];
#pragma unroll
        for (int c = 0; c < cap::kPairChunks; ++c) h[c] = c < cps ? __ldcg(hs + (int64_t)c * n) : 0;
        int32_t* ps = prefix + s * cps * n + e;
        int32_t run = 0;
#pragma unroll
        for (int c = 0; c < cap::kPairChunks; ++c)
            if (c < cps) {
                ps[(int64_t)c * n] = run;
                run += h[c];
            }
        const int32_t kept = run < capacity ? run : capacity;
        routed_count[pr] = run;
        kept_count[pr] = kept;
        kept_sh[pr] = kept;
    }
    __syncthreads();
    int64_t ktot = 0;
    if (tid < n)
        for (int64_t s = 0; s < nseg; ++s) ktot += kept_sh[s * n + tid];
    int64_t total;
    const int64_t off = block_exclusive_scan(tid < n ? ktot : 0, sh, total);
    if (tid < n) {
        expert_offsets[tid] = (int32_t)off;
        int64_t base = off;
        for (int64_t s = 0; s < nseg; ++s) {
            seg_base[s * n + tid] = (int32_t)base;
            base += kept_sh[s * n + tid];
        }
    }
    if (tid == 0) expert_offsets[n] = (int32_t)total;
}

// Per-chunk expert histogram (shared-memory integer atomics); the last CTA to finish (a ticket
// taken after a fence) then runs the scan over all chunks.
__global__ void __launch_bounds__(cap::kThreads)
cap_count_scan_kernel(const int32_t* __restrict__ idx, int k, int n, int64_t seg_len, int64_t cps, int64_t nchunks,
                      int64_t nseg, int32_t capacity, int32_t* hist, int32_t* __restrict__ prefix,
                      int32_t* __restrict__ seg_base, int32_t* __restrict__ expert_offsets,
                      int32_t* __restrict__ routed_count, int32_t* __restrict__ kept_count, int32_t* ticket) {
    __shared__ int cnt[kMaxExperts];
    __shared__ int s_last;
    pdl_trigger();
    pdl_wait();
    for (int e = threadIdx.x; e < n; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    int64_t seg, t0, t1;
    chunk_range(blockIdx.x, cps, seg_len, seg, t0, t1);
    const int64_t a0 = t0 * k, a1 = t1 * k;
    for (int64_t q = a0 + threadIdx.x; q < a1; q += blockDim.x) {
        const int e = idx[q];
        if (e < 0 || e >= n) record_error(kErrExpertIndex);
        else atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) hist[(int64_t)blockIdx.x * n + e] = cnt[e];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1) == (int)(nchunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (nseg * n <= cap::kPairCap && cps <= cap::kPairChunks)
        cap_scan_pairs(hist, n, nseg, cps, capacity, prefix, seg_base, expert_offsets, routed_count, kept_count);
    else
        cap_scan_body(hist, n, nseg, cps, capacity, prefix, seg_base, expert_offsets, routed_count, kept_count);
}

__global__ void __launch_bounds__(cap::kThreads)
cap_assign_kernel(const int32_t* __restrict__ idx, int k, int n, int64_t seg_len, int64_t cps, int32_t capacity,
                  const int32_t* __restrict__ prefix, const int32_t* __restrict__ seg_base,
                  int32_t* __restrict__ slot, int32_t* __restrict__ dest_row, int32_t* __restrict__ src_token) {
    __shared__ int wcnt[cap::kWarps][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_trigger();
    pdl_wait();
    for (int q = tid; q < cap::kWarps * kMaxExperts; q += cap::kThreads) (&wcnt[0][0])[q] = 0;
    __syncthreads();
    int64_t seg, t0, t1;
    const int64_t chunk = blockIdx.x;
    chunk_range(chunk, cps, seg_len, seg, t0, t1);
    const int64_t a0 = t0 * k, A = (t1 - t0) * k;
    const int64_t per_warp = (A + cap::kWarps - 1) / cap::kWarps;
    const int64_t w0 = a0 + min((int64_t)warp * per_warp, A), w1 = a0 + min((int64_t)(warp + 1) * per_warp, A);
    const uint32_t lt_mask = (1u << lane) - 1u;

    // pass 1: per-warp expert counts over the warp's contiguous sub-range
    for (int64_t b = w0; b < w1; b += 32) {
        const int64_t q = b + lane;
        int e = q < w1 ? idx[q] : -1;
        if (e >= n) e = -1;
        const uint32_t grp = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (grp & lt_mask) == 0) wcnt[warp][e] += __popc(grp);
    }
    __syncthreads();
    // exclusive prefix over warps, seeded with the chunk's prefix within its segment
    for (int e = tid; e < n; e += cap::kThreads) {
        int run = prefix[chunk * n + e];
        for (int w = 0; w < cap::kWarps; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    // pass 2: ranks in order
    for (int64_t b = w0; b < w1; b += 32) {
        const int64_t q = b + lane;
        int e = q < w1 ? idx[q] : -1;
        if (e >= n) e = -1;
        const uint32_t grp = __match_any_sync(0xffffffffu, e);
        int rank = 0;
        if (e >= 0) rank = wcnt[warp][e] + __popc(grp & lt_mask);
        __syncwarp();
        if (e >= 0 && (grp & lt_mask) == 0) wcnt[warp][e] += __popc(grp);
        __syncwarp();
        if (q < w1) {
            int32_t sl = -1, dr = -1;
            if (e >= 0 && rank < capacity) {
                sl = rank;
                dr = seg_base[seg * n + e] + rank;
                src_token[dr] = (int32_t)(q / k);
            }
            slot[q] = sl;
            dest_row[q] = dr;
        }
    }
}

cudaError_t launch_capacity(const int32_t* topk_idx, int64_t m, int k, int n, int32_t capacity, int64_t seg_len,
                            int32_t* slot, int32_t* dest_row, int32_t* src_token, int32_t* expert_offsets,
                            int32_t* routed_count, int32_t* kept_count, void* workspace, cudaStream_t stream) {
    CapGeometry g = cap_geometry(m, seg_len);
    int32_t* hist = static_cast<int32_t*>(workspace);
    int32_t* prefix = hist + g.nchunks * n;
    int32_t* seg_base = prefix + g.nchunks * n;
    int32_t* ticket = seg_base + g.nseg * n;
    if (g.nchunks == 0) {
        // no tokens: empty layout, nothing to count
        cudaError_t e = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(n + 1), stream);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    {
        cudaError_t e = cudaMemsetAsync(ticket, 0, sizeof(int32_t), stream);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_pdl(cap_count_scan_kernel, dim3((unsigned)g.nchunks), dim3(cap::kThreads), 0, stream,
                               topk_idx, k, n, seg_len, g.cps, g.nchunks, g.nseg, capacity, hist, prefix, seg_base,
                               expert_offsets, routed_count, kept_count, ticket);
    if (e != cudaSuccess) return e;
    return launch_pdl(cap_assign_kernel, dim3((unsigned)g.nchunks), dim3(cap::kThreads), 0, stream, topk_idx, k, n,
                      seg_len, g.cps, capacity, (const int32_t*)prefix, (const int32_t*)seg_base, slot, dest_row,
                      src_token);
}

}  // namespace moe
