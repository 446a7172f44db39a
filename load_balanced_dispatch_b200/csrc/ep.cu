// ep.cu -- expert parallelism: the experts of the layer split over G ranks (one GPU each), the
// token rows moved by direct stores into, and loads from, the peers' buffers.
//
// "Switch Transformer read for implementation" (molayo1419.me), Expert Parallelism: experts sit
// on different devices, so the dispatch permutation and the return of the expert outputs become
// exchanges between devices, kept apart from the compute. "Switch Transformers paper review"
// (tildalice.io/?p=118), distributed training and communication cost: an all-to-all before the
// experts and one after them.
//
// Rank q owns experts q E .. q E + E - 1 (E = n / G). Every rank routes its own m tokens over
// all n experts and assigns capacity slots over its own tokens (moe_capacity_slots: capacity is
// decided per source rank). The exchange plan: each rank's expert_offsets [n + 1] are gathered
// over the ranks ([G, n + 1], one all-gather by the caller); from them every kept row has one
// place in its owner's receive buffer. Owner q's buffer holds its local experts in order; each
// expert's rows come from source rank 0 first, then rank 1, ..., and each source's rows keep that
// source's expert-major order. These are exactly the rows the one-GPU layer gives expert e on the
// concatenated batch with one capacity segment per rank, so the owner's FFN sees the same rows.
//
//   ep_plan_kernel      [G, n + 1] offsets -> this rank's send bases [n] (where its rows of
//                       expert e start in e's owner's buffer) and receive offsets [E + 1]
//   ep_dispatch_kernel  warp per token: its row is read once and stored into each kept pick's
//                       row of the owner's buffer (a peer pointer); the row index is kept
//   ep_combine_kernel   warp per token: y = residual + sum of gate x the owner's output rows
//                       (peer loads), fp32 accumulation, the combine's order of operations
// Plain 16-byte loads and stores through the peer pointers (no TMA, no multicast). The kernels
// wait on nothing: the caller orders the ranks between dispatch, the FFN and the combine.
#include "common.cuh"

namespace moe {

constexpr int kEpThreads = 256;

__global__ void __launch_bounds__(kMaxExperts)
ep_plan_kernel(const int32_t* __restrict__ offsets_all, int G, int n, int rank, int32_t* __restrict__ send_base,
               int32_t* __restrict__ recv_offsets) {
    __shared__ int32_t tot[kMaxExperts];
    const int e = threadIdx.x;
    const int E = n / G;
    int32_t total = 0, before = 0;
    if (e < n) {
        for (int src = 0; src < G; ++src) {
            const int32_t* off = offsets_all + (int64_t)src * (n + 1);
            const int32_t kept = off[e + 1] - off[e];
            if (kept < 0) record_error(kErrRowOverflow);
            total += kept;
            if (src < rank) before += kept;
        }
        tot[e] = total;
    }
    __syncthreads();
    if (e < n) {
        const int q = e / E;
        int32_t base = 0;  // rows of the owner's earlier local experts
        for (int e2 = q * E; e2 < e; ++e2) base += tot[e2];
        send_base[e] = base + before;
        if (q == rank) recv_offsets[e - q * E] = base;
        if (q == rank && e == q * E + E - 1) recv_offsets[E] = base + total;
    }
}

__global__ void __launch_bounds__(kEpThreads)
ep_dispatch_kernel(const uint4* __restrict__ x, int64_t m, int64_t vec_per_row, int k, int n, int E,
                   const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ dest_row,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ send_base,
                   uint4* const* __restrict__ peers, int64_t max_recv_rows, int32_t* __restrict__ ep_row) {
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kEpThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5); i < m; i += warps) {
        for (int r0 = 0; r0 < k; r0 += 32) {
            // lane t holds pick r0 + t: its owner and its row in the owner's buffer (or -1)
            int32_t row = -1, owner = 0;
            if (r0 + lane < k) {
                const int32_t dr = dest_row[i * k + r0 + lane];
                if (dr >= 0) {
                    const int32_t e = topk_idx[i * k + r0 + lane];
                    if (e < 0 || e >= n) {
                        record_error(kErrExpertIndex);
                    } else {
                        owner = e / E;
                        const int64_t rr = (int64_t)send_base[e] + dr - offsets[e];
                        if (rr < 0 || rr >= max_recv_rows) record_error(kErrRowOverflow);
                        else row = (int32_t)rr;
                    }
                }
                ep_row[i * k + r0 + lane] = row;
            }
            const uint32_t kept = __ballot_sync(0xffffffffu, row >= 0);
            if (!kept) continue;
            const uint4* src = x + i * vec_per_row;
            // the pass count is warp-uniform, so every lane reaches the shuffles below (rows of
            // fewer than 32 vectors leave the upper lanes without columns, not outside the loop)
            for (int64_t cb = 0; cb < vec_per_row; cb += 32 * 8) {
                const int64_t c0 = cb + lane;
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int64_t c = c0 + 32 * u;
                    if (c < vec_per_row) v[u] = src[c];
                }
                uint32_t rest = kept;
                while (rest) {
                    const int b = __ffs(rest) - 1;
                    rest &= rest - 1;
                    const int64_t dr = __shfl_sync(0xffffffffu, row, b);
                    const int q = __shfl_sync(0xffffffffu, owner, b);
                    uint4* dst = peers[q] + dr * vec_per_row;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int64_t c = c0 + 32 * u;
                        if (c < vec_per_row) dst[c] = v[u];
                    }
                }
            }
        }
    }
}

// y[i] = (residual[i]) + sum_r g_ir * out_owner(r)[ep_row[i,r]] (fp32 accumulation, picks in order).
template <typename T>
__global__ void __launch_bounds__(kEpThreads)
ep_combine_kernel(const T* const* __restrict__ peers, const int32_t* __restrict__ ep_row,
                  const int32_t* __restrict__ topk_idx, int n, int E, const float* __restrict__ gate,
                  const T* __restrict__ residual, int64_t m, int k, int d, int gate_bf16, T* __restrict__ y) {
    constexpr int V = Vec16<T>::N;
    const int lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();
    const int nvec = d / V;
    const int64_t warps = (int64_t)gridDim.x * (kEpThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (kEpThreads / 32) + (threadIdx.x >> 5); i < m; i += warps) {
        for (int c = lane; c < nvec; c += 32) {
            float acc[V];
            if (residual) {
                Vec16<T>::load(residual + i * d + (int64_t)c * V, acc);
            } else {
#pragma unroll
                for (int q = 0; q < V; ++q) acc[q] = 0.f;
            }
            for (int r = 0; r < k; ++r) {
                const int32_t row = ep_row[i * k + r];
                if (row < 0) continue;
                const int32_t e = topk_idx[i * k + r];
                if (e < 0 || e >= n) continue;
                float g = gate[i * k + r];
                if (gate_bf16) g = round_to_bf16(g);
                float v[V];
                Vec16<T>::load(peers[e / E] + (int64_t)row * d + (int64_t)c * V, v);
#pragma unroll
                for (int q = 0; q < V; ++q) acc[q] = fmaf(g, v[q], acc[q]);
            }
            Vec16<T>::store(y + i * d + (int64_t)c * V, acc);
        }
    }
}

static unsigned ep_grid(int64_t rows) {
    int64_t blocks = (rows + (kEpThreads / 32) - 1) / (kEpThreads / 32);
    const int64_t cap = (int64_t)kNumSMs * 16;
    if (blocks > cap) blocks = cap;
    return (unsigned)(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_ep_plan(const int32_t* offsets_all, int G, int n, int rank, int32_t* send_base,
                           int32_t* recv_offsets, cudaStream_t stream) {
    ep_plan_kernel<<<1, kMaxExperts, 0, stream>>>(offsets_all, G, n, rank, send_base, recv_offsets);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const void* x, moe_dtype dt, int64_t m, int d, int k, int n, int G,
                               const int32_t* topk_idx, const int32_t* dest_row, const int32_t* offsets,
                               const int32_t* send_base, void* const* peers, int64_t max_recv_rows, int32_t* ep_row,
                               cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    const int64_t vec = (int64_t)d * (dt == MOE_BF16 ? 2 : 4) / 16;
    return launch_pdl(ep_dispatch_kernel, dim3(ep_grid(m)), dim3(kEpThreads), 0, stream,
                      static_cast<const uint4*>(x), m, vec, k, n, n / G, topk_idx, dest_row, offsets, send_base,
                      reinterpret_cast<uint4* const*>(peers), max_recv_rows, ep_row);
}

cudaError_t launch_ep_combine(const void* const* peers, moe_dtype dt, const int32_t* ep_row, const int32_t* topk_idx,
                              int n, int G, const float* gate, const void* residual, int64_t m, int k, int d, void* y,
                              cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    if (dt == MOE_BF16)
        return launch_pdl(ep_combine_kernel<__nv_bfloat16>, dim3(ep_grid(m)), dim3(kEpThreads), 0, stream,
                          reinterpret_cast<const __nv_bfloat16* const*>(peers), ep_row, topk_idx, n, n / G, gate,
                          static_cast<const __nv_bfloat16*>(residual), m, k, d, 1, static_cast<__nv_bfloat16*>(y));
    return launch_pdl(ep_combine_kernel<float>, dim3(ep_grid(m)), dim3(kEpThreads), 0, stream,
                      reinterpret_cast<const float* const*>(peers), ep_row, topk_idx, n, n / G, gate,
                      static_cast<const float*>(residual), m, k, d, 0, static_cast<float*>(y));
}

}  // namespace moe
