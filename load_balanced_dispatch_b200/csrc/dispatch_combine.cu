// dispatch_combine.cu -- the two permutations of the layer and the gated combine.
//
// Switch Transformer read for implementation (molayo1419.me): the forward pass
// changes token order twice -- group tokens by expert before the FFN, restore
// token order after it, multiply by the gate and join the residual path;
// overflow tokens keep only the residual. Switch Transformers paper review
// (tildalice.io/?p=118), Step 3: y = p_i* E_i*(x).
//
// All kernels are HBM-bound row copies: one warp per row (or per token), 16-byte
// vectors, grid sized to a multiple of the SM count and striding over rows.
#include "common.cuh"

namespace moe {

constexpr int kRowThreads = 256;

static unsigned row_grid(int64_t rows) {
    const int64_t per_block = kRowThreads / 32;
    int64_t blocks = (rows + per_block - 1) / per_block;
    const int64_t cap = (int64_t)kNumSMs * 16;
    if (blocks > cap) blocks = cap;
    return (unsigned)(blocks < 1 ? 1 : blocks);
}

// xbuf[r] = x[src_token[r]] for r < expert_offsets[n]; raw 16-byte copies.
__global__ void __launch_bounds__(kRowThreads)
dispatch_kernel(const uint4* __restrict__ x, int64_t m, int64_t vec_per_row, const int32_t* __restrict__ src_token,
                const int32_t* __restrict__ expert_offsets, int n, int64_t max_rows, uint4* __restrict__ xbuf) {
    pdl_trigger();
    pdl_wait();
    int64_t rows = expert_offsets[n];
    if (rows > max_rows) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_error(kErrRowOverflow);
        rows = max_rows;
    }
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kRowThreads / 32);
    for (int64_t r = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int32_t t = src_token[r];
        if (t < 0 || t >= m) {
            if (lane == 0) record_error(kErrTokenIndex);
            continue;
        }
        const uint4* src = x + (int64_t)t * vec_per_row;
        uint4* dst = xbuf + r * vec_per_row;
        // up to 8 independent 16-byte loads in flight per lane before the stores
        for (int64_t c0 = lane; c0 < vec_per_row; c0 += 32 * 8) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t c = c0 + 32 * u;
                if (c < vec_per_row) v[u] = src[c];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t c = c0 + 32 * u;
                if (c < vec_per_row) dst[c] = v[u];
            }
        }
    }
}

// Token-major dispatch: xbuf[dest_row[i, r]] = x[i] for every kept pick (dest_row >= 0). Each
// token's row is read from HBM once, whatever the number of its kept picks, and written to each
// of its rows: the same xbuf as dispatch_kernel (the kept rows are exactly rows 0 .. rows-1).
// One warp per token; a lane moves 16-byte vectors, eight loads in flight before the stores.
__global__ void __launch_bounds__(kRowThreads)
dispatch_tokens_kernel(const uint4* __restrict__ x, int64_t m, int64_t vec_per_row, int k,
                       const int32_t* __restrict__ dest_row, int64_t max_rows, uint4* __restrict__ xbuf) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kRowThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); i < m; i += warps) {
        // the token's kept rows, gathered into lanes 0 .. nk-1 (k <= 32 per pass of picks)
        for (int r0 = 0; r0 < k; r0 += 32) {
            int32_t row = -1;
            if (r0 + lane < k) row = dest_row[i * k + r0 + lane];
            if (row >= max_rows) {
                record_error(kErrRowOverflow);
                row = -1;
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
                    uint4* dst = xbuf + dr * vec_per_row;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int64_t c = c0 + 32 * u;
                        if (c < vec_per_row) dst[c] = v[u];
                    }
                }
            }
        }
    }
    pdl_trigger();  // after this CTA's rows: the dependent launch starts as the grid drains
}

// y[i] = (residual[i]) + sum_r g_ir * ybuf[dest_row[i,r]]  (fp32 accumulation).
template <typename T>
__global__ void __launch_bounds__(kRowThreads)
combine_kernel(const T* __restrict__ ybuf, const int32_t* __restrict__ dest_row, const float* __restrict__ gate,
               const T* __restrict__ residual, int64_t m, int k, int d, int gate_bf16, T* __restrict__ y) {
    constexpr int V = Vec16<T>::N;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    const int nvec = d / V;
    const int64_t warps = (int64_t)gridDim.x * (kRowThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); i < m; i += warps) {
        // two 16-byte column chunks per lane at a time: their k row loads are independent
        for (int c0 = lane; c0 < nvec; c0 += 64) {
            const int c1 = c0 + 32;
            const bool has1 = c1 < nvec;
            float acc0[V], acc1[V];
            if (residual) {
                Vec16<T>::load(residual + i * d + (int64_t)c0 * V, acc0);
                if (has1) Vec16<T>::load(residual + i * d + (int64_t)c1 * V, acc1);
            } else {
#pragma unroll
                for (int q = 0; q < V; ++q) { acc0[q] = 0.f; acc1[q] = 0.f; }
            }
            for (int r = 0; r < k; ++r) {
                const int32_t row = dest_row[i * k + r];
                if (row < 0) continue;
                float g = gate[i * k + r];
                if (gate_bf16) g = round_to_bf16(g);
                float v0[V], v1[V];
                const T* yr = ybuf + (int64_t)row * d;
                Vec16<T>::load(yr + (int64_t)c0 * V, v0);
                if (has1) Vec16<T>::load(yr + (int64_t)c1 * V, v1);
#pragma unroll
                for (int q = 0; q < V; ++q) {
                    acc0[q] = fmaf(g, v0[q], acc0[q]);
                    if (has1) acc1[q] = fmaf(g, v1[q], acc1[q]);
                }
            }
            Vec16<T>::store(y + i * d + (int64_t)c0 * V, acc0);
            if (has1) Vec16<T>::store(y + i * d + (int64_t)c1 * V, acc1);
        }
    }
    pdl_trigger();  // after this CTA's tokens: the dependent launch starts as the grid drains
}

// The same combine for k <= KMAX: a token's rows and gates are read once (lane r holds pick r's),
// and each pass covers U 16-byte column chunks per lane with every kept row's loads issued before
// the adds (the adds in pick order, as above: the same bits).
template <typename T, int KMAX, int U>
__global__ void __launch_bounds__(kRowThreads)
combine_rows_kernel(const T* __restrict__ ybuf, const int32_t* __restrict__ dest_row, const float* __restrict__ gate,
                    const T* __restrict__ residual, int64_t m, int k, int d, int gate_bf16, T* __restrict__ y) {
    constexpr int V = Vec16<T>::N;
    const int lane = threadIdx.x & 31;
    pdl_wait();
    const int nvec = d / V;
    const int64_t warps = (int64_t)gridDim.x * (kRowThreads / 32);
    for (int64_t i = (int64_t)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); i < m; i += warps) {
        int32_t myrow = -1;
        float myg = 0.f;
        if (lane < k) {
            myrow = dest_row[i * k + lane];
            myg = gate[i * k + lane];
            if (gate_bf16) myg = round_to_bf16(myg);
        }
        int32_t rows[KMAX];
        float gs[KMAX];
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
            rows[r] = __shfl_sync(0xffffffffu, myrow, r);
            gs[r] = __shfl_sync(0xffffffffu, myg, r);
        }
        for (int c0 = lane; c0 < nvec; c0 += 32 * U) {
            float acc[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (residual && c < nvec) {
                    Vec16<T>::load(residual + i * d + (int64_t)c * V, acc[u]);
                } else {
#pragma unroll
                    for (int q = 0; q < V; ++q) acc[u][q] = 0.f;
                }
            }
            uint4 raw[KMAX][U];
#pragma unroll
            for (int r = 0; r < KMAX; ++r)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + 32 * u;
                    if (r < k && rows[r] >= 0 && c < nvec)
                        raw[r][u] = *reinterpret_cast<const uint4*>(ybuf + (int64_t)rows[r] * d + (int64_t)c * V);
                }
#pragma unroll
            for (int r = 0; r < KMAX; ++r) {
                if (r >= k || rows[r] < 0) continue;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    float v[V];
                    Vec16<T>::load(reinterpret_cast<const T*>(&raw[r][u]), v);
#pragma unroll
                    for (int q = 0; q < V; ++q) acc[u][q] = fmaf(gs[r], v[q], acc[u][q]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (c < nvec) Vec16<T>::store(y + i * d + (int64_t)c * V, acc[u]);
            }
        }
    }
    pdl_trigger();
}

cudaError_t launch_dispatch(const void* x, moe_dtype dt, int64_t m, int d, const int32_t* src_token,
                            const int32_t* expert_offsets, int n, int64_t max_rows, void* xbuf,
                            cudaStream_t stream) {
    const int64_t bytes_per_row = (int64_t)d * (dt == MOE_BF16 ? 2 : 4);
    return launch_pdl(dispatch_kernel, dim3(row_grid(max_rows)), dim3(kRowThreads), 0, stream,
                      static_cast<const uint4*>(x), m, bytes_per_row / 16, src_token, expert_offsets, n, max_rows,
                      static_cast<uint4*>(xbuf));
}

cudaError_t launch_dispatch_tokens(const void* x, moe_dtype dt, int64_t m, int d, int k, const int32_t* dest_row,
                                   int64_t max_rows, void* xbuf, cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    const int64_t bytes_per_row = (int64_t)d * (dt == MOE_BF16 ? 2 : 4);
    return launch_pdl(dispatch_tokens_kernel, dim3(row_grid(m)), dim3(kRowThreads), 0, stream,
                      static_cast<const uint4*>(x), m, bytes_per_row / 16, k, dest_row, max_rows,
                      static_cast<uint4*>(xbuf));
}

cudaError_t launch_combine(const void* ybuf, moe_dtype dt, const int32_t* dest_row, const float* topk_gate,
                           const void* residual, int64_t m, int k, int d, void* y, cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    if (dt == MOE_BF16 && k <= 8) {
        // two chunks per lane per pass: 155.6 us at 65536 x 4096, k = 2, against 169.7 us for
        // combine_kernel and 187.7 us with four chunks per pass
#define MOE_COMBINE_ROWS(KM)                                                                                     \
    return launch_pdl(combine_rows_kernel<__nv_bfloat16, KM, 2>, dim3(row_grid(m)), dim3(kRowThreads), 0, stream, \
                      static_cast<const __nv_bfloat16*>(ybuf), dest_row, topk_gate,                             \
                      static_cast<const __nv_bfloat16*>(residual), m, k, d, 1, static_cast<__nv_bfloat16*>(y))
        if (k <= 2) MOE_COMBINE_ROWS(2);
        if (k <= 4) MOE_COMBINE_ROWS(4);
        MOE_COMBINE_ROWS(8);
#undef MOE_COMBINE_ROWS
    }
    if (dt == MOE_BF16) {
        return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(row_grid(m)), dim3(kRowThreads), 0, stream,
                          static_cast<const __nv_bfloat16*>(ybuf), dest_row, topk_gate,
                          static_cast<const __nv_bfloat16*>(residual), m, k, d, 1, static_cast<__nv_bfloat16*>(y));
    }
    return launch_pdl(combine_kernel<float>, dim3(row_grid(m)), dim3(kRowThreads), 0, stream,
                      static_cast<const float*>(ybuf), dest_row, topk_gate, static_cast<const float*>(residual), m, k,
                      d, 0, static_cast<float*>(y));
}

}  // namespace moe
