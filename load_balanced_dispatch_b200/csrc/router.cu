// router.cu -- router projection h = x W_r (fp32), score function, top-k and gates.
//
// Switch Transformers paper review (tildalice.io/?p=118), Switch Routing Steps
// 1-3 with selective precision (projection and softmax in fp32); the Shazeer
// gate Softmax(TopK(.)) for k >= 2; MoE travelogue 6 (kexue.fm/archives/11619)
// eq. (1): a Loss-Free bias enters the ranking only.
//
// One CTA computes the fp32 logits of TM tokens against all n <= 256 experts
// with SIMT FMAs (K-tiles of x and W_r staged in shared memory), parks the
// logit tile in shared memory, and one warp per token row finishes the row in
// registers: max/exp/sum (softmax) or the logistic function, the ranking key,
// k rounds of a warp arg-max (ties -> lower index) and the gates. Logits never
// reach HBM.
#include "common.cuh"

namespace moe {

namespace router {
constexpr int TM = 32;       // tokens per CTA
constexpr int TK = 32;       // K-tile
constexpr int XS = TM + 1;   // padded stride of the transposed x tile
constexpr int kThreads = 256;
}  // namespace router

template <typename T>
__device__ __forceinline__ void load4(const T* p, int64_t avail, float* out);
template <>
__device__ __forceinline__ void load4<float>(const float* p, int64_t avail, float* out) {
    if (avail >= 4 && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) out[q] = q < avail ? p[q] : 0.f;
    }
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, int64_t avail, float* out) {
    if (avail >= 4 && (reinterpret_cast<uintptr_t>(p) & 7) == 0) {
        uint2 v = *reinterpret_cast<const uint2*>(p);
        out[0] = __uint_as_float(v.x << 16); out[1] = __uint_as_float(v.x & 0xffff0000u);
        out[2] = __uint_as_float(v.y << 16); out[3] = __uint_as_float(v.y & 0xffff0000u);
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) out[q] = q < avail ? __bfloat162float(p[q]) : 0.f;
    }
}

// Finish one token row held by a warp: lane owns experts j = lane + 32 q (q < NT).
template <int NT>
__device__ __forceinline__ void finish_row(const float (&h)[NT], int64_t row, int n, int k, int fn, int renorm,
                                           const float* rank_bias, float* probs_out, int32_t* topk_idx,
                                           float* topk_gate) {
    const int lane = threadIdx.x & 31;
    float p[NT], key[NT];
    if (fn == MOE_SOFTMAX) {
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < NT; ++q) if (lane + 32 * q < n) mx = fmaxf(mx, h[q]);
        mx = warp_max(mx);
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            p[q] = (lane + 32 * q < n) ? expf(h[q] - mx) : 0.f;
            s += p[q];
        }
        s = warp_sum(s);
#pragma unroll
        for (int q = 0; q < NT; ++q) p[q] = p[q] / s;
    } else {
#pragma unroll
        for (int q = 0; q < NT; ++q) p[q] = 1.f / (1.f + expf(-h[q]));
    }
#pragma unroll
    for (int q = 0; q < NT; ++q) {
        const int j = lane + 32 * q;
        if (j >= n) { key[q] = -INFINITY; continue; }
        if (rank_bias) key[q] = __fadd_rn(p[q], rank_bias[j]);
        else key[q] = (fn == MOE_SOFTMAX) ? h[q] : p[q];
    }
    if (probs_out) {
#pragma unroll
        for (int q = 0; q < NT; ++q)
            if (lane + 32 * q < n) probs_out[row * n + lane + 32 * q] = p[q];
    }
    uint32_t taken = 0;
    float selsum = 0.f;
    float mysel_p = 0.f;   // lane r (< k) keeps the score of pick r
    int mysel_i = 0;
    for (int r = 0; r < k; ++r) {
        float bk = -INFINITY;
        int bi = 0x7fffffff;
        float bp = 0.f;
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const int j = lane + 32 * q;
            if (j < n && !(taken & (1u << q)) && ranks_before(key[q], j, bk, bi)) { bk = key[q]; bi = j; bp = p[q]; }
        }
        float wk = bk;
        int wi = bi;
        warp_best(wk, wi);
        const int owner = wi & 31;
        if (lane == owner && wi < n) taken |= 1u << (wi >> 5);
        const float wp = __shfl_sync(0xffffffffu, bp, owner);
        selsum += wp;
        if (r < 32 && lane == r) { mysel_p = wp; mysel_i = wi; }
        if (r >= 32 && lane == 0) {  // k > 32: write picks beyond the first 32 as they come
            topk_idx[row * k + r] = wi;
            topk_gate[row * k + r] = wp;  // divided by the selected sum below when renormalising
        }
    }
    if (lane < k && lane < 32) {
        topk_idx[row * k + lane] = mysel_i;
        topk_gate[row * k + lane] = (fn == MOE_SOFTMAX && renorm) ? mysel_p / selsum : mysel_p;
    }
    if (k > 32 && fn == MOE_SOFTMAX && renorm) {
        __syncwarp();
        for (int r = 32 + lane; r < k; r += 32) topk_gate[row * k + r] = topk_gate[row * k + r] / selsum;
    }
}

// One row finished by one thread from its n <= NV logits in registers v (k <= K): the operations of
// finish_row, except that the softmax sum adds the terms in expert order (not a warp tree). The
// K best (key, expert, score) are kept sorted while the experts are scanned in ascending order; a
// key enters only if it beats the K-th kept one, so ties keep the lower index.
// v is overwritten with the scores.
template <int NV, int K>
__device__ __forceinline__ void finish_row_thread(float (&v)[NV], int64_t row, int n, int k, int fn, int renorm,
                                                  const float* rank_bias, float* probs_out, int32_t* topk_idx,
                                                  float* topk_gate) {
    float tk[K], tp[K];
    int ti[K];
#pragma unroll
    for (int q = 0; q < K; ++q) { tk[q] = -INFINITY; tp[q] = 0.f; ti[q] = 0; }
    auto offer = [&](float key, int j, float pj) {
        if (key > tk[K - 1]) {
#pragma unroll
            for (int q = K - 1; q > 0; --q) {
                if (key > tk[q - 1]) { tk[q] = tk[q - 1]; ti[q] = ti[q - 1]; tp[q] = tp[q - 1]; }
                else if (key > tk[q]) { tk[q] = key; ti[q] = j; tp[q] = pj; }
            }
            if (key > tk[0]) { tk[0] = key; ti[0] = j; tp[0] = pj; }
        }
    };
    if (fn == MOE_SOFTMAX) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < NV; ++j) if (j < n) mx = fmaxf(mx, v[j]);
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const float e = j < n ? expf(v[j] - mx) : 0.f;
            if (!rank_bias && j < n) offer(v[j], j, e);  // the logit ranks; the score is divided below
            v[j] = e;
            s += e;
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) v[j] = v[j] / s;
        if (rank_bias) {
#pragma unroll
            for (int j = 0; j < NV; ++j) if (j < n) offer(__fadd_rn(v[j], __ldg(rank_bias + j)), j, v[j]);
        } else {
#pragma unroll
            for (int q = 0; q < K; ++q) tp[q] = tp[q] / s;
        }
    } else {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            v[j] = 1.f / (1.f + expf(-v[j]));
            if (j < n) offer(rank_bias ? __fadd_rn(v[j], __ldg(rank_bias + j)) : v[j], j, v[j]);
        }
    }
    if (probs_out) {
        float* pr = probs_out + row * n;
        if ((n & 3) == 0 && (reinterpret_cast<uintptr_t>(probs_out) & 15) == 0) {
#pragma unroll
            for (int c = 0; c < NV / 4; ++c)
                if (4 * c < n)
                    *reinterpret_cast<float4*>(pr + 4 * c) = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) if (j < n) pr[j] = v[j];
        }
    }
    float selsum = 0.f;
#pragma unroll
    for (int q = 0; q < K; ++q) if (q < k) selsum += tp[q];
    const bool rn = fn == MOE_SOFTMAX && renorm;
#pragma unroll
    for (int q = 0; q < K; ++q)
        if (q < k) {
            topk_idx[row * k + q] = ti[q];
            topk_gate[row * k + q] = rn ? tp[q] / selsum : tp[q];
        }
}

template <typename T, int NT>
__global__ void __launch_bounds__(router::kThreads)
router_topk_kernel(const T* __restrict__ x, const float* __restrict__ w_r, const float* __restrict__ logits_in,
                   int64_t m, int d, int n, int k, int fn, int renorm, const float* __restrict__ rank_bias,
                   float* __restrict__ probs_out, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate) {
    using namespace router;
    constexpr int NPAD = 32 * NT;
    __shared__ __align__(16) float smem[(TK * XS + TK * NPAD) > (TM * (NPAD + 1)) ? (TK * XS + TK * NPAD)
                                                                                   : (TM * (NPAD + 1))];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row0 = (int64_t)blockIdx.x * TM;

    if (logits_in) {
        for (int rr = warp; rr < TM; rr += kThreads / 32) {
            const int64_t row = row0 + rr;
            if (row >= m) break;
            float h[NT];
#pragma unroll
            for (int q = 0; q < NT; ++q) h[q] = (lane + 32 * q < n) ? logits_in[row * n + lane + 32 * q] : 0.f;
            finish_row<NT>(h, row, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
        }
        return;
    }

    float* xs = smem;              // [TK][XS]: x tile transposed (k-major)
    float* ws = smem + TK * XS;    // [TK][NPAD]
    const int tx = lane, ty = warp;  // thread computes tokens ty*4 .. ty*4+3, experts tx + 32 q
    float acc[4][NT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < NT; ++q) acc[i][q] = 0.f;

    const int lr = tid >> 3, lc = tid & 7;  // x tile loader: row lr, k-chunk lc (4 elements)
    for (int k0 = 0; k0 < d; k0 += TK) {
        {
            const int64_t gr = row0 + lr;
            const int gk = k0 + lc * 4;
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            if (gr < m && gk < d) load4<T>(x + gr * d + gk, d - gk, v);
#pragma unroll
            for (int q = 0; q < 4; ++q) xs[(lc * 4 + q) * XS + lr] = v[q];
        }
        for (int e = tid; e < TK * NPAD; e += kThreads) {
            const int kk = e / NPAD, j = e - kk * NPAD;
            const int gk = k0 + kk;
            ws[e] = (gk < d && j < n) ? w_r[(int64_t)gk * n + j] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float xv[4], wv[NT];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[kk * XS + ty * 4 + i];
#pragma unroll
            for (int q = 0; q < NT; ++q) wv[q] = ws[kk * NPAD + tx + 32 * q];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < NT; ++q) acc[i][q] = fmaf(xv[i], wv[q], acc[i][q]);
        }
        __syncthreads();
    }
    float* lg = smem;  // [TM][NPAD+1]
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < NT; ++q) lg[(ty * 4 + i) * (NPAD + 1) + tx + 32 * q] = acc[i][q];
    __syncthreads();
    for (int rr = warp; rr < TM; rr += kThreads / 32) {
        const int64_t row = row0 + rr;
        if (row >= m) break;
        float h[NT];
#pragma unroll
        for (int q = 0; q < NT; ++q) h[q] = lg[rr * (NPAD + 1) + lane + 32 * q];
        finish_row<NT>(h, row, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    }
}

// Finish rows whose fp32 logits are already in memory: h [m, n]. `probs_out` may be h itself
// (each warp loads its whole row into registers before writing any of it), so neither pointer
// is declared restrict. One warp per row, grid-stride over rows.
constexpr int kFinishThreads = 256;
template <int NT>
__global__ void __launch_bounds__(kFinishThreads)
router_finish_kernel(const float* h, int64_t m, int n, int k, int fn, int renorm, const float* __restrict__ rank_bias,
                     float* probs_out, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate) {
    const int lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();
    const int64_t warps = (int64_t)gridDim.x * (kFinishThreads / 32);
    // the next row's logits are loaded before this row is finished (one row in flight ahead)
    int64_t row = (int64_t)blockIdx.x * (kFinishThreads / 32) + (threadIdx.x >> 5);
    float hv[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) hv[q] = (row < m && lane + 32 * q < n) ? h[row * n + lane + 32 * q] : 0.f;
    for (; row < m; row += warps) {
        const int64_t nr = row + warps;
        float nx[NT];
#pragma unroll
        for (int q = 0; q < NT; ++q) nx[q] = (nr < m && lane + 32 * q < n) ? h[nr * n + lane + 32 * q] : 0.f;
        __syncwarp();
        finish_row<NT>(hv, row, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
#pragma unroll
        for (int q = 0; q < NT; ++q) hv[q] = nx[q];
    }
}

cudaError_t launch_router_finish(const float* h, int64_t m, int n, int k, int fn, int renorm, const float* rank_bias,
                                 float* probs_out, int32_t* topk_idx, float* topk_gate, cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    int64_t blocks = (m + kFinishThreads / 32 - 1) / (kFinishThreads / 32);
    const int64_t cap = (int64_t)kNumSMs * 8;
    if (blocks > cap) blocks = cap;
    if (n <= 32)
        return launch_pdl(router_finish_kernel<1>, dim3((unsigned)blocks), dim3(kFinishThreads), 0, stream, h, m, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    else if (n <= 64)
        return launch_pdl(router_finish_kernel<2>, dim3((unsigned)blocks), dim3(kFinishThreads), 0, stream, h, m, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    else if (n <= 128)
        return launch_pdl(router_finish_kernel<4>, dim3((unsigned)blocks), dim3(kFinishThreads), 0, stream, h, m, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    else
        return launch_pdl(router_finish_kernel<8>, dim3((unsigned)blocks), dim3(kFinishThreads), 0, stream, h, m, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    return cudaGetLastError();
}

template <typename T, int NT>
static cudaError_t launch_router_t(const void* x, const float* w_r, const float* logits_in, int64_t m, int d, int n,
                                   int k, int fn, int renorm, const float* rank_bias, float* probs_out,
                                   int32_t* topk_idx, float* topk_gate, cudaStream_t stream) {
    const int64_t blocks = (m + router::TM - 1) / router::TM;
    if (blocks == 0) return cudaSuccess;
    router_topk_kernel<T, NT><<<(unsigned)blocks, router::kThreads, 0, stream>>>(
        static_cast<const T*>(x), w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_router_dt(const void* x, const float* w_r, const float* logits_in, int64_t m, int d, int n,
                                    int k, int fn, int renorm, const float* rank_bias, float* probs_out,
                                    int32_t* topk_idx, float* topk_gate, cudaStream_t stream) {
    if (n <= 32) return launch_router_t<T, 1>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
    if (n <= 64) return launch_router_t<T, 2>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
    if (n <= 128) return launch_router_t<T, 4>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
    return launch_router_t<T, 8>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
}

cudaError_t launch_router_tc(const void* x, const float* w_r, int64_t m, int d, int n, int k, int fn, int renorm,
                             const float* rank_bias, float* probs_out, int32_t* topk_idx, float* topk_gate,
                             void* workspace, cudaStream_t stream);

// bf16 activations projected on the tensor cores (W_r split into three bf16 parts) when the
// expert row fits the register drain (n <= 128); fp32 activations, given logits or n > 128 use the
// FMA kernel.
bool router_tc_supported(int n, int k);
bool router_uses_tc(moe_dtype dt, const float* logits_in, int n, int k) {
    return dt == MOE_BF16 && !logits_in && router_tc_supported(n, k);
}

cudaError_t launch_router(const void* x, moe_dtype dt, const float* w_r, const float* logits_in, int64_t m, int d,
                          int n, int k, int fn, int renorm, const float* rank_bias, float* probs_out,
                          int32_t* topk_idx, float* topk_gate, void* workspace, cudaStream_t stream) {
    if (router_uses_tc(dt, logits_in, n, k))
        return launch_router_tc(x, w_r, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, workspace,
                                stream);
    if (dt == MOE_BF16)
        return launch_router_dt<__nv_bfloat16>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out,
                                               topk_idx, topk_gate, stream);
    return launch_router_dt<float>(x, w_r, logits_in, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx,
                                   topk_gate, stream);
}

}  // namespace moe
