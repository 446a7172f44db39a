// ffn_simt.cu -- expert FFN with fp32 FMAs (the fp32 layer path).
//
// Switch Transformers paper review (tildalice.io/?p=118), Switch Layer:
// FFN(x) = max(0, x W1 + b1) W2 + b2 with one weight set per expert.
//
// A grouped GEMM C_e = A_e B_e^T (+ bias, optional ReLU) over the expert-major
// rows: the group sizes live on the device (expert_offsets), so every CTA
// rebuilds the tile list from them in shared memory and strides over it -- no
// host synchronisation. 64x64 output tiles, 256 threads with 4x4 register
// tiles, K-tiles of 16 staged in shared memory. fp32 inputs stay fp32 (a
// tensor-core tf32 path would miss the fp32 tolerance).
#include "common.cuh"
#include "groups.cuh"

namespace moe {

namespace simt {
constexpr int BM = 64, BN = 64, BK = 16, kThreads = 256;
constexpr int PAD = 4;
}  // namespace simt

template <typename T, bool RELU>
__global__ void __launch_bounds__(simt::kThreads)
grouped_gemm_simt(const T* __restrict__ A, const T* __restrict__ B, const T* __restrict__ bias,
                  const int32_t* __restrict__ offsets, int n, int N, int K, int64_t max_rows, T* __restrict__ Cout) {
    using namespace simt;
    __shared__ GroupTable g;
    __shared__ __align__(16) float As[BK][BM + PAD];
    __shared__ __align__(16) float Bs[BK][BN + PAD];
    const int tid = threadIdx.x;
    const int ntn = (N + BN - 1) / BN;
    if (tid < 32) build_group_table(offsets, n, ntn, BM, max_rows, g);
    __syncthreads();
    const int total = g.tile_start[n];
    const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads, each 4 x 4 outputs
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int e = group_of_tile(g, n, tile);
        const int local = tile - g.tile_start[e];
        const int mt = local / ntn, nt = local - mt * ntn;
        const int64_t row0 = (int64_t)g.row_start[e] + (int64_t)mt * BM;
        const int64_t row_end = min((int64_t)g.row_start[e + 1], (int64_t)max_rows);
        const int col0 = nt * BN;
        const T* Be = B + (int64_t)e * N * K;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int k0 = 0; k0 < K; k0 += BK) {
            // 64 x 16 tiles of A and B: thread loads 4 elements of each (row tid/4, k-run (tid%4)*4)
            const int lr = tid >> 2, lk = (tid & 3) * 4;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int kk = k0 + lk + q;
                const int64_t ar = row0 + lr;
                As[lk + q][lr] = (ar < row_end && kk < K) ? Elem<T>::load(A + ar * K + kk) : 0.f;
                const int bc = col0 + lr;
                Bs[lk + q][lr] = (bc < N && kk < K) ? Elem<T>::load(Be + (int64_t)bc * K + kk) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < BK; ++kk) {
                const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
                const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
                const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t r = row0 + ty * 4 + i;
            if (r >= row_end) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = col0 + tx * 4 + j;
                if (c >= N) continue;
                float v = acc[i][j] + Elem<T>::load(bias + (int64_t)e * N + c);
                if (RELU) v = fmaxf(v, 0.f);
                Elem<T>::store(Cout + r * N + c, v);
            }
        }
    }
}

template <typename T>
static cudaError_t launch_ffn_simt_t(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                                     const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf,
                                     void* hbuf, cudaStream_t stream) {
    const unsigned grid = kNumSMs * 4;
    grouped_gemm_simt<T, true><<<grid, simt::kThreads, 0, stream>>>(
        static_cast<const T*>(xbuf), static_cast<const T*>(w1), static_cast<const T*>(b1), offsets, n, d_ff, d,
        max_rows, static_cast<T*>(hbuf));
    grouped_gemm_simt<T, false><<<grid, simt::kThreads, 0, stream>>>(
        static_cast<const T*>(hbuf), static_cast<const T*>(w2), static_cast<const T*>(b2), offsets, n, d, d_ff,
        max_rows, static_cast<T*>(ybuf));
    return cudaGetLastError();
}

cudaError_t launch_ffn_simt(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                            const void* b2, const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows,
                            void* ybuf, void* hbuf, cudaStream_t stream) {
    if (dt == MOE_BF16)
        return launch_ffn_simt_t<__nv_bfloat16>(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf,
                                                stream);
    return launch_ffn_simt_t<float>(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, stream);
}

}  // namespace moe
