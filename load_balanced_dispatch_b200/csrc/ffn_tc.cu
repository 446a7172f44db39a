// ffn_tc.cu -- bf16 expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Switch Transformers paper review (tildalice.io/?p=118), Switch Layer:
// FFN(x) = max(0, x W1 + b1) W2 + b2 per expert. Two launches of one grouped
// GEMM kernel: h = relu(xbuf W1_e^T + b1_e) (bf16), then ybuf = h W2_e^T + b2_e.
//
// Kernel (one CTA per SM, persistent over a device-built tile list):
//   warp 0   TMA producer: 128x64 A tile + BNx64 B tile per stage (128-byte
//            swizzle, K-major), STAGES-deep ring, mbarrier transaction counts.
//   warp 1   MMA issuer (one thread): tcgen05.mma kind::f16 M=128 N=BN K=16,
//            bf16 x bf16 -> fp32 accumulator in TMEM; commit frees the stage.
//   warps 2-5 epilogue: tcgen05.ld 32 columns at a time from the lane quarter
//            the warp may access, + bias, ReLU, bf16, 16-byte stores; rows past
//            the expert's end and columns past N are masked.
// Two TMEM accumulators (2 x BN fp32 columns) let the epilogue of tile t
// overlap the MMAs of tile t+1. Every wait is bounded: a timed-out wait sets
// the device error word and an abort flag, and all roles leave their loops.
// The A rows of a tile may run past its expert into the next expert's rows or
// past the buffer (TMA zero fill); those rows are computed and never stored.
#include "groups.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace tc {
constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int kThreads = 192;
constexpr int A_BYTES = BM * BK * 2;
template <int BN> struct Cfg {
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN);
};
struct Shared {
    uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2];
    uint32_t tmem_base;
    int abort_flag;
    GroupTable g;
};
template <int BN>
constexpr size_t smem_bytes() { return 1024 + (size_t)STAGES * Cfg<BN>::STAGE_BYTES + sizeof(Shared); }
}  // namespace tc

template <int BN, bool RELU>
__global__ void __launch_bounds__(tc::kThreads, 1)
ffn_gemm_tc(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
            const __nv_bfloat16* __restrict__ bias, const int32_t* __restrict__ offsets, int n, int N, int K,
            int64_t max_rows, __nv_bfloat16* __restrict__ out) {
    using namespace tc;
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Shared* sh = reinterpret_cast<Shared*>(smem + STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntn = (N + BN - 1) / BN;
    const int nkb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { ptx::mbar_init(&sh->full[s], 1); ptx::mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < 2; ++b) { ptx::mbar_init(&sh->tfull[b], 1); ptx::mbar_init(&sh->tempty[b], 128); }
        sh->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::prefetch_tensormap(&map_a);
        ptx::prefetch_tensormap(&map_b);
    }
    if (warp == 1) ptx::tmem_alloc(&sh->tmem_base, C::TMEM_COLS);
    if (warp == 2) build_group_table(offsets, n, ntn, BM, max_rows, sh->g);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = sh->tmem_base;
    const int total = sh->g.tile_start[n];
    volatile int* abort_flag = &sh->abort_flag;

    // tile -> (expert, row tile, column tile); row tiles vary fastest so neighbouring CTAs share B tiles in L2
    auto decode = [&](int tile, int& e, int64_t& row0, int64_t& row_end, int& n0) {
        e = group_of_tile(sh->g, n, tile);
        const int local = tile - sh->g.tile_start[e];
        const int rows_e = sh->g.row_start[e + 1] - sh->g.row_start[e];
        const int mtiles = (rows_e + BM - 1) / BM;
        const int nt = local / mtiles, mt = local - nt * mtiles;
        row0 = (int64_t)sh->g.row_start[e] + (int64_t)mt * BM;
        row_end = sh->g.row_start[e + 1];
        n0 = nt * BN;
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                int e, n0;
                int64_t row0, row_end;
                decode(tile, e, row0, row_end, n0);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + stage * C::STAGE_BYTES;
                    ptx::mbar_expect_tx(&sh->full[stage], C::STAGE_BYTES);
                    ptx::tma_load_2d(sa, &map_a, &sh->full[stage], kb * BK, (int)row0);
                    ptx::tma_load_3d(sa + A_BYTES, &map_b, &sh->full[stage], kb * BK, n0, e);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, aphase = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
                if (!ptx::mbar_wait(&sh->tempty[acc], aphase ^ 1u, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t tmem_d = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&sh->full[stage], phase, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint64_t adesc = ptx::sw128_kmajor_desc(sa);
                    const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)  // K step of 16 bf16 = 32 bytes = 2 descriptor units
                        ptx::umma_bf16(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, C::IDESC, (kb | kk) != 0);
                    ptx::umma_commit(&sh->empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::umma_commit(&sh->tfull[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1u; }
            }
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows 32*(w%4) + lane
        const int quad = warp & 3;
        int acc = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int e, n0;
            int64_t row0, row_end;
            decode(tile, e, row0, row_end, n0);
            if (!ptx::mbar_wait(&sh->tfull[acc], aphase, abort_flag)) break;
            ptx::tc_fence_after();
            const int64_t r = row0 + quad * 32 + lane;
            const bool row_ok = r < row_end;
            const __nv_bfloat16* be = bias + (int64_t)e * N;
            for (int c = 0; c < BN / 32; ++c) {
                const int col0 = n0 + c * 32;
                if (col0 >= N) break;  // warp-uniform
                uint32_t v[32];
                ptx::tmem_ld32(tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN + c * 32), v);
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    const int col = col0 + g8 * 8;
                    if (col >= N) break;
                    float f[8], bv[8];
                    Vec16<__nv_bfloat16>::load(be + col, bv);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        f[q] = __uint_as_float(v[g8 * 8 + q]) + bv[q];
                        if (RELU) f[q] = fmaxf(f[q], 0.f);
                    }
                    if (row_ok) Vec16<__nv_bfloat16>::store(out + r * N + col, f);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sh->tempty[acc]);
            if (++acc == 2) { acc = 0; aphase ^= 1u; }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace moe

// ------------------------------------------------------------------ host side
namespace moe {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 [rows, cols] row-major, box [box_rows, 64], 128-byte swizzle
static bool map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [groups, rows, cols] row-major, box [1, box_rows, 64], 128-byte swizzle
static bool map_3d(CUtensorMap* m, const void* base, uint64_t groups, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {cols, rows, groups};
    cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = kNumSMs;
    }
    return sms;
}

template <int BN, bool RELU>
static cudaError_t launch_gemm_tc(const void* A, const void* B, const void* bias, const int32_t* offsets, int n,
                                  int N, int K, int64_t max_rows, void* out, cudaStream_t stream) {
    CUtensorMap ma, mb;
    if (!map_2d(&ma, A, (uint64_t)max_rows, (uint64_t)K, tc::BM)) return cudaErrorInvalidValue;
    if (!map_3d(&mb, B, (uint64_t)n, (uint64_t)N, (uint64_t)K, BN)) return cudaErrorInvalidValue;
    static bool attr_set = false;
    const size_t smem = tc::smem_bytes<BN>();
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(ffn_gemm_tc<BN, RELU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    ffn_gemm_tc<BN, RELU><<<num_sms(), tc::kThreads, smem, stream>>>(
        ma, mb, static_cast<const __nv_bfloat16*>(bias), offsets, n, N, K, max_rows,
        static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
}

cudaError_t launch_ffn_fused(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                             const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                             int* done1, cudaStream_t stream);

// Both GEMMs in one persistent launch; the per-expert completion counters follow h in the workspace.
cudaError_t launch_ffn_tc(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                          const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                          cudaStream_t stream) {
    const size_t hbytes = ((size_t)max_rows * (size_t)d_ff * 2 + 255) & ~(size_t)255;
    int* done1 = reinterpret_cast<int*>(static_cast<char*>(hbuf) + hbytes);
    return launch_ffn_fused(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, done1, stream);
}

}  // namespace moe
