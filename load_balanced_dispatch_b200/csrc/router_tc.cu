// router_tc.cu -- fp32-accurate router projection on the bf16 tensor cores, then the
// score function, ranking and top-k.
//
// Switch Transformers paper review (tildalice.io/?p=118), selective precision:
// the router runs in fp32. x is bf16 (exact in fp32); W_r is fp32. Each W_r
// entry is split into three bf16 parts w = w0 + w1 + w2 (w0 = bf16(w),
// w1 = bf16(w - w0), w2 = bf16(w - w0 - w1): 3 x 8 mantissa bits = fp32's 24),
// so x.W_r = x.w0 + x.w1 + x.w2 where every bf16 x bf16 product is exact and
// the tensor core accumulates in fp32: fp32-accurate logits at tensor-core speed.
//
//   router_split_kernel  W_r [d, n] fp32 -> workspace [3, n, d] bf16 (K-major B operand);
//                        run once per weight by moe_router_prepare, or on every call.
//   router_tc_kernel     one CTA per 128 tokens and column tile of experts, 192 threads:
//     warp 0 lane 0   TMA: x tile 128x64 + the three W parts of the tile per stage
//     warp 1 lane 0   tcgen05.mma kind::f16 M=128, N = the tile width (3 parts x 4 K-steps)
//     warps 2-5       drain: thread t of warp w owns token row 32(w%4) + t (its TMEM
//                     lane); each K block's product lands in a fresh TMEM accumulator
//                     (two, ping-pong) and is added into fp32 registers with
//                     round-to-nearest adds, which keeps the sum fp32-accurate.
//   Finish: softmax or logistic, ranking key, top-k with ties to the lower index, gates.
//   Logits mode: the tile's logits are stored (coalesced) and router_finish_kernel (one
//   warp per row, the whole GPU) finishes them in place. Rows mode (no probs_out, or
//   n <= 64 on a grid of more tiles than SMs): each CTA takes whole rows (one tile of all
//   n experts) and finishes them in the kernel, a thread per row up to 64 experts (from
//   the drain thread's registers), a warp per row above.
#include "tc_ptx.cuh"

namespace moe {

namespace rtc {
constexpr int BM = 128, BK = 64, NMAX = 128, kMaxStages = 5;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 drain + epilogue
constexpr int A_BYTES = BM * BK * 2;
}  // namespace rtc

struct RouterTcShared {
    uint64_t full[rtc::kMaxStages], empty[rtc::kMaxStages], tfull[2], tempty[2];
    uint32_t tmem_base;
    int abort_flag;
};

__host__ __device__ inline int router_np(int n) { return ((n + 31) / 32) * 32; }
__host__ __device__ inline int router_stage_bytes(int np) { return rtc::A_BYTES + 3 * np * 128; }
__host__ __device__ inline uint32_t router_tmem_cols(int np) {
    uint32_t c = 32;
    while ((int)c < 2 * np) c <<= 1;
    return c;
}
inline size_t router_tc_smem(int np, int stages) {
    return 1024 + (size_t)stages * router_stage_bytes(np) + sizeof(RouterTcShared);
}

// W_r [d, n] fp32 -> out [3, n, d] bf16 with w = out[0] + out[1] + out[2] (32x32 tiles through shared memory).
__global__ void router_split_kernel(const float* __restrict__ w_r, int d, int n, __nv_bfloat16* __restrict__ out) {
    __shared__ float tile[32][33];
    pdl_trigger();
    pdl_wait();
    const int t0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int t = t0 + r, j = j0 + tx;
        tile[r][tx] = (t < d && j < n) ? w_r[(int64_t)t * n + j] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int j = j0 + r, t = t0 + tx;
        if (j >= n || t >= d) continue;
        const float w = tile[tx][r];
        const __nv_bfloat16 p0 = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(p0);
        const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(p1);
        const __nv_bfloat16 p2 = __float2bfloat16_rn(r2);
        const int64_t o = (int64_t)j * d + t, plane = (int64_t)n * d;
        out[o] = p0;
        out[plane + o] = p1;
        out[2 * plane + o] = p2;
    }
}

namespace rtc {
enum { kModeLogits = 0, kModeRows = 2 };
}  // namespace rtc

// FUSED (3 NP <= 256): the three W parts sit as one 3 NP-row B operand and one MMA per K step
// (N = 3 NP) forms all three products, so each K step reads the x tile from shared memory once
// instead of three times; the drain adds the parts' block products in fp32, small parts first.
template <int NCH, int STAGES, bool FUSED>
__global__ void __launch_bounds__(rtc::kThreads, STAGES == 2 ? 2 : 1)  // two-stage rings: two CTAs per SM
router_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, int64_t m,
                 int d, int n, int k, int fn, int renorm, const float* __restrict__ rank_bias,
                 float* __restrict__ probs_out, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                 int mode) {
    using namespace rtc;
    constexpr int NP = NCH * 32;
    constexpr int STAGE_BYTES = A_BYTES + 3 * NP * 128;
    constexpr int ACOLS = FUSED ? 3 * NP : NP;  // accumulator columns per buffer
    static_assert(STAGES <= kMaxStages, "ring deeper than the barrier arrays");
    static_assert(!FUSED || 3 * NP <= 256, "one MMA takes N <= 256");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RouterTcShared* sh = reinterpret_cast<RouterTcShared*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (d + BK - 1) / BK;
    const uint32_t tcols = router_tmem_cols(ACOLS);
    const int64_t row0 = (int64_t)blockIdx.x * BM;
    const int col0 = blockIdx.y * NP;  // first expert of this CTA's column tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { ptx::mbar_init(&sh->full[s], 1); ptx::mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < 2; ++b) { ptx::mbar_init(&sh->tfull[b], 1); ptx::mbar_init(&sh->tempty[b], 128); }
        sh->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_w);
    }
    if (warp == 1) ptx::tmem_alloc(&sh->tmem_base, tcols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    pdl_trigger();
    pdl_wait();  // the W split and x come from earlier launches
    const uint32_t tmem = sh->tmem_base;
    volatile int* abort_flag = &sh->abort_flag;
    bool drain_ok = true;  // this drain thread received every K block

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag)) break;
                uint8_t* st = smem + stage * STAGE_BYTES;
                ptx::mbar_expect_tx(&sh->full[stage], (uint32_t)STAGE_BYTES);
                ptx::tma_load_2d(st, &map_x, &sh->full[stage], kb * BK, (int)row0);
                for (int part = 0; part < 3; ++part)
                    ptx::tma_load_3d(st + A_BYTES + part * NP * 128, &map_w, &sh->full[stage], kb * BK, col0, part);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, ACOLS);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&sh->tempty[buf], bphase ^ 1u, abort_flag)) break;
                if (!ptx::mbar_wait(&sh->full[stage], phase, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t sa = ptx::smem_u32(smem + stage * STAGE_BYTES);
                const uint64_t adesc = ptx::sw128_kmajor_desc(sa);
                if (FUSED) {
                    // a fresh accumulator per K block: part p's products in columns p NP .. p NP + NP - 1
                    const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        ptx::umma_bf16(tmem + (uint32_t)(buf * ACOLS), adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                       kk != 0 ? 1u : 0u);
                } else {
                    // a fresh accumulator per K block; the small parts of W first, the leading part last
                    for (int part = 2; part >= 0; --part) {
                        const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES + part * NP * 128);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            ptx::umma_bf16(tmem + (uint32_t)(buf * NP), adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                           (part != 2 || kk != 0) ? 1u : 0u);
                    }
                }
                ptx::umma_commit(&sh->empty[stage]);
                ptx::umma_commit(&sh->tfull[buf]);
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                if (++buf == 2) { buf = 0; bphase ^= 1u; }
            }
        }
    } else {
        // drain: thread owns token row 32*(warp%4) + lane; block results added in fp32 (round to nearest)
        const int quad = warp & 3;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        float acc[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[j] = 0.f;
        int buf = 0;
        uint32_t bphase = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            // every lane waits; the warp leaves together if any lane gave up (a timeout), since the
            // TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sh->tfull[buf], bphase, abort_flag))) { drain_ok = false; break; }
            ptx::tc_fence_after();
            if (FUSED) {
                // per 32-column chunk, the three parts' block products: (p2 + p1) + p0, then into acc
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    uint32_t v[3][32];
#pragma unroll
                    for (int p = 0; p < 3; ++p)
                        ptx::tmem_ld32_issue(trow + (uint32_t)(buf * ACOLS + p * NP + c * 32), v[p]);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        const float blk = __fadd_rn(__fadd_rn(__uint_as_float(v[2][q]), __uint_as_float(v[1][q])),
                                                    __uint_as_float(v[0][q]));
                        acc[c * 32 + q] = __fadd_rn(acc[c * 32 + q], blk);
                    }
                }
            } else {
                // every column chunk of the block in flight at once, one wait
                uint32_t v[NCH][32];
#pragma unroll
                for (int c = 0; c < NCH; ++c) ptx::tmem_ld32_issue(trow + (uint32_t)(buf * NP + c * 32), v[c]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < NCH; ++c)
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        acc[c * 32 + q] = __fadd_rn(acc[c * 32 + q], __uint_as_float(v[c][q]));
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sh->tempty[buf]);
            if (++buf == 2) { buf = 0; bphase ^= 1u; }
        }
        bool finished = false;
        if constexpr (NP <= 64) {
            if (drain_ok && mode == kModeRows && k <= 8) {
                // whole rows in this CTA: the thread finishes the row it drained, from its registers
                const int64_t r = row0 + quad * 32 + lane;
                if (r < m) {
                    if (k <= 2) finish_row_thread<NP, 2>(acc, r, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
                    else finish_row_thread<NP, 8>(acc, r, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
                }
                finished = true;
            }
        }
        if (drain_ok && !finished) {
            // park the warp's 32 logit rows in the (now idle) stage memory
            float* rows = reinterpret_cast<float*>(smem) + (size_t)quad * 32 * (NP + 1);
#pragma unroll
            for (int j = 0; j < NP; ++j) rows[lane * (NP + 1) + j] = acc[j];
            __syncwarp();
            if (mode == kModeLogits) {
                // logits out, coalesced (a warp stores one row's 128-byte runs per instruction);
                // router_finish_kernel turns them into scores and picks in place
                for (int rr = 0; rr < 32; ++rr) {
                    const int64_t r = row0 + quad * 32 + rr;
                    if (r >= m) break;
#pragma unroll
                    for (int q = 0; q < NCH; ++q) {
                        const int j = col0 + lane + 32 * q;
                        if (j < n) probs_out[r * n + j] = rows[rr * (NP + 1) + lane + 32 * q];
                    }
                }
            } else if (mode == kModeRows) {
                // whole rows in this CTA (more than 64 experts): a warp finishes each row
                for (int rr = 0; rr < 32; ++rr) {
                    const int64_t r = row0 + quad * 32 + rr;
                    if (r >= m) break;
                    float hv[NCH];
#pragma unroll
                    for (int q = 0; q < NCH; ++q) hv[q] = rows[rr * (NP + 1) + lane + 32 * q];
                    finish_row<NCH>(hv, r, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tcols);
    }
}

size_t router_workspace_bytes(int32_t d, int32_t n, moe_dtype dt) {
    if (dt != MOE_BF16 || d < 1 || n < 1) return 0;
    return (size_t)3 * n * d * 2 + 256;
}

template <int NCH, int ST, bool FUSED>
static cudaError_t launch_router_tc_st(const CUtensorMap& mx, const CUtensorMap& mw, int64_t m, int d, int n, int k,
                                       int fn, int renorm, const float* rank_bias, float* probs_out,
                                       int32_t* topk_idx, float* topk_gate, dim3 grid, int mode,
                                       cudaStream_t stream) {
    const size_t smem = router_tc_smem(NCH * 32, ST);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<NCH, ST, FUSED>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(rtc::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_tc_kernel<NCH, ST, FUSED>, mx, mw, m, d, n, k, fn, renorm, rank_bias,
                              probs_out, topk_idx, topk_gate, mode);
}

// When every CTA has an SM to itself the ring is as deep as shared memory allows (five 40 KB
// stages for a 64-wide tile, three 64 KB stages for a 128-wide one): the x tiles come from HBM
// and the deeper ring keeps more of them in flight. When the grid is larger than the GPU, two
// stages, so that two CTAs (each with its own TMEM accumulators) share an SM: at 65536 x 4096 x 64
// 162 us, against 173 us for one CTA per SM with the three parts in one MMA and 230 us for two
// CTAs per SM with that MMA and one accumulator each.
template <int NCH>
static cudaError_t launch_router_tc_t(const CUtensorMap& mx, const CUtensorMap& mw, int64_t m, int d, int n, int k,
                                      int fn, int renorm, const float* rank_bias, float* probs_out,
                                      int32_t* topk_idx, float* topk_gate, int mode, cudaStream_t stream) {
    const int64_t blocks = (m + rtc::BM - 1) / rtc::BM;
    const unsigned ctiles = (unsigned)((router_np(n) + NCH * 32 - 1) / (NCH * 32));
    const dim3 grid((unsigned)blocks, ctiles);
    if (blocks * ctiles > num_sms())
        return launch_router_tc_st<NCH, 2, false>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx,
                                                  topk_gate, grid, mode, stream);
    if constexpr (NCH <= 2) {
        // one MMA for the three parts (its two 3 NP-column accumulators fill the TMEM of one CTA):
        // 38.4 against 43.1 us at 16384 x 2048 x 64, 16.4 against 18.2 us at 8192 x 768 x 128
        return launch_router_tc_st<NCH, 5, true>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx,
                                                 topk_gate, grid, mode, stream);
    } else {
        return launch_router_tc_st<NCH, 3, false>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx,
                                                  topk_gate, grid, mode, stream);
    }
}

// Tensor-core router for bf16 activations with n <= 128 (the drain keeps a token's n logits in registers).
bool router_tc_supported(int n, int k) { (void)k; return n <= rtc::NMAX; }

// W_r [d, n] fp32 -> the [3, n, d] bf16 split in the workspace (moe_router_prepare, or every call).
cudaError_t launch_router_split(const float* w_r, int d, int n, void* workspace, cudaStream_t stream) {
    dim3 tb(32, 8), tg((unsigned)((d + 31) / 32), (unsigned)((n + 31) / 32));
    return launch_pdl(router_split_kernel, tg, tb, 0, stream, w_r, d, n, static_cast<__nv_bfloat16*>(workspace));
}

// w_r == nullptr: the workspace already holds the split of the router weight (moe_router_prepare).
cudaError_t launch_router_tc(const void* x, const float* w_r, int64_t m, int d, int n, int k, int fn, int renorm,
                             const float* rank_bias, float* probs_out, int32_t* topk_idx, float* topk_gate,
                             void* workspace, cudaStream_t stream) {
    if (!router_tc_supported(n, k)) return cudaErrorNotSupported;
    if (m == 0) return cudaSuccess;
    __nv_bfloat16* wsplit = static_cast<__nv_bfloat16*>(workspace);
    if (w_r) {
        const cudaError_t e = launch_router_split(w_r, d, n, workspace, stream);
        if (e != cudaSuccess) return e;
    }
    const int np = router_np(n);
    CUtensorMap mx, mw;
    if (!map_2d(&mx, x, (uint64_t)m, (uint64_t)d, rtc::BM)) return cudaErrorInvalidValue;
    // Two ways to finish the rows. Logits mode: the projection stores the fp32 logits in 64-wide
    // column tiles and router_finish_kernel (a warp per row, over the whole GPU) finishes them in
    // place. Rows mode: a CTA holds whole rows (one column tile of all n experts) and finishes
    // them itself -- each drain thread its own row from its registers up to 64 experts, a warp
    // per row above. Rows mode is taken without probs_out, and with it when n <= 64 and there are
    // more 128-row tiles than SMs (two CTAs per SM: one CTA's finish runs while the other streams
    // x): 146.5 against 163.6 us at 65536 x 4096 x 64. With one CTA per SM the finish would run
    // on an otherwise idle SM, and logits mode is faster (38.2 against 41.5 us at
    // 16384 x 2048 x 64). A persistent kernel that finished the rows in the same launch (a
    // logits tile in shared memory, four finish warps) measured 204 against 162 us at
    // 65536 x 4096 x 64, its one K-block pipeline per SM latency-bound (33% issue-active).
    const bool many_tiles = (m + rtc::BM - 1) / rtc::BM > (int64_t)num_sms();
    const int mode = (probs_out && !(np <= 64 && many_tiles)) ? rtc::kModeLogits : rtc::kModeRows;
    const int tile = mode == rtc::kModeRows ? np : (np < 64 ? np : 64);
    if (!map_3d(&mw, wsplit, 3, (uint64_t)n, (uint64_t)d, (uint32_t)tile)) return cudaErrorInvalidValue;
    cudaError_t e;
    switch (tile / 32) {
        case 1: e = launch_router_tc_t<1>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, mode, stream); break;
        case 2: e = launch_router_tc_t<2>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, mode, stream); break;
        case 3: e = launch_router_tc_t<3>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, mode, stream); break;
        default: e = launch_router_tc_t<4>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, mode, stream); break;
    }
    if (e != cudaSuccess || mode != rtc::kModeLogits) return e;
    // the tensor-core kernel left the fp32 logits in probs_out: finish them there, one warp per row
    return launch_router_finish(probs_out, m, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
}

}  // namespace moe
