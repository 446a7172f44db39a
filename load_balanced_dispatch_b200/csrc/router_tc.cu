// router_tc.cu -- fp32-accurate router projection on the bf16 tensor cores, with the
// score function, ranking and top-k fused into the epilogue.
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
//   router_rows_kernel   (k <= 8) persistent, one CTA per SM, 320 threads, each CTA
//                        taking 128-token blocks in turn with all n <= 128 experts:
//     warp 0 lane 0   TMA: x tiles 128x64 + the three W parts (all n rows), two 64-deep
//                     K blocks per stage for n <= 64
//     warp 1 lane 0   tcgen05.mma kind::f16 M=128, N = n rounded up to 32 (3 parts x 4 K-steps)
//     warps 2-5       drain: thread t of warp w owns token row 32(w%4) + t (its TMEM lane);
//                     each K block's product lands in a fresh TMEM accumulator (four,
//                     taken in turn, so the MMAs run up to four K blocks ahead of the
//                     drain) and is added into fp32 registers with round-to-nearest
//                     adds, which keeps the sum fp32-accurate. After a block's last K
//                     block the rows go to a shared-memory logits tile.
//     warps 6-9       finish: a warp per row, 32 rows per warp (softmax or logistic,
//                     ranking key, top-k with ties to the lower index, gates, scores
//                     stored coalesced) while the drain accumulates the next block.
//                     Logits never reach HBM.
//   router_tc_kernel     (k > 8) one CTA per 128 tokens and column tile: with probs_out
//                        the logits are stored and router_finish_kernel (a warp per row)
//                        finishes them in place; without it each CTA takes whole rows and
//                        a warp finishes each.
#include "tc_ptx.cuh"

namespace moe {

namespace rtc {
constexpr int BM = 128, BK = 64, NMAX = 128, kMaxStages = 5;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 drain + epilogue
constexpr int A_BYTES = BM * BK * 2;
}  // namespace rtc

// Shared state of the rows kernel: up to kRowsMaxStages ring stages, kRowsAcc TMEM accumulators.
namespace rtc {
constexpr int kRowsMaxStages = 6, kRowsAcc = 4;
constexpr int kRowsThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2-5 drain, warps 6-9 finish
}  // namespace rtc
struct RouterRowsShared {
    uint64_t full[rtc::kRowsMaxStages], empty[rtc::kRowsMaxStages], tfull[rtc::kRowsAcc], tempty[rtc::kRowsAcc];
    uint64_t park_full, park_empty;  // a token block's logits handed from the drain to the finish warps
    uint32_t tmem_base;
    int abort_flag;
};

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

constexpr int KTHREAD = 8;  // largest k finished one row per thread

namespace rtc {
enum { kModeLogits = 0, kModeRows = 2 };
}  // namespace rtc

// Insert (key, j, p) into a best-first list of length k <= KTHREAD (ties: the lower index first).
__device__ __forceinline__ void topk_insert(float (&kk)[KTHREAD], int (&ki)[KTHREAD], float (&kp)[KTHREAD], int k,
                                            float key, int j, float p) {
    bool placed = false;
#pragma unroll
    for (int t = KTHREAD - 1; t >= 0; --t) {
        if (t < k && !placed) {
            const int u = t > 0 ? t - 1 : 0;
            if (t > 0 && ranks_before(key, j, kk[u], ki[u])) {
                kk[t] = kk[u]; ki[t] = ki[u]; kp[t] = kp[u];
            } else {
                if (ranks_before(key, j, kk[t], ki[t])) { kk[t] = key; ki[t] = j; kp[t] = p; }
                placed = true;
            }
        }
    }
}

template <int NCH, int STAGES>
__global__ void __launch_bounds__(rtc::kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, int64_t m,
                 int d, int n, int k, int fn, int renorm, const float* __restrict__ rank_bias,
                 float* __restrict__ probs_out, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
                 int mode) {
    using namespace rtc;
    constexpr int NP = NCH * 32;
    constexpr int STAGE_BYTES = A_BYTES + 3 * NP * 128;
    static_assert(STAGES <= kMaxStages, "ring deeper than the barrier arrays");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RouterTcShared* sh = reinterpret_cast<RouterTcShared*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (d + BK - 1) / BK;
    const uint32_t tcols = router_tmem_cols(NP);
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
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, NP);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&sh->tempty[buf], bphase ^ 1u, abort_flag)) break;
                if (!ptx::mbar_wait(&sh->full[stage], phase, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t sa = ptx::smem_u32(smem + stage * STAGE_BYTES);
                const uint64_t adesc = ptx::sw128_kmajor_desc(sa);
                // a fresh accumulator per K block; the small parts of W first, the leading part last
                for (int part = 2; part >= 0; --part) {
                    const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES + part * NP * 128);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        ptx::umma_bf16(tmem + (uint32_t)(buf * NP), adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                       (part != 2 || kk != 0) ? 1u : 0u);
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
            if (!ptx::mbar_wait(&sh->tfull[buf], bphase, abort_flag)) { drain_ok = false; break; }
            ptx::tc_fence_after();
            // every column chunk of the block in flight at once, one wait
            uint32_t v[NCH][32];
#pragma unroll
            for (int c = 0; c < NCH; ++c) ptx::tmem_ld32_issue(trow + (uint32_t)(buf * NP + c * 32), v[c]);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < NCH; ++c)
#pragma unroll
                for (int q = 0; q < 32; ++q) acc[c * 32 + q] = __fadd_rn(acc[c * 32 + q], __uint_as_float(v[c][q]));
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sh->tempty[buf]);
            if (++buf == 2) { buf = 0; bphase ^= 1u; }
        }
        // park the warp's 32 logit rows in the (now idle) stage memory
        if (drain_ok) {
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
                // whole rows in this CTA (k > KTHREAD, no scores out): a warp finishes each row
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

// Persistent full-row router (k <= KTHREAD): see the file header. Every barrier wait is bounded;
// on a timeout all roles leave their loops and TMEM is freed.
template <int NCH, int STAGES, int H>
__global__ void __launch_bounds__(rtc::kRowsThreads, 1)
router_rows_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, int64_t m,
                   int d, int n, int k, int fn, int renorm, const float* __restrict__ rank_bias,
                   float* __restrict__ probs_out, int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate) {
    using namespace rtc;
    constexpr int NP = NCH * 32;
    // a stage holds H consecutive 64-deep K blocks: x boxes first, then per block the three W
    // parts' boxes, adjacent (so that for n <= 64 one N = 3 NP MMA takes all three parts)
    constexpr int W_BYTES = NP * 128;
    constexpr int STAGE_BYTES = H * (A_BYTES + 3 * W_BYTES);
    constexpr bool FUSEP = NP <= 64;               // the three parts in one MMA, separate columns
    constexpr int WIDTH = FUSEP ? 3 * NP : NP;     // TMEM columns of one accumulator
    constexpr int NACC = (FUSEP && NP == 64) ? 2 : kRowsAcc;
    constexpr int PITCH = NP + 1;  // odd row pitch of the logits tile: no shared-memory bank conflicts
    static_assert(STAGES <= kRowsMaxStages, "ring deeper than the barrier arrays");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* park = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);  // [BM][PITCH] logits of one block
    RouterRowsShared* sh = reinterpret_cast<RouterRowsShared*>(park + BM * PITCH);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = ((d + BK - 1) / BK + H - 1) / H * H;  // a stage's blocks past d are zero fill
    const int64_t nblocks = (m + BM - 1) / BM;
    uint32_t tcols = 32;
    while ((int)tcols < NACC * WIDTH) tcols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { ptx::mbar_init(&sh->full[s], 1); ptx::mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < NACC; ++b) { ptx::mbar_init(&sh->tfull[b], 1); ptx::mbar_init(&sh->tempty[b], 128); }
        ptx::mbar_init(&sh->park_full, 128);
        ptx::mbar_init(&sh->park_empty, 128);
        sh->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_w);
    }
    if (warp == 1) ptx::tmem_alloc(&sh->tmem_base, tcols);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    pdl_wait();  // x (and the W split when made by this call) come from earlier launches
    const uint32_t tmem = sh->tmem_base;
    volatile int* abort_flag = &sh->abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int64_t tb = blockIdx.x; tb < nblocks && ok; tb += gridDim.x) {
                for (int kb = 0; kb < nkb; kb += H) {
                    if (!ptx::mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* st = smem + stage * STAGE_BYTES;
                    ptx::mbar_expect_tx(&sh->full[stage], (uint32_t)STAGE_BYTES);
#pragma unroll
                    for (int h = 0; h < H; ++h)
                        ptx::tma_load_2d(st + h * A_BYTES, &map_x, &sh->full[stage], (kb + h) * BK, (int)(tb * BM));
#pragma unroll
                    for (int h = 0; h < H; ++h)
                        for (int part = 0; part < 3; ++part)
                            ptx::tma_load_3d(st + H * A_BYTES + (h * 3 + part) * W_BYTES, &map_w, &sh->full[stage],
                                             (kb + h) * BK, 0, part);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(BM, WIDTH);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int64_t tb = blockIdx.x; tb < nblocks && ok; tb += gridDim.x) {
                for (int kb = 0; kb < nkb; kb += H) {
                    if (!ptx::mbar_wait(&sh->full[stage], phase, abort_flag)) { ok = false; break; }
                    const uint32_t sa = ptx::smem_u32(smem + stage * STAGE_BYTES);
                    for (int h = 0; h < H; ++h) {
                        if (!ptx::mbar_wait(&sh->tempty[buf], bphase ^ 1u, abort_flag)) { ok = false; break; }
                        ptx::tc_fence_after();
                        const uint64_t adesc = ptx::sw128_kmajor_desc(sa + h * A_BYTES);
                        const uint32_t wbase = sa + H * A_BYTES + h * 3 * W_BYTES;
                        if (FUSEP) {
                            // a fresh accumulator per K block; part p's products in columns p NP ..
                            const uint64_t bdesc = ptx::sw128_kmajor_desc(wbase);
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                ptx::umma_bf16(tmem + (uint32_t)(buf * WIDTH), adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                               kk != 0 ? 1u : 0u);
                        } else {
                            // a fresh accumulator per K block; the small parts of W first, the leading part last
                            for (int part = 2; part >= 0; --part) {
                                const uint64_t bdesc = ptx::sw128_kmajor_desc(wbase + part * W_BYTES);
#pragma unroll
                                for (int kk = 0; kk < BK / 16; ++kk)
                                    ptx::umma_bf16(tmem + (uint32_t)(buf * WIDTH), adesc + 2 * kk, bdesc + 2 * kk,
                                                   idesc, (part != 2 || kk != 0) ? 1u : 0u);
                            }
                        }
                        ptx::umma_commit(&sh->tfull[buf]);
                        if (++buf == NACC) { buf = 0; bphase ^= 1u; }
                    }
                    if (!ok) break;
                    ptx::umma_commit(&sh->empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp < 6) {
        // drain: thread t of this warp owns the block's row 32 quad + t (its TMEM lane)
        const int quad = warp & 3;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        float* prow = park + (quad * 32 + lane) * PITCH;
        int buf = 0;
        uint32_t bphase = 0, pphase = 0;
        bool ok = true;
        for (int64_t tb = blockIdx.x; tb < nblocks && ok; tb += gridDim.x) {
            float acc[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) acc[j] = 0.f;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!ptx::mbar_wait(&sh->tfull[buf], bphase, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                if (FUSEP) {
                    // per 32 experts: the three parts' products in flight together, added smallest
                    // first ((w2 + w1) + w0), then into the running sum (all round to nearest)
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        uint32_t v[2][32];
                        ptx::tmem_ld32_issue(trow + (uint32_t)(buf * WIDTH + 2 * NP + c * 32), v[0]);
                        ptx::tmem_ld32_issue(trow + (uint32_t)(buf * WIDTH + NP + c * 32), v[1]);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            v[1][q] = __float_as_uint(__fadd_rn(__uint_as_float(v[0][q]), __uint_as_float(v[1][q])));
                        ptx::tmem_ld32_issue(trow + (uint32_t)(buf * WIDTH + c * 32), v[0]);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            acc[c * 32 + q] = __fadd_rn(acc[c * 32 + q],
                                                        __fadd_rn(__uint_as_float(v[1][q]), __uint_as_float(v[0][q])));
                    }
                } else {
                    // two 32-column chunks in flight per wait
#pragma unroll
                    for (int c = 0; c < NCH; c += 2) {
                        uint32_t v[2][32];
                        ptx::tmem_ld32_issue(trow + (uint32_t)(buf * WIDTH + c * 32), v[0]);
                        if (c + 1 < NCH) ptx::tmem_ld32_issue(trow + (uint32_t)(buf * WIDTH + (c + 1) * 32), v[1]);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            acc[c * 32 + q] = __fadd_rn(acc[c * 32 + q], __uint_as_float(v[0][q]));
                        if (c + 1 < NCH) {
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                acc[(c + 1) * 32 + q] = __fadd_rn(acc[(c + 1) * 32 + q], __uint_as_float(v[1][q]));
                        }
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&sh->tempty[buf]);
                if (++buf == NACC) { buf = 0; bphase ^= 1u; }
            }
            if (!ok) break;
            // hand the block's logits to the finish warps once they are done with the previous block
            if (!ptx::mbar_wait(&sh->park_empty, pphase ^ 1u, abort_flag)) break;
#pragma unroll
            for (int j = 0; j < NP; ++j) prow[j] = acc[j];
            ptx::mbar_arrive(&sh->park_full);
            pphase ^= 1u;
        }
    } else {
        // finish: warp f takes rows 32 f .. 32 f + 31 of each block, one row at a time with the
        // whole warp (lane holds experts lane + 32 q): scores, ranking keys, top-k, gates, and the
        // scores stored coalesced, while the drain accumulates the next block
        const int fw = warp - 6;
        uint32_t pphase = 0;
        for (int64_t tb = blockIdx.x; tb < nblocks; tb += gridDim.x) {
            if (!ptx::mbar_wait(&sh->park_full, pphase, abort_flag)) break;
            for (int rr = 0; rr < 32; ++rr) {
                const int r = fw * 32 + rr;
                const int64_t row = tb * BM + r;
                if (row >= m) break;
                float hv[NCH];
#pragma unroll
                for (int q = 0; q < NCH; ++q) hv[q] = park[r * PITCH + lane + 32 * q];
                finish_row<NCH>(hv, row, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
            }
            __syncwarp();
            ptx::mbar_arrive(&sh->park_empty);
            pphase ^= 1u;
        }
    }
    pdl_trigger();  // the dependent launch may start while this grid drains
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tcols);
    }
}

inline size_t router_rows_smem(int np, int stages, int h) {
    return 1024 + (size_t)stages * h * router_stage_bytes(np) + (size_t)rtc::BM * (np + 1) * 4 +
           sizeof(RouterRowsShared);
}

// Ring of the rows kernel: H K blocks per stage (two for up to 64 experts: each x row is then
// read 256 contiguous bytes at a time), and as many stages as fit next to the logits tile.
constexpr int router_rows_h(int nch) { return nch <= 2 ? 2 : 1; }
constexpr int router_rows_stages(int nch) { return nch == 1 ? 3 : (nch == 2 ? 2 : (nch == 3 ? 3 : 2)); }

template <int NCH>
static cudaError_t launch_router_rows_t(const CUtensorMap& mx, const CUtensorMap& mw, int64_t m, int d, int n, int k,
                                        int fn, int renorm, const float* rank_bias, float* probs_out,
                                        int32_t* topk_idx, float* topk_gate, cudaStream_t stream) {
    constexpr int ST = router_rows_stages(NCH), H = router_rows_h(NCH);
    const size_t smem = router_rows_smem(NCH * 32, ST, H);
    static bool attr = false;
    if (!attr) {
        const cudaError_t e = cudaFuncSetAttribute(router_rows_kernel<NCH, ST, H>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const int64_t blocks = (m + rtc::BM - 1) / rtc::BM;
    const int64_t cap = (int64_t)num_sms();
    const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
    return launch_pdl(router_rows_kernel<NCH, ST, H>, dim3(grid), dim3(rtc::kRowsThreads), smem, stream, mx, mw, m, d, n,
                      k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate);
}

size_t router_workspace_bytes(int32_t d, int32_t n, moe_dtype dt) {
    if (dt != MOE_BF16 || d < 1 || n < 1) return 0;
    return (size_t)3 * n * d * 2 + 256;
}

template <int NCH, int ST>
static cudaError_t launch_router_tc_st(const CUtensorMap& mx, const CUtensorMap& mw, int64_t m, int d, int n, int k,
                                       int fn, int renorm, const float* rank_bias, float* probs_out,
                                       int32_t* topk_idx, float* topk_gate, dim3 grid, int mode,
                                       cudaStream_t stream) {
    const size_t smem = router_tc_smem(NCH * 32, ST);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<NCH, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
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
    return cudaLaunchKernelEx(&cfg, router_tc_kernel<NCH, ST>, mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out,
                              topk_idx, topk_gate, mode);
}

// When every CTA has an SM to itself the ring is as deep as shared memory allows (five 40 KB
// stages for a 64-wide tile, three 64 KB stages for a 128-wide one): the x tiles come from HBM
// and the deeper ring keeps more of them in flight. When the grid is larger than the GPU, two
// stages, so that two CTAs (each with its own TMEM accumulators) share an SM.
template <int NCH>
static cudaError_t launch_router_tc_t(const CUtensorMap& mx, const CUtensorMap& mw, int64_t m, int d, int n, int k,
                                      int fn, int renorm, const float* rank_bias, float* probs_out,
                                      int32_t* topk_idx, float* topk_gate, int mode, cudaStream_t stream) {
    const int64_t blocks = (m + rtc::BM - 1) / rtc::BM;
    const unsigned ctiles = (unsigned)((router_np(n) + NCH * 32 - 1) / (NCH * 32));
    const dim3 grid((unsigned)blocks, ctiles);
    if (blocks * ctiles > num_sms())
        return launch_router_tc_st<NCH, 2>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate,
                                           grid, mode, stream);
    constexpr int kDeep = NCH <= 2 ? 5 : 3;
    return launch_router_tc_st<NCH, kDeep>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx,
                                           topk_gate, grid, mode, stream);
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
    if (k <= KTHREAD) {
        // every expert in one tile: the drain threads finish their rows in registers
        if (!map_3d(&mw, wsplit, 3, (uint64_t)n, (uint64_t)d, (uint32_t)np)) return cudaErrorInvalidValue;
        switch (np / 32) {
            case 1: return launch_router_rows_t<1>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
            case 2: return launch_router_rows_t<2>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
            case 3: return launch_router_rows_t<3>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
            default: return launch_router_rows_t<4>(mx, mw, m, d, n, k, fn, renorm, rank_bias, probs_out, topk_idx, topk_gate, stream);
        }
    }
    // k > KTHREAD. With probs_out the logits go to memory in 64-wide column tiles and
    // router_finish_kernel (a warp per row, the whole GPU) finishes them in place; without it
    // (nothing to store them in) each CTA keeps whole rows and a warp finishes each.
    const int mode = probs_out ? rtc::kModeLogits : rtc::kModeRows;
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
