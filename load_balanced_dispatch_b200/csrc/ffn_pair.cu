// ffn_pair.cu -- the bf16 expert FFN on two-SM tensor-core tiles (tcgen05 cta_group::2).
//
// Switch Transformers paper review (tildalice.io/?p=118), Switch Layer:
// FFN(x) = max(0, x W1 + b1) W2 + b2 per expert.
//
// The schedule is the one of ffn_fused.cu -- one persistent launch, every GEMM1 tile
// (h = relu(xbuf W1_e^T + b1_e), bf16) then every GEMM2 tile (ybuf = h W2_e^T + b2_e), taken
// from one global ticket counter, a GEMM2 tile of expert e waiting (bounded) for the GEMM1
// tiles of e -- but a tile is 256 rows x 256 columns and belongs to a cluster pair of CTAs on
// two SMs. Each CTA loads its own 128 rows of A and its own 128 rows (of the tile's 256
// columns) of B; the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16),
// which reads both CTAs' halves and accumulates each CTA's 128 rows in that CTA's TMEM. For the
// same products per SM a 64-deep K block now refills 32 KB of shared memory instead of the
// 48 KB of a one-SM 128 x 256 tile: the operand traffic from L2, which holds the one-SM tiles
// below the tensor-core rate at the tensor-bound shapes, drops by a third. No TMA multicast:
// each CTA loads its own halves (the loads only count their bytes on the even CTA's barrier).
//
// When d and d_ff are multiples of 512 a tile is 256 x 512 instead: each K step's A block
// serves two N = 256 MMAs (PairCfg below).
//
// Per CTA, 192 threads: warp 0 is the producer (the even CTA's also takes the tickets and hands
// each tile id to both CTAs), warp 1 lane 0 of the even CTA issues the MMAs, warps 2-5 drain
// the CTA's TMEM rows (bias, ReLU for GEMM1, bf16, 16-byte stores) while the other of two
// accumulators fills (256-column tiles; a 512-column tile fills the TMEM, and its drain and the
// next tile's MMAs take turns). Barriers (E = even CTA, both = one in each CTA):
//   full[s]    E, 1 arrival (E's producer, with the byte count of both CTAs' loads) plus the
//              bytes of both CTAs' TMA loads;
//   empty[s]   both, 1 arrival: the MMA commit of the stage, sent to both CTAs;
//   tfull[a]   both, 1 arrival: the MMA commit of a finished accumulator;
//   tempty[a]  E, 8 arrivals: the 4 epilogue warps of each CTA, after draining accumulator a;
//   tready[r]  both, 1 arrival: E's producer, after writing tile id r into both rings;
//   tfree[r]   E, 10 arrivals: E's MMA warp and epilogue warps, the odd CTA's producer and
//              epilogue warps, once each has read tile id r.
// Every wait is bounded (about 2 s); a timeout sets the device error word and the CTA's abort
// flag, and every role leaves its loop. Before TMEM is freed the even CTA waits (bounded) for
// its last MMAs and both CTAs meet at a cluster barrier.
#include "groups.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace fpair {
constexpr int HM = 128, BM = 256, HN = 128, BN = 256, BK = 64;
constexpr int A_BYTES = HM * BK * 2, B_BYTES = HN * BK * 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr int RING = 4;
}  // namespace fpair

// NW 256-column MMAs per tile: a tile is 256 rows x (NW x 256) columns, and each K step's A
// block serves NW MMAs, so the shared-memory fill per flop drops by a quarter at NW = 2.
// NW = 1: six 32 KB stages, two accumulators (the drain of one overlaps the MMAs of the other).
// NW = 2: four 48 KB stages (A plus two B boxes per CTA), one 512-column accumulator whose drain
// the MMAs wait for. Against NW = 1 in the same calls: at the global-batch shape (d = d_ff =
// 4096) the FFN ran 1.4-2.4% faster, at d_ff = 1408 (Loss-Free) 2.7% slower (a 384-column last
// tile, a longer tail of the persistent schedule). Eight epilogue warps (two per TMEM lane
// quarter, a 256-column half each) gained nothing more: 0.9-2.1% faster at the global-batch
// shape, 4.7% slower at Loss-Free.
template <int NW>
struct PairCfg {
    static constexpr int TW = NW * fpair::BN;                          // tile width (columns)
    static constexpr int STAGES = NW == 1 ? 6 : 4;
    static constexpr int STAGE_BYTES = fpair::A_BYTES + NW * fpair::B_BYTES;
    static constexpr int NACC = (int)fpair::TMEM_COLS / TW;            // accumulators in TMEM
    static constexpr int EPI = 4;                                      // epilogue warps
    static constexpr int CW = TW * 4 / EPI;                            // columns drained per warp
    static constexpr int THREADS = 64 + 32 * EPI;
    // tile-id ring arrivals: the even CTA's MMA warp and epilogue warps, the odd CTA's producer
    // and epilogue warps
    static constexpr uint32_t TFREE = 2 + 2 * EPI;
};

template <int NW>
struct PairShared {
    uint64_t full[PairCfg<NW>::STAGES], empty[PairCfg<NW>::STAGES], tfull[PairCfg<NW>::NACC],
        tempty[PairCfg<NW>::NACC];
    uint64_t tready[fpair::RING], tfree[fpair::RING];
    uint64_t mma_done;
    int tile_ring[fpair::RING];
    __align__(16) __nv_bfloat16 bias_stage[PairCfg<NW>::EPI][PairCfg<NW>::CW];  // each epilogue warp's columns
    uint32_t tmem_base;
    int abort_flag;
    GroupTable g1, g2;
};

template <int NW>
constexpr size_t pair_smem_bytes() {
    return 1024 + (size_t)PairCfg<NW>::STAGES * PairCfg<NW>::STAGE_BYTES + sizeof(PairShared<NW>);
}

struct PairTile {
    int phase, e, n0, N, K, mtiles;
    int nb;        // 256-column MMAs with valid columns (1 .. NW)
    int nt_last;   // width of the last of them: 128 when at most 128 of its columns are valid, else 256
    int64_t row0, row_end;
};

// Ticket -> tile: every GEMM1 tile (expert-major, then column-major within the expert) comes
// before every GEMM2 tile. A 256-column MMA with at most 128 valid columns runs at N = 128
// (then each CTA supplies 64 rows of B).
template <int NW>
__device__ __forceinline__ PairTile pair_decode(const PairShared<NW>* sh, int ticket, int n, int d, int d_ff) {
    PairTile t;
    const int T1 = sh->g1.tile_start[n];
    t.phase = ticket < T1 ? 1 : 2;
    const int lt = ticket < T1 ? ticket : ticket - T1;
    const GroupTable& g = t.phase == 1 ? sh->g1 : sh->g2;
    t.e = group_of_tile(g, n, lt);
    const int local = lt - g.tile_start[t.e];
    const int rows_e = g.row_start[t.e + 1] - g.row_start[t.e];
    t.mtiles = (rows_e + fpair::BM - 1) / fpair::BM;
    const int nt = local / t.mtiles, mt = local - nt * t.mtiles;
    t.row0 = (int64_t)g.row_start[t.e] + (int64_t)mt * fpair::BM;
    t.row_end = g.row_start[t.e + 1];
    t.n0 = nt * PairCfg<NW>::TW;
    t.N = t.phase == 1 ? d_ff : d;
    t.K = t.phase == 1 ? d : d_ff;
    const int valid = t.N - t.n0;  // > 0
    t.nb = valid >= PairCfg<NW>::TW ? NW : (valid + fpair::BN - 1) / fpair::BN;
    const int last = valid - (t.nb - 1) * fpair::BN;
    t.nt_last = last <= fpair::HN ? fpair::HN : fpair::BN;
    return t;
}

template <int NW>
__global__ void __launch_bounds__(PairCfg<NW>::THREADS, 1)
ffn_pair_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w1,
            const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w2,
            const __nv_bfloat16* __restrict__ b1, const __nv_bfloat16* __restrict__ b2,
            const int32_t* __restrict__ offsets, int n, int d, int d_ff, int64_t max_rows,
            __nv_bfloat16* __restrict__ h, __nv_bfloat16* __restrict__ y, int* __restrict__ done1,
            int* __restrict__ next_tile) {
    using namespace fpair;
    constexpr int TW = PairCfg<NW>::TW, STAGES = PairCfg<NW>::STAGES, STAGE_BYTES = PairCfg<NW>::STAGE_BYTES;
    constexpr int NACC = PairCfg<NW>::NACC, EPI = PairCfg<NW>::EPI;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairShared<NW>* sh = reinterpret_cast<PairShared<NW>*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();  // 0 (issues the MMAs) or 1 within the pair
    const bool leader = rank == 0;
    const int ntn1 = (d_ff + TW - 1) / TW, ntn2 = (d + TW - 1) / TW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { ptx::mbar_init(&sh->full[s], 1); ptx::mbar_init(&sh->empty[s], 1); }
        for (int b = 0; b < NACC; ++b) { ptx::mbar_init(&sh->tfull[b], 1); ptx::mbar_init(&sh->tempty[b], 2 * EPI); }
        for (int r = 0; r < RING; ++r) {
            ptx::mbar_init(&sh->tready[r], 1);
            ptx::mbar_init(&sh->tfree[r], PairCfg<NW>::TFREE);
        }
        ptx::mbar_init(&sh->mma_done, 1);
        sh->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_w1);
        ptx::prefetch_tensormap(&map_h);
        ptx::prefetch_tensormap(&map_w2);
    }
    if (warp == 1) ptx::tmem_alloc_pair(&sh->tmem_base, TMEM_COLS);
    pdl_wait();  // expert_offsets, xbuf and the counters come from earlier launches
    if (warp == 2) build_group_table(offsets, n, ntn1, BM, max_rows, sh->g1);
    if (warp == 3) build_group_table(offsets, n, ntn2, BM, max_rows, sh->g2);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
    ptx::tc_fence_after();
    const uint32_t tmem_base = sh->tmem_base;
    const int total = sh->g1.tile_start[n] + sh->g2.tile_start[n];
    volatile int* abort_flag = &sh->abort_flag;
    // shared::cluster address of this CTA's object at the same offset in CTA `r` of the pair
    auto in_cta = [](const void* p, uint32_t r) { return ptx::mapa_shared(ptx::smem_u32(p), r); };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, slot = 0;
            uint32_t phase = 0, rphase = 0;
            const uint64_t wpolicy = ptx::l2_policy_evict_first();
            for (;;) {
                int tile;
                if (leader) {
                    // take the next tile and hand its id to both CTAs
                    if (!ptx::mbar_wait_cluster(&sh->tfree[slot], rphase ^ 1u, abort_flag)) break;
                    const int tk = atomicAdd(next_tile, 1);
                    tile = tk < total ? tk : -1;
                    sh->tile_ring[slot] = tile;
                    ptx::st_cluster_s32(in_cta(&sh->tile_ring[slot], 1), tile);
                    ptx::mbar_arrive(&sh->tready[slot]);
                    ptx::mbar_arrive_cluster(in_cta(&sh->tready[slot], 1));
                } else {
                    if (!ptx::mbar_wait_cluster(&sh->tready[slot], rphase, abort_flag)) break;
                    tile = *(volatile int*)&sh->tile_ring[slot];
                    ptx::mbar_arrive_cluster(in_cta(&sh->tfree[slot], 0));
                }
                if (++slot == RING) { slot = 0; rphase ^= 1u; }
                if (tile < 0) break;
                const PairTile t = pair_decode(sh, tile, n, d, d_ff);
                if (t.phase == 2) {
                    // every GEMM1 tile of expert e, each signalled by every epilogue warp of its pair
                    const int need = t.mtiles * ntn1 * EPI * 2;
                    if (!ptx::wait_count_geq(done1 + t.e, need, abort_flag, ptx::kWaitCycles)) break;
                    ptx::fence_proxy_async_global();
                }
                const CUtensorMap* ma = t.phase == 1 ? &map_x : &map_h;
                const CUtensorMap* mb = t.phase == 1 ? &map_w1 : &map_w2;
                const int nkb = (t.K + BK - 1) / BK;
                const int arow = (int)(t.row0 + (int64_t)HM * rank);  // this CTA's half of the rows
                // this CTA's half of each 256-column MMA's columns
                int brow[NW];
#pragma unroll
                for (int w = 0; w < NW; ++w)
                    brow[w] = t.n0 + BN * w + ((w == t.nb - 1 ? t.nt_last : BN) / 2) * (int)rank;
                const uint32_t stage_tx = 2u * (uint32_t)(A_BYTES + t.nb * B_BYTES);  // both CTAs' loads
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait_cluster(&sh->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    const uint32_t fb = in_cta(&sh->full[stage], 0);
                    if (leader) ptx::mbar_expect_tx(&sh->full[stage], stage_tx);
                    ptx::tma_load_2d_pair(sa, ma, fb, kb * BK, arow);
                    // an expert with one row tile reads each weight tile once: evict-first, so the
                    // hidden rows h that its GEMM2 tiles read back stay in L2
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        if (w >= t.nb) break;
                        if (t.mtiles == 1)
                            ptx::tma_load_3d_pair_hint(sa + A_BYTES + w * B_BYTES, mb, fb, kb * BK, brow[w], t.e,
                                                       wpolicy);
                        else
                            ptx::tma_load_3d_pair(sa + A_BYTES + w * B_BYTES, mb, fb, kb * BK, brow[w], t.e);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            int stage = 0, acc = 0, slot = 0;
            uint32_t phase = 0, aphase = 0, rphase = 0;
            for (;;) {
                if (!ptx::mbar_wait(&sh->tready[slot], rphase, abort_flag)) break;
                const int tile = *(volatile int*)&sh->tile_ring[slot];
                ptx::mbar_arrive(&sh->tfree[slot]);
                if (++slot == RING) { slot = 0; rphase ^= 1u; }
                if (tile < 0) break;
                const PairTile t = pair_decode(sh, tile, n, d, d_ff);
                const int nkb = (t.K + BK - 1) / BK;
                const uint32_t idesc_full = ptx::idesc_bf16_f32(BM, BN);
                const uint32_t idesc_last = ptx::idesc_bf16_f32(BM, t.nt_last);
                // both CTAs' epilogues have drained this accumulator
                if (!ptx::mbar_wait_cluster(&sh->tempty[acc], aphase ^ 1u, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t tmem_d = tmem_base + (uint32_t)(acc * TW);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait_cluster(&sh->full[stage], phase, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(smem + stage * STAGE_BYTES);
                    const uint64_t adesc = ptx::sw128_kmajor_desc(sa);
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        if (w >= t.nb) break;
                        const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES + w * B_BYTES);
                        const uint32_t idesc = w == t.nb - 1 ? idesc_last : idesc_full;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            ptx::umma_bf16_pair(tmem_d + (uint32_t)(w * BN), adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                                (kb | kk) != 0);
                    }
                    ptx::umma_commit_pair(&sh->empty[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::umma_commit_pair(&sh->tfull[acc], 0x3);
                if (++acc == NACC) { acc = 0; aphase ^= 1u; }
            }
            // every MMA this pair issued has completed before either CTA frees its TMEM
            ptx::umma_commit_pair(&sh->mma_done, 0x1);
            for (long long it = 0; it < (1LL << 26) && !ptx::mbar_try_wait(&sh->mma_done, 0u); ++it) {
            }
        }
    } else {
        const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31 belong to this warp
        constexpr int CW = PairCfg<NW>::CW;
        const int cbase = CW * ((warp - 2) / 4);  // this warp's CW columns of the tile
        int acc = 0, slot = 0;
        uint32_t aphase = 0, rphase = 0;
        for (;;) {
            // every lane waits; the warp leaves together if any lane gave up (a timeout): the
            // warp-collective TMEM loads and __syncwarp below need all 32 lanes
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster(&sh->tready[slot], rphase, abort_flag))) break;
            const int tile = *(volatile int*)&sh->tile_ring[slot];
            __syncwarp();
            if (lane == 0) {
                if (leader) ptx::mbar_arrive(&sh->tfree[slot]);
                else ptx::mbar_arrive_cluster(in_cta(&sh->tfree[slot], 0));
            }
            if (++slot == RING) { slot = 0; rphase ^= 1u; }
            if (tile < 0) break;
            const PairTile t = pair_decode(sh, tile, n, d, d_ff);
            // the accumulator columns the tile's MMAs write, and this warp's share of them
            const int tw_valid = (t.nb - 1) * BN + t.nt_last;
            const int cend = tw_valid < cbase + CW ? tw_valid : cbase + CW;
            // stage the bias of this warp's columns in shared memory while the accumulator fills
            __nv_bfloat16* be = sh->bias_stage[warp - 2];
            {
                const __nv_bfloat16* gb = (t.phase == 1 ? b1 : b2) + (int64_t)t.e * t.N;
#pragma unroll
                for (int p = 0; p < CW / 256; ++p) {
                    const int c = cbase + p * 256 + lane * 8;
                    if (c < cend && t.n0 + c < t.N)
                        *reinterpret_cast<uint4*>(be + p * 256 + lane * 8) =
                            *reinterpret_cast<const uint4*>(gb + t.n0 + c);
                }
                __syncwarp();
            }
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster(&sh->tfull[acc], aphase, abort_flag))) break;
            ptx::tc_fence_after();
            const int64_t r = t.row0 + (int64_t)HM * rank + quad * 32 + lane;
            const bool row_ok = r < t.row_end;
            const bool relu = t.phase == 1;
            __nv_bfloat16* out = t.phase == 1 ? h : y;
            // two 32-column chunks in flight per wait
            for (int c2 = cbase / 32; c2 < cend / 32; c2 += 2) {
                const int colA = t.n0 + c2 * 32;
                if (colA >= t.N) break;  // warp-uniform
                const bool hasB = colA + 32 < t.N;
                uint32_t v2[2][32];
                const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * TW + c2 * 32);
                ptx::tmem_ld32_issue(tbase, v2[0]);
                if (hasB) ptx::tmem_ld32_issue(tbase + 32, v2[1]);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (half == 1 && !hasB) break;
                    const int col0 = colA + half * 32;
                    const uint32_t (&v)[32] = v2[half];
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int col = col0 + g8 * 8;
                        if (col >= t.N) break;
                        float f[8], bv[8];
                        Vec16<__nv_bfloat16>::load(be + (col - t.n0 - cbase), bv);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            f[q] = __uint_as_float(v[g8 * 8 + q]) + bv[q];
                            if (relu) f[q] = fmaxf(f[q], 0.f);
                        }
                        if (row_ok) Vec16<__nv_bfloat16>::store(out + r * t.N + col, f);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(in_cta(&sh->tempty[acc], 0));
            if (t.phase == 1) {
                // publish this warp's h rows to the TMA loads of the GEMM2 tiles of expert e
                ptx::fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(done1 + t.e, 1);
                }
            }
            if (++acc == NACC) { acc = 0; aphase ^= 1u; }
        }
    }
    pdl_trigger();  // the dependent launch may start while the pairs drain
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // neither CTA frees its TMEM while the pair may still use it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// Pairs of CTAs that can be resident at once (one CTA per SM), times two: the persistent grid.
template <int NW>
static unsigned pair_grid(size_t smem) {
    static unsigned grid = 0;
    if (!grid) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(PairCfg<NW>::THREADS);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = 2;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, ffn_pair_tc<NW>, &cfg) != cudaSuccess || clusters <= 0)
            clusters = num_sms() / 2;
        grid = 2u * (unsigned)clusters;
    }
    return grid;
}

template <int NW>
static cudaError_t launch_ffn_pair_t(const CUtensorMap& mx, const CUtensorMap& mw1, const CUtensorMap& mh,
                                     const CUtensorMap& mw2, const void* b1, const void* b2, const int32_t* offsets,
                                     int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf, int* counters,
                                     cudaStream_t stream) {
    const size_t smem = pair_smem_bytes<NW>();
    static bool attr = false;
    if (!attr) {
        const cudaError_t e =
            cudaFuncSetAttribute(ffn_pair_tc<NW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pair_grid<NW>(smem));
    cfg.blockDim = dim3(PairCfg<NW>::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = 2;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, ffn_pair_tc<NW>, mx, mw1, mh, mw2, static_cast<const __nv_bfloat16*>(b1),
                              static_cast<const __nv_bfloat16*>(b2), offsets, n, d, d_ff, max_rows,
                              static_cast<__nv_bfloat16*>(hbuf), static_cast<__nv_bfloat16*>(ybuf), counters,
                              counters + n);
}


// The two-SM FFN: xbuf [max_rows, d] expert-major rows -> ybuf [max_rows, d], h the workspace.
cudaError_t launch_ffn_pair(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                            const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                            int* counters, cudaStream_t stream) {
    CUtensorMap mx, mw1, mh, mw2;
    if (!map_2d(&mx, xbuf, (uint64_t)max_rows, (uint64_t)d, fpair::HM)) return cudaErrorInvalidValue;
    if (!map_3d(&mw1, w1, (uint64_t)n, (uint64_t)d_ff, (uint64_t)d, fpair::HN)) return cudaErrorInvalidValue;
    if (!map_2d(&mh, hbuf, (uint64_t)max_rows, (uint64_t)d_ff, fpair::HM)) return cudaErrorInvalidValue;
    if (!map_3d(&mw2, w2, (uint64_t)n, (uint64_t)d, (uint64_t)d_ff, fpair::HN)) return cudaErrorInvalidValue;
    // counters[0..n-1]: GEMM1 completions per expert; counters[n]: next tile ticket
    cudaError_t e = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)(n + 1), stream);
    if (e != cudaSuccess) return e;
    // 512-column tiles when both GEMMs' widths are multiples of 512 (no partial wide tile)
    if (d % 512 == 0 && d_ff % 512 == 0)
        return launch_ffn_pair_t<2>(mx, mw1, mh, mw2, b1, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, counters,
                                    stream);
    return launch_ffn_pair_t<1>(mx, mw1, mh, mw2, b1, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, counters,
                                stream);
}

}  // namespace moe
