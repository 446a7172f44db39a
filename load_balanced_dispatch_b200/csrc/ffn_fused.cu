// ffn_fused.cu -- the bf16 expert FFN as ONE persistent tcgen05 launch over both GEMMs.
//
// Switch Transformers paper review (tildalice.io/?p=118), Switch Layer:
// FFN(x) = max(0, x W1 + b1) W2 + b2 per expert.
//
// The tile list holds every GEMM1 tile (h = relu(xbuf W1_e^T + b1_e), bf16)
// followed by every GEMM2 tile (ybuf = h W2_e^T + b2_e). CTAs take tiles from
// a global ticket counter (dynamic scheduling balances the unequal tiles: a
// GEMM2 tile streams four times the weight bytes of a GEMM1 tile at the
// Switch-Base shape). Tickets are taken in list order and only by running
// CTAs, so every GEMM1 tile a GEMM2 tile waits for is held by a running CTA
// that needs nothing else to finish it: no deadlock without co-residency.
// A GEMM2 tile of expert e waits for a per-expert counter in global memory:
// each epilogue warp of a GEMM1 tile stores its h rows, fences them for the
// async (TMA) proxy and release-adds 1; the producer of a GEMM2 tile
// acquire-polls the counter (bounded), fences, then loads h with TMA. One
// launch instead of two removes the second kernel's prologue and the wave
// tail between the GEMMs.
//
// One CTA per SM, 192 threads: warp 0 takes tickets and runs the TMA producer
// (4-stage ring of a 128x64 A tile and a 256x64 B tile, 128-byte swizzle,
// K-major, no multicast); warp 1's lane 0 issues tcgen05.mma kind::f16
// (M=128, N=256, K=16, bf16 x bf16 -> fp32 in TMEM; N=128 for a tile with at
// most 128 valid columns) and commits each stage back; warps 2-5 drain one of two TMEM accumulators (tcgen05.ld, + bias,
// ReLU for GEMM1, bf16, 16-byte stores) while the other fills. Row tails past
// an expert's end are computed and masked; column and K tails are TMA zero
// fill. Every wait is bounded (about 2 s), after which the device error word
// and an abort flag are set and all roles leave their loops.
//
// With one pick per token (k = 1) the GEMM2 epilogue can also do the gated
// combine (moe_expert_ffn_combine): each output row is written, gated, to its
// token's row of y, so ybuf and the combine launch disappear; the few dropped
// tokens get their residual (or zeros) from combine_dropped_kernel, which also
// clears the FFN's counters so that the FFN launch directly follows it.
#include "groups.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace fz {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kLoadWarps = 4;
// warp 0 TMA, warp 1 MMA, warps 2-5 epilogue; with the row gather also warps 6-9
constexpr int threads(bool gather) { return gather ? 320 : 192; }
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = ptx::idesc_bf16_f32(BM, BN);
// a tile with at most BN / 2 valid columns (the last one when N % BN <= BN / 2) issues N = BN / 2
// MMAs over the first half of its B tile; the epilogue never reads the other half
constexpr uint32_t IDESC_HALF = ptx::idesc_bf16_f32(BM, BN / 2);
constexpr int kEpiWarps = 4;
constexpr int RING = 4;   // tile ids handed from the producer to the MMA and epilogue warps
}  // namespace fz

struct FusedShared {
    uint64_t full[fz::STAGES], empty[fz::STAGES], tfull[2], tempty[2];
    uint64_t tready[fz::RING], tfree[fz::RING];
    int tile_ring[fz::RING];
    __align__(16) __nv_bfloat16 bias_stage[fz::kEpiWarps][fz::BN];  // each epilogue warp's copy of its tile's bias
    uint32_t tmem_base;
    int abort_flag;
    GroupTable g1, g2;
};

constexpr size_t fused_smem_bytes() { return 1024 + (size_t)fz::STAGES * fz::STAGE_BYTES + sizeof(FusedShared); }

// The gated combine for one pick per token (k = 1), done by the GEMM2 epilogue: row r of the
// expert-major output belongs to token src_token[r] alone, so the epilogue writes
// y[token] = bf16(fma(bf16(gate[token]), bf16(out_r), residual[token] or 0)) -- the same
// operations, in the same order, as the combine kernel applied to ybuf. y == nullptr: the
// epilogue writes ybuf instead.
struct FusedCombine {
    const int32_t* src_token;
    const float* gate;                 // [m] (k = 1)
    const __nv_bfloat16* residual;     // [m, d] or nullptr
    __nv_bfloat16* y;                  // [m, d] or nullptr
    int64_t m;
};

// Dispatch fused into the first GEMM (the GATHER instantiation): the GEMM1 A tiles are gathered
// straight from the token-major activations, row r of the expert-major order being
// x[src_token[r]], by four loader warps (16-byte cp.async into the 128-byte-swizzled K-major
// layout, a proxy fence, then an arrival on the stage's mbarrier), so xbuf is never formed.
// Measured slower than dispatch + TMA tile loads (the loaders cannot feed the tensor cores at
// the rate one TMA tile load per stage does); it saves the xbuf buffer, rows x d elements.
struct FusedGather {
    const __nv_bfloat16* x;     // [m, d] or nullptr (A tiles from xbuf by TMA)
    const int32_t* src_token;   // [rows]
    int64_t m;
};

struct FusedTile {
    int phase, e, n0, N, K, mtiles1;
    int64_t row0, row_end;
};

// Ticket order. Pair j = 0 .. n + L - 1 holds expert j's GEMM1 tiles (j < n) and then expert
// (j - L)'s GEMM2 tiles (j >= L), so an expert's second GEMM follows its first by L experts'
// worth of tiles; L = n puts every GEMM2 tile after every GEMM1 tile. For any L every GEMM2
// tile comes after all GEMM1 tiles of its expert in ticket order, which keeps the launch free
// of deadlock (tickets are taken in order, by running CTAs only).
__device__ __forceinline__ int pair_start(const FusedShared* sh, int n, int L, int j) {
    const int a = j < n ? j : n;
    int b = j - L;
    b = b < 0 ? 0 : (b > n ? n : b);
    return sh->g1.tile_start[a] + sh->g2.tile_start[b];
}
// ticket -> (phase, index of the tile in its phase's list)
__device__ __forceinline__ void ticket_decode(const FusedShared* sh, int n, int L, int ticket, int& phase, int& lt) {
    int lo = 0, hi = n + L;  // the largest pair j with pair_start(j) <= ticket
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pair_start(sh, n, L, mid) <= ticket) lo = mid;
        else hi = mid;
    }
    const int off = ticket - pair_start(sh, n, L, lo);
    const int len1 = lo < n ? sh->g1.tile_start[lo + 1] - sh->g1.tile_start[lo] : 0;
    if (off < len1) {
        phase = 1;
        lt = sh->g1.tile_start[lo] + off;
    } else {
        phase = 2;
        lt = sh->g2.tile_start[lo - L] + (off - len1);
    }
}

__device__ __forceinline__ FusedTile fused_decode(const FusedShared* sh, int ticket, int L, int n, int d, int d_ff) {
    FusedTile t;
    int lt;
    ticket_decode(sh, n, L, ticket, t.phase, lt);
    const GroupTable& g = t.phase == 1 ? sh->g1 : sh->g2;
    t.e = group_of_tile(g, n, lt);
    const int local = lt - g.tile_start[t.e];
    const int rows_e = g.row_start[t.e + 1] - g.row_start[t.e];
    const int mtiles = (rows_e + fz::BM - 1) / fz::BM;
    const int nt = local / mtiles, mt = local - nt * mtiles;
    t.row0 = (int64_t)g.row_start[t.e] + (int64_t)mt * fz::BM;
    t.row_end = g.row_start[t.e + 1];
    t.n0 = nt * fz::BN;
    t.N = t.phase == 1 ? d_ff : d;
    t.K = t.phase == 1 ? d : d_ff;
    t.mtiles1 = mtiles;
    return t;
}

template <bool GATHER>
__global__ void __launch_bounds__(fz::threads(GATHER), 1)
ffn_fused_tc(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w1,
             const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w2,
             const __nv_bfloat16* __restrict__ b1, const __nv_bfloat16* __restrict__ b2,
             const int32_t* __restrict__ offsets, int n, int d, int d_ff, int64_t max_rows,
             __nv_bfloat16* __restrict__ h, __nv_bfloat16* __restrict__ y, int* __restrict__ done1,
             int* __restrict__ next_tile, FusedCombine cmb, FusedGather gth) {
    using namespace fz;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    FusedShared* sh = reinterpret_cast<FusedShared*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntn1 = (d_ff + BN - 1) / BN, ntn2 = (d + BN - 1) / BN;

    if (threadIdx.x == 0) {
        const bool gather = GATHER;
        // full: the producer's arrival (+ TMA bytes), and with the gather the 128 loader threads'
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&sh->full[s], 1 + (gather ? 32 * kLoadWarps : 0));
            ptx::mbar_init(&sh->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) { ptx::mbar_init(&sh->tfull[b], 1); ptx::mbar_init(&sh->tempty[b], 128); }
        for (int r = 0; r < RING; ++r) {
            ptx::mbar_init(&sh->tready[r], 1);
            ptx::mbar_init(&sh->tfree[r], 1 + kEpiWarps + (gather ? kLoadWarps : 0));
        }
        sh->abort_flag = 0;
        ptx::fence_barrier_init();
        ptx::prefetch_tensormap(&map_x);
        ptx::prefetch_tensormap(&map_w1);
        ptx::prefetch_tensormap(&map_h);
        ptx::prefetch_tensormap(&map_w2);
    }
    if (warp == 1) ptx::tmem_alloc(&sh->tmem_base, TMEM_COLS);
    pdl_wait();  // expert_offsets, xbuf and the counters come from earlier launches
    if (warp == 2) build_group_table(offsets, n, ntn1, BM, max_rows, sh->g1);
    if (warp == 3) build_group_table(offsets, n, ntn2, BM, max_rows, sh->g2);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = sh->tmem_base;
    const int T1 = sh->g1.tile_start[n];
    const int total = T1 + sh->g2.tile_start[n];
    // Lag between an expert's two GEMMs. A lag of about one wave was measured: it kept h in L2 but
    // GEMM2 producers then waited on GEMM1 tiles still in flight (each producer runs up to RING
    // tiles ahead) and the launch got slower, so every GEMM2 tile follows every GEMM1 tile.
    const int L = n;
    volatile int* abort_flag = &sh->abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0, slot = 0;
            uint32_t phase = 0, rphase = 0;
            const uint64_t wpolicy = ptx::l2_policy_evict_first();
            for (;;) {
                // take the next tile of the launch and hand its id to the MMA and epilogue warps
                if (!ptx::mbar_wait(&sh->tfree[slot], rphase ^ 1u, abort_flag)) break;
                const int tile = atomicAdd(next_tile, 1);
                sh->tile_ring[slot] = tile < total ? tile : -1;
                ptx::mbar_arrive(&sh->tready[slot]);
                if (++slot == RING) { slot = 0; rphase ^= 1u; }
                if (tile >= total) break;
                const FusedTile t = fused_decode(sh, tile, L, n, d, d_ff);
                if (t.phase == 2) {
                    // all GEMM1 tiles of expert e, each signalled by its 4 epilogue warps
                    const int rows_e = sh->g1.row_start[t.e + 1] - sh->g1.row_start[t.e];
                    const int need = ((rows_e + BM - 1) / BM) * ntn1 * kEpiWarps;
                    if (!ptx::wait_count_geq(done1 + t.e, need, abort_flag, ptx::kWaitCycles)) break;
                    ptx::fence_proxy_async_global();
                }
                const CUtensorMap* ma = t.phase == 1 ? &map_x : &map_h;
                const CUtensorMap* mb = t.phase == 1 ? &map_w1 : &map_w2;
                const int nkb = (t.K + BK - 1) / BK;
                const bool a_by_tma = t.phase == 2 || !GATHER;  // else the loader warps gather A
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    ptx::mbar_expect_tx(&sh->full[stage], a_by_tma ? STAGE_BYTES : B_BYTES);
                    if (a_by_tma) ptx::tma_load_2d(sa, ma, &sh->full[stage], kb * BK, (int)t.row0);
                    // an expert with one row tile reads each weight tile once: evict-first, so the
                    // hidden rows h that the GEMM2 tiles read back stay in L2 (with more row tiles
                    // the weight tiles are re-read and keep the normal policy)
                    if (t.mtiles1 == 1)
                        ptx::tma_load_3d_hint(sa + A_BYTES, mb, &sh->full[stage], kb * BK, t.n0, t.e, wpolicy);
                    else
                        ptx::tma_load_3d(sa + A_BYTES, mb, &sh->full[stage], kb * BK, t.n0, t.e);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, acc = 0, slot = 0;
            uint32_t phase = 0, aphase = 0, rphase = 0;
            for (;;) {
                if (!ptx::mbar_wait(&sh->tready[slot], rphase, abort_flag)) break;
                const int tile = *(volatile int*)&sh->tile_ring[slot];
                ptx::mbar_arrive(&sh->tfree[slot]);
                if (++slot == RING) { slot = 0; rphase ^= 1u; }
                if (tile < 0) break;
                const FusedTile t = fused_decode(sh, tile, L, n, d, d_ff);
                const int nkb = (t.K + BK - 1) / BK;
                const uint32_t idesc = t.N - t.n0 <= BN / 2 ? IDESC_HALF : IDESC;
                if (!ptx::mbar_wait(&sh->tempty[acc], aphase ^ 1u, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t tmem_d = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!ptx::mbar_wait(&sh->full[stage], phase, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(smem + stage * STAGE_BYTES);
                    const uint64_t adesc = ptx::sw128_kmajor_desc(sa);
                    const uint64_t bdesc = ptx::sw128_kmajor_desc(sa + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        ptx::umma_bf16(tmem_d, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
                    ptx::umma_commit(&sh->empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::umma_commit(&sh->tfull[acc]);
                if (++acc == 2) { acc = 0; aphase ^= 1u; }
            }
        }
    } else if (warp >= 2 + kEpiWarps) {
        // row gather (warps 6-9): thread l copies row l of each GEMM1 A tile, 8 x 16 bytes per
        // K block, from x[src_token[row]] (zeros past the expert's rows or past d); the arrival
        // for a stage waits until the next stage's copies are issued, so two are in flight
        if (GATHER) {
            const int ltid = (warp - 2 - kEpiWarps) * 32 + lane;
            int stage = 0, slot = 0, pend = -1;
            uint32_t phase = 0, rphase = 0;
            bool ok = true;
            for (;;) {
                bool w = true;
                if (lane == 0) w = ptx::mbar_wait(&sh->tready[slot], rphase, abort_flag);
                if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
                const int tile = *(volatile int*)&sh->tile_ring[slot];
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sh->tfree[slot]);
                if (++slot == RING) { slot = 0; rphase ^= 1u; }
                if (tile < 0) break;
                const FusedTile t = fused_decode(sh, tile, L, n, d, d_ff);
                const int64_t r = t.row0 + ltid;
                bool valid = t.phase == 1 && r < t.row_end;
                int64_t tok = 0;
                if (valid) {
                    tok = gth.src_token[r];
                    if (tok < 0 || tok >= gth.m) { record_error(kErrTokenIndex); valid = false; tok = 0; }
                }
                const __nv_bfloat16* xrow = gth.x + tok * d;
                const int nkb = (t.K + BK - 1) / BK;
                for (int kb = 0; kb < nkb; ++kb) {
                    bool e = true;
                    if (lane == 0) e = ptx::mbar_wait(&sh->empty[stage], phase ^ 1u, abort_flag);
                    if (!__shfl_sync(0xffffffffu, e, 0)) { ok = false; break; }
                    if (t.phase == 1) {
                        const uint32_t dst = ptx::smem_u32(smem + stage * STAGE_BYTES) + (uint32_t)ltid * 128u;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int col = kb * BK + c * 8;
                            const bool in = valid && col < d;
                            ptx::cp_async16(dst + ((uint32_t)(c ^ (ltid & 7)) << 4), in ? (const void*)(xrow + col)
                                                                                         : (const void*)gth.x,
                                            in ? 16u : 0u);
                        }
                    }
                    ptx::cp_async_commit();
                    if (pend >= 0) {
                        ptx::cp_async_wait_group<1>();
                        ptx::fence_proxy_async_shared();
                        ptx::mbar_arrive(&sh->full[pend]);
                    }
                    pend = stage;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            if (ok && pend >= 0) {
                ptx::cp_async_wait_group<0>();
                ptx::fence_proxy_async_shared();
                ptx::mbar_arrive(&sh->full[pend]);
            }
        }
    } else {
        const int quad = warp & 3;
        int acc = 0, slot = 0;
        uint32_t aphase = 0, rphase = 0;
        for (;;) {
            // every lane waits; the warp leaves together if any lane gave up (a timeout): the
            // warp-collective TMEM loads below need all 32 lanes
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sh->tready[slot], rphase, abort_flag))) break;
            const int tile = *(volatile int*)&sh->tile_ring[slot];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sh->tfree[slot]);
            if (++slot == RING) { slot = 0; rphase ^= 1u; }
            if (tile < 0) break;
            const FusedTile t = fused_decode(sh, tile, L, n, d, d_ff);
            // stage the tile's 256 bias values in shared memory while the accumulator fills
            __nv_bfloat16* be = sh->bias_stage[warp - 2];
            {
                const __nv_bfloat16* gb = (t.phase == 1 ? b1 : b2) + (int64_t)t.e * t.N;
                const int col = t.n0 + lane * 8;
                if (col < t.N)
                    *reinterpret_cast<uint4*>(be + lane * 8) = *reinterpret_cast<const uint4*>(gb + col);
                __syncwarp();
            }
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&sh->tfull[acc], aphase, abort_flag))) break;
            ptx::tc_fence_after();
            const int64_t r = t.row0 + quad * 32 + lane;
            bool row_ok = r < t.row_end;
            const bool relu = t.phase == 1;
            __nv_bfloat16* out = t.phase == 1 ? h : y;
            // combined output: this row goes straight to its token's row of y, scaled by its gate
            const bool comb = t.phase == 2 && cmb.y != nullptr;
            int64_t tok = 0;
            float gk = 0.f;
            if (comb && row_ok) {
                tok = cmb.src_token[r];
                if (tok < 0 || tok >= cmb.m) {
                    record_error(kErrTokenIndex);
                    row_ok = false;
                } else {
                    gk = round_to_bf16(cmb.gate[tok]);
                }
            }
            // two 32-column chunks in flight per wait
            for (int c2 = 0; c2 < BN / 32; c2 += 2) {
                const int colA = t.n0 + c2 * 32;
                if (colA >= t.N) break;  // warp-uniform
                const bool hasB = colA + 32 < t.N;
                uint32_t v2[2][32];
                const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN + c2 * 32);
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
                    Vec16<__nv_bfloat16>::load(be + (col - t.n0), bv);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        f[q] = __uint_as_float(v[g8 * 8 + q]) + bv[q];
                        if (relu) f[q] = fmaxf(f[q], 0.f);
                    }
                    if (!row_ok) continue;
                    if (comb) {
                        float acc[8];
                        if (cmb.residual) {
                            Vec16<__nv_bfloat16>::load(cmb.residual + tok * t.N + col, acc);
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[q] = fmaf(gk, round_to_bf16(f[q]), acc[q]);
                        Vec16<__nv_bfloat16>::store(cmb.y + tok * t.N + col, acc);
                    } else {
                        Vec16<__nv_bfloat16>::store(out + r * t.N + col, f);
                    }
                }
              }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sh->tempty[acc]);
            if (t.phase == 1) {
                // publish this warp's h rows to the TMA loads of the GEMM2 tiles of expert e
                ptx::fence_proxy_async_global();
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(done1 + t.e, 1);
                }
            }
            if (++acc == 2) { acc = 0; aphase ^= 1u; }
        }
    }
    pdl_trigger();  // the dependent launch may start while this grid drains
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// y rows of tokens whose pick was dropped (k = 1, dest_row < 0): the residual, or zeros. CTA 0
// also clears the FFN's tile counters (the FFN launch that follows waits for this one), so no
// memset sits between the launches.
__global__ void __launch_bounds__(256)
combine_dropped_kernel(const int32_t* __restrict__ dest_row, const uint4* __restrict__ residual, int64_t m,
                       int64_t vec_per_row, uint4* __restrict__ y, int* __restrict__ counters, int ncounters) {
    const int lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();
    if (blockIdx.x == 0)
        for (int c = threadIdx.x; c < ncounters; c += blockDim.x) counters[c] = 0;
    const int64_t warps = (int64_t)gridDim.x * 8;
    for (int64_t i0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * 32; i0 < m; i0 += warps * 32) {
        const int64_t i = i0 + lane;
        const bool dropped = i < m && dest_row[i] < 0;
        uint32_t mask = __ballot_sync(0xffffffffu, dropped);
        while (mask) {  // the warp copies (or clears) each dropped row of its 32 tokens
            const int b = __ffs(mask) - 1;
            mask &= mask - 1;
            const int64_t tok = i0 + b;
            for (int64_t c = lane; c < vec_per_row; c += 32)
                y[tok * vec_per_row + c] = residual ? residual[tok * vec_per_row + c] : make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

cudaError_t launch_combine_dropped(const int32_t* dest_row, const void* residual, int64_t m, int d, void* y,
                                   int* counters, int ncounters, cudaStream_t stream) {
    if (m == 0) return cudaSuccess;
    int64_t blocks = (m + 255) / 256;
    if (blocks > (int64_t)num_sms() * 4) blocks = (int64_t)num_sms() * 4;
    return launch_pdl(combine_dropped_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, dest_row,
                      static_cast<const uint4*>(residual), m, (int64_t)d * 2 / 16, static_cast<uint4*>(y), counters,
                      ncounters);
}

// xbuf: the expert-major rows [max_rows, d], or with gth the token-major x [gth->m, d] whose
// rows the kernel gathers by gth->src_token.
cudaError_t launch_ffn_fused(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                             const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                             int* counters, cudaStream_t stream, const FusedCombine* cmb = nullptr,
                             bool zero_counters = true, const FusedGather* gth = nullptr) {
    CUtensorMap mx, mw1, mh, mw2;
    const uint64_t xrows = gth ? (uint64_t)gth->m : (uint64_t)max_rows;  // the A map is unused when gathering
    if (!map_2d(&mx, xbuf, xrows, (uint64_t)d, fz::BM)) return cudaErrorInvalidValue;
    if (!map_3d(&mw1, w1, (uint64_t)n, (uint64_t)d_ff, (uint64_t)d, fz::BN)) return cudaErrorInvalidValue;
    if (!map_2d(&mh, hbuf, (uint64_t)max_rows, (uint64_t)d_ff, fz::BM)) return cudaErrorInvalidValue;
    if (!map_3d(&mw2, w2, (uint64_t)n, (uint64_t)d, (uint64_t)d_ff, fz::BN)) return cudaErrorInvalidValue;
    static bool attr = false;
    const size_t smem = fused_smem_bytes();
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(ffn_fused_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(ffn_fused_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    // counters[0..n-1]: GEMM1 completions per expert; counters[n]: next tile ticket
    if (zero_counters) {
        cudaError_t e = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)(n + 1), stream);
        if (e != cudaSuccess) return e;
    }
    const FusedCombine c = cmb ? *cmb : FusedCombine{nullptr, nullptr, nullptr, nullptr, 0};
    if (gth)
        return launch_pdl(ffn_fused_tc<true>, dim3(num_sms()), dim3(fz::threads(true)), smem, stream, mx, mw1, mh,
                          mw2, static_cast<const __nv_bfloat16*>(b1), static_cast<const __nv_bfloat16*>(b2), offsets,
                          n, d, d_ff, max_rows, static_cast<__nv_bfloat16*>(hbuf), static_cast<__nv_bfloat16*>(ybuf),
                          counters, counters + n, c, *gth);
    return launch_pdl(ffn_fused_tc<false>, dim3(num_sms()), dim3(fz::threads(false)), smem, stream, mx, mw1, mh, mw2,
                      static_cast<const __nv_bfloat16*>(b1), static_cast<const __nv_bfloat16*>(b2), offsets, n, d,
                      d_ff, max_rows, static_cast<__nv_bfloat16*>(hbuf), static_cast<__nv_bfloat16*>(ybuf), counters,
                      counters + n, c, FusedGather{nullptr, nullptr, 0});
}

// Both GEMMs in one persistent launch; its counters (per-expert completions, tile ticket) follow h.
static int* ffn_counters(void* hbuf, int64_t max_rows, int d_ff) {
    const size_t hbytes = ((size_t)max_rows * (size_t)d_ff * 2 + 255) & ~(size_t)255;
    return reinterpret_cast<int*>(static_cast<char*>(hbuf) + hbytes);
}

cudaError_t launch_ffn_pair(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                            const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                            int* counters, cudaStream_t stream);

// moe_expert_ffn in bf16: the two-SM tiles of ffn_pair.cu (the one-SM kernel here serves the
// fused-combine and row-gather variants).
cudaError_t launch_ffn_tc(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                          const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                          cudaStream_t stream) {
    return launch_ffn_pair(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf,
                           ffn_counters(hbuf, max_rows, d_ff), stream);
}

// The FFN reading its rows straight from x by src_token (the dispatch fused into the first GEMM).
cudaError_t launch_ffn_tc_gather(const void* x, const int32_t* src_token, int64_t m, const void* w1, const void* b1,
                                 const void* w2, const void* b2, const int32_t* offsets, int n, int d, int d_ff,
                                 int64_t max_rows, void* ybuf, void* hbuf, cudaStream_t stream) {
    const FusedGather gth{static_cast<const __nv_bfloat16*>(x), src_token, m};
    return launch_ffn_fused(x, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf,
                            ffn_counters(hbuf, max_rows, d_ff), stream, nullptr, true, &gth);
}

// The FFN with the k = 1 gated combine in its GEMM2 epilogue, plus the dropped tokens' rows.
cudaError_t launch_ffn_tc_combine(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                                  const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* hbuf,
                                  const int32_t* src_token, const int32_t* dest_row, const float* gate,
                                  const void* residual, int64_t m, void* y, cudaStream_t stream) {
    // the dropped rows' kernel also clears the FFN's counters, so the FFN directly follows a
    // kernel (programmatic dependent launch) and no memset sits in the chain
    int* counters = ffn_counters(hbuf, max_rows, d_ff);
    cudaError_t e = launch_combine_dropped(dest_row, residual, m, d, y, counters, max_rows > 0 ? n + 1 : 0, stream);
    if (e != cudaSuccess || max_rows == 0) return e;
    const FusedCombine cmb{src_token, gate, static_cast<const __nv_bfloat16*>(residual),
                           static_cast<__nv_bfloat16*>(y), m};
    return launch_ffn_fused(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, nullptr, hbuf, counters, stream,
                            &cmb, false);
}

}  // namespace moe
