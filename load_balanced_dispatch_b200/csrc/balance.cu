// balance.cu -- optimal-assignment balancing (Quantile Balancing) and its exact finish.
//
// MoE travelogue 6: optimal assignment promotes balance (kexue.fm/archives/11619):
// the balance LP (3)/(4), its dual (8), the alternating updates
//   alpha_i = threshold between the k-th and (k+1)-th largest of s_i - beta,
//   beta_j  = threshold between the C-th and (C+1)-th largest of s_:j - alpha,
// the QB algorithm box and its one-step practical form (select with the old
// beta, then update). Both thresholds are computed in fp32 exactly as defined
// (v = fp32(s - beta), u = fp32(s - alpha), midpoint fp32(fp32(a + b) * 0.5)),
// so every decision is reproducible bit for bit.
//
// Kernels:
//   qb_row_tpr2 the row pass, one thread per token (when k + 1 <= the number of
//              column groups): a warp reads 32 rows coalesced and forms the
//              row's 32 column-group maxima of v = s - beta; T, the (k+1)-th
//              largest of them, bounds the row's (k+1)-th value from below; the
//              thread lists its row's elements at or above T (or the lower T'
//              that also covers the window sweep), sorts their keys and takes
//              the top-k set (ascending expert order), the k-th and (k+1)-th
//              values (alpha) and a tie flag. Before a column pass it also runs
//              that pass's window sweep on the listed elements (keys of
//              u = s - alpha above a window around the current beta_j counted,
//              those inside listed), and in the sign step it counts
//              fp32(s - alpha) > beta_j, so s is read once per iteration.
//   qb_row_tpr the same selection on rows staged in shared memory, for the
//              first row pass of a SOLVE, which also writes s transposed
//              (sT [n, m]) for the column pass's full path.
//   qb_row     one warp per token (k + 1 above the group count, and rows whose
//              list overflows): the lane maxima bound the (k+1)-th key, the
//              keys reaching it are ranked (k + 1 rounds of a warp arg-max when
//              more than 32 reach it).
//   qb_col     one CTA per expert column: when the C-th largest fell inside
//              the window, the C-th and (C+1)-th largest come from the column's
//              list (radix digits over order-preserving uint32 keys); otherwise
//              an exact radix select over the whole column (from sT, or from s
//              with stride n).
//   repair     successive shortest paths on the n-expert graph (exact finish
//              when the QB iterate is not yet balanced): arc a -> b costs
//              W[a][b] = min over tokens i holding a but not b of s_ia - s_ib
//              (fp64, lowest token on ties); an 8-CTA cluster (W's columns
//              split over the CTAs' shared memory) runs Jacobi Bellman-Ford
//              rounds from the over-full experts, picks the nearest under-full
//              expert (lowest index on ties), follows predecessors settled in
//              an earlier round back to an over-full expert and moves each
//              arc's argmin token. The number of moves equals the excess, so the host
//              enqueues exactly that many rounds without waiting in between.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace qb {
constexpr int kRowThreads = 256;
constexpr int kRowTile = 32;      // rows of s per shared-memory tile of the row pass (one bulk copy)
constexpr int kColThreads = 512;  // qb_col_kernel block size (its scan buffer is sized by it)
// status words kept in the workspace
// kStDone: repair finished; kStQbDone: a row pass found every count equal to C (later passes return at once);
// kStIters: beta updates done; kStTies0/1: tie counts of the row passes (ping-pong with the counts buffers)
enum { kStDone = 0, kStAugments = 1, kStError = 2, kStQbDone = 4, kStIters = 5, kStTies0 = 6, kStTies1 = 7,
       kStWords = 8 };
constexpr int kBatch = 16;  // QB iterations enqueued between host checks
constexpr int kRowPairCap = 512;  // window pairs buffered per row-pass CTA (flushed at tile boundaries)
constexpr int64_t kMaxMiniBatches = 4096;  // mini-batches of one averaged-beta step
}  // namespace qb

namespace qb {
constexpr int kCandCap = 16384;                         // candidate keys kept in shared memory
constexpr int kColUnroll = 4;                           // float4 pairs in flight per thread in a column sweep
constexpr int kGCap = 8192;                             // window candidates kept per column (global lists)
constexpr size_t kColSmem = 4096 * 4 + kColThreads * 4 + kCandCap * 4;
// key-space half-widths of the window around the previous beta_j
// kWinSweep: the sweep's windows are at most this wide
constexpr uint32_t kWinDefault = 1u << 18, kWinMin = 1u << 12, kWinMax = 1u << 26, kWinSweep = 1u << 21;
}  // namespace qb

// Threshold between the q-th (a) and (q+1)-th (b) largest: midpoint, the (q+1)-th, or the
// (q+1)-th clipped at zero (BIP's non-negative duals).
__device__ __forceinline__ float qb_threshold(float a, float b, int rule) {
    if (rule == MOE_QB_BOUNDARY) return b;
    if (rule == MOE_QB_BIP) return b > 0.f ? b : 0.f;
    return __fmul_rn(__fadd_rn(a, b), 0.5f);
}

// order-preserving key: larger float -> larger key; -0 is folded onto +0
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t b = __float_as_uint(f);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// float_key with -0 folded by an IEEE add of +0 (branch-free; the same key for every float)
__device__ __forceinline__ uint32_t float_key_nz(float f) {
    const uint32_t b = __float_as_uint(__fadd_rn(f, 0.0f));
    return b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
}

// Top-(k+1) of one row held by a warp: lane owns j = lane + 32 q (q < NT); key = float_key(v),
// 0 for j >= n (every real key is above 0). Output: `taken` (bit q: j = lane + 32 q is among the
// k best), the k-th and (k+1)-th best values vk, vk1. Ranking: larger key first, equal keys by
// lower j.
//
// Rounds: each of the k + 1 rounds takes the best untaken key: a lane-local scan (lowest q on
// ties), __reduce_max_sync over keys, __reduce_min_sync over the candidate indices.
template <int NT>
__device__ __forceinline__ void row_topk_rounds(const uint32_t (&key)[NT], const float (&v)[NT], int n, int k,
                                                uint32_t& taken, float& vk, float& vk1) {
    const int lane = threadIdx.x & 31;
    taken = 0;
    vk = vk1 = 0.f;
    for (int r = 0; r <= k; ++r) {
        uint32_t lb = 0;
        int lq = -1;
        float lv = 0.f;
#pragma unroll
        for (int q = 0; q < NT; ++q)
            if (!((taken >> q) & 1u) && key[q] > lb) { lb = key[q]; lq = q; lv = v[q]; }
        const uint32_t mx = __reduce_max_sync(0xffffffffu, lb);
        const uint32_t cand = (lq >= 0 && lb == mx) ? (uint32_t)(lq * 32 + lane) : 0xffffffffu;
        const uint32_t wj = __reduce_min_sync(0xffffffffu, cand);
        const float wv = __shfl_sync(0xffffffffu, lv, (int)(wj & 31u));
        if (r < k && wj < (uint32_t)n && (int)(wj & 31u) == lane) taken |= 1u << (wj >> 5);
        if (r == k - 1) vk = wv;
        if (r == k) vk1 = wv;
    }
}

// Same result, far fewer instructions (k < 32, k < n), and the picks are written here.
// T = the (k+1)-th largest of the 32 lane maxima, counted with multiplicity, is a lower bound of
// the row's (k+1)-th largest key: k + 1 distinct keys reach it. So every pick has key >= T.
// When at most 32 keys reach T, they are gathered one per lane in ascending j through this
// warp's 32 shared slots. Each candidate's rank is then the number of candidates ranking before
// it (a larger key, or an equal key at a lower j, that is at a lower slot). Ranks below k are
// the picks, already in ascending j, and ranks k - 1 and k give vk and vk1.
// Returns false, with nothing written, when more than 32 keys reach T.
template <int NT>
__device__ __forceinline__ bool row_topk_ranked(const uint32_t (&key)[NT], const float (&v)[NT], int k, int64_t i,
                                                uint32_t* sk, int* sj, float* sv, int32_t* __restrict__ topk_idx,
                                                int* cnt, float& vk, float& vk1) {
    const int lane = threadIdx.x & 31;
    const uint32_t full = 0xffffffffu, lt = (1u << lane) - 1u;
    uint32_t cur = 0;
#pragma unroll
    for (int q = 0; q < NT; ++q) cur = max(cur, key[q]);
    // remove the largest remaining lane maximum k times (one lane at a time); T = the next one
    for (int r = 0; r < k; ++r) {
        const uint32_t mx = __reduce_max_sync(full, cur);
        const uint32_t own = __ballot_sync(full, cur == mx);
        if (lane == __ffs(own) - 1) cur = 0;
    }
    uint32_t T = __reduce_max_sync(full, cur);
    if (T == 0) T = 1;  // fewer than k + 1 lanes hold keys: every key is a candidate
    // gather the keys >= T in ascending j (q-major, then lane)
    int N = 0;
#pragma unroll
    for (int q = 0; q < NT; ++q) {
        const bool c = key[q] >= T;
        const uint32_t b = __ballot_sync(full, c);
        const int pos = N + __popc(b & lt);
        N += __popc(b);
        if (c && pos < 32) { sk[pos] = key[q]; sj[pos] = lane + 32 * q; sv[pos] = v[q]; }
    }
    if (N > 32) return false;
    __syncwarp();
    const bool has = lane < N;
    const uint32_t ck = has ? sk[lane] : 0u;
    const int cj = has ? sj[lane] : 0;
    const float cv = has ? sv[lane] : 0.f;
    __syncwarp();
    int rank = 0;
    for (int c = 0; c < N; ++c) {
        const uint32_t kc = __shfl_sync(full, ck, c);
        rank += (kc > ck || (kc == ck && c < lane)) ? 1 : 0;
    }
    const bool pick = has && rank < k;
    const uint32_t pb = __ballot_sync(full, pick);
    if (pick) {
        topk_idx[i * k + __popc(pb & lt)] = cj;
        atomicAdd(&cnt[cj], 1);
    }
    const uint32_t bk = __ballot_sync(full, has && rank == k - 1);
    const uint32_t bk1 = __ballot_sync(full, has && rank == k);
    vk = __shfl_sync(full, cv, __ffs(bk) - 1);
    vk1 = __shfl_sync(full, cv, __ffs(bk1) - 1);
    return true;
}

// One warp per token. CTAs stream tiles of kRowTile consecutive rows of s into shared memory
// with bulk copies, two tiles in flight (double buffer, one mbarrier each; the partial last tile
// and unaligned inputs take plain loads), so the selection reads its rows from shared memory.
// Each row takes the ranked selection, or the plain rounds when it does not apply. beta for the
// lane's columns stays in registers. TRANS: the tile is also written out transposed (sT [n, m],
// each expert's column contiguous) for the column pass's full path.
// The window sweep of the column pass, done by the row pass on the rows it holds (SWEEP): once a
// warp has alpha_i, the keys of u_ij = fp32(s_ij - alpha_i) of its row are compared with a window
// [lo_j, hi_j] around the current beta_j (half-width min(win_j, kWinSweep), the previous select's
// width): keys above the window are counted (per lane, per column) and keys inside it are
// buffered in shared memory as (column, key) pairs, which the CTA appends to the column's global
// candidate list (g_cand[j], kGCap long, count g_ncand[j]) at tile boundaries once the buffer is
// half full, and at the end. A column whose pairs do not fit is marked full (its count pushed
// past kGCap), so the select takes the exact full path. This removes the second read of s.
struct RowSweep {
    const uint32_t* win;   // [n] window half-widths (0: default)
    uint32_t* g_above;     // [n] keys above the window
    uint32_t* g_ncand;     // [n] keys inside it
    uint32_t* g_cand;      // [n][kGCap] the keys inside it
};

// Append the CTA's buffered (column, key) pairs to the global candidate lists (all threads); the
// buffer holds min(*npairs, cap) pairs.
__device__ __forceinline__ void sweep_flush(const uint2* pairs, unsigned* npairs, uint32_t* scnt, uint32_t* sbase,
                                            unsigned char* sfull, int n, const RowSweep& sw,
                                            unsigned cap = (unsigned)qb::kRowPairCap) {
    const int tid = threadIdx.x, T = blockDim.x;
    const unsigned np = min(*npairs, cap);
    for (unsigned p = tid; p < np; p += T) atomicAdd(&scnt[pairs[p].x], 1u);
    __syncthreads();
    for (int j = tid; j < n; j += T) {
        // a full column: its count goes past kGCap, its pairs are not stored
        const uint32_t add = sfull[j] ? scnt[j] + (uint32_t)qb::kGCap + 1u : scnt[j];
        sbase[j] = add ? atomicAdd(&sw.g_ncand[j], add) : 0u;
        if (sfull[j]) sbase[j] = (uint32_t)qb::kGCap;
        scnt[j] = 0;
    }
    __syncthreads();
    for (unsigned p = tid; p < np; p += T) {
        const uint2 pr = pairs[p];
        const uint32_t pos = sbase[pr.x] + atomicAdd(&scnt[pr.x], 1u);
        if (pos < (uint32_t)qb::kGCap) sw.g_cand[(int64_t)pr.x * qb::kGCap + pos] = pr.y;
    }
    __syncthreads();
    for (int j = tid; j < n; j += T) { scnt[j] = 0; sfull[j] = 0; }
    if (tid == 0) *npairs = 0;
    __syncthreads();
}

template <int NT, bool TRANS, bool SWEEP>
__global__ void __launch_bounds__(qb::kRowThreads, 3)
qb_row_kernel(const float* __restrict__ s, int64_t m, int n, int k, const float* __restrict__ beta, int rule,
              float* __restrict__ alpha, int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts,
              int32_t* __restrict__ status, int tie_slot, int skip_if_done, float* __restrict__ sT, int bulk,
              RowSweep sw) {
    if (skip_if_done && *(volatile int32_t*)&status[qb::kStQbDone]) return;
    constexpr int RT = qb::kRowTile;
    extern __shared__ __align__(128) float rtile[];  // [2][RT * n]
    __shared__ __align__(8) uint64_t bar[2];
    __shared__ int cnt[kMaxExperts];
    __shared__ int nties;
    __shared__ int abort_flag;
    __shared__ uint32_t s_key[qb::kRowThreads];
    __shared__ int s_j[qb::kRowThreads];
    __shared__ float s_v[qb::kRowThreads];
    // window sweep: buffered pairs and per-column scratch of the flush
    __shared__ uint2 pairs[SWEEP ? qb::kRowPairCap : 1];
    __shared__ uint32_t scnt[SWEEP ? kMaxExperts : 1], sbase[SWEEP ? kMaxExperts : 1];
    __shared__ unsigned char sfull[SWEEP ? kMaxExperts : 1];
    __shared__ unsigned npairs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wbase = tid & ~31;  // this warp's 32 shared slots
    const int64_t ntiles = (m + RT - 1) / RT;
    const int64_t tile_floats = (int64_t)RT * n;
    const uint32_t tile_bytes = (uint32_t)(tile_floats * sizeof(float));
    for (int j = tid; j < n; j += blockDim.x) cnt[j] = 0;
    if (SWEEP)
        for (int j = tid; j < n; j += blockDim.x) { scnt[j] = 0; sfull[j] = 0; }
    if (tid == 0) {
        nties = 0;
        npairs = 0;
        abort_flag = 0;
        ptx::mbar_init(&bar[0], 1);
        ptx::mbar_init(&bar[1], 1);
        ptx::fence_barrier_init();
    }
    __syncthreads();
    float bq[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) bq[q] = lane + 32 * q < n ? beta[lane + 32 * q] : 0.f;
    // the lane's windows (padding columns get lo = hi = the largest key, which no float reaches)
    uint32_t lo[NT], hi[NT], above[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) {
        above[q] = 0;
        lo[q] = hi[q] = 0xffffffffu;
        const int j = lane + 32 * q;
        if (SWEEP && j < n) {
            const uint32_t pk = float_key(bq[q]);
            uint32_t w = sw.win[j] ? sw.win[j] : qb::kWinDefault;
            if (w > qb::kWinSweep) w = qb::kWinSweep;
            lo[q] = pk > w ? pk - w : 0u;
            hi[q] = pk < 0xffffffffu - w ? pk + w : 0xffffffffu;
        }
    }
    const uint32_t lt = (1u << lane) - 1u;
    const bool prune = k < 32 && k < n;
    // copies issued and consumed per buffer (thread 0's bookkeeping, for a clean exit on abort)
    int issued[2] = {0, 0}, consumed[2] = {0, 0};
    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            const int64_t t = blockIdx.x + (int64_t)b * gridDim.x;
            if (bulk && t < ntiles && (t + 1) * RT <= m) {
                ptx::mbar_expect_tx(&bar[b], tile_bytes);
                ptx::bulk_load(rtile + b * tile_floats, s + t * tile_floats, tile_bytes, &bar[b]);
                ++issued[b];
            }
        }
    }
    int u = 0;
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++u) {
        const int b = u & 1;
        float* tl = rtile + b * tile_floats;
        const int64_t i0 = t * RT;
        const int rows = (int)min((int64_t)RT, m - i0);
        if (bulk && rows == RT) {
            ptx::mbar_wait(&bar[b], (uint32_t)((u >> 1) & 1), &abort_flag);
            if (tid == 0) ++consumed[b];
        } else {
            for (int64_t q = tid; q < (int64_t)rows * n; q += blockDim.x) tl[q] = s[i0 * n + q];
        }
        __syncthreads();
        if (abort_flag) break;  // the same value in every thread after the barrier
        if (TRANS) {
            // thread j stores column j of the tile's rows: 16-byte pieces when they are aligned
            for (int j = tid; j < n; j += blockDim.x) {
                float* dst = sT + (int64_t)j * m + i0;
                if (rows == RT && ((reinterpret_cast<uintptr_t>(dst) & 15) == 0)) {
#pragma unroll
                    for (int r4 = 0; r4 < RT; r4 += 4)
                        *reinterpret_cast<float4*>(dst + r4) =
                            make_float4(tl[r4 * n + j], tl[(r4 + 1) * n + j], tl[(r4 + 2) * n + j],
                                        tl[(r4 + 3) * n + j]);
                } else {
                    for (int r = 0; r < rows; ++r) dst[r] = tl[r * n + j];
                }
            }
        }
        for (int r = warp; r < rows; r += qb::kRowThreads / 32) {
            const int64_t i = i0 + r;
            const float* row = tl + r * n;
            float v[NT];
            uint32_t key[NT];
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const int j = lane + 32 * q;
                const bool ok = j < n;
                v[q] = ok ? __fsub_rn(row[j], bq[q]) : 0.f;
                key[q] = ok ? float_key(v[q]) : 0u;
            }
            float vk, vk1;
            if (!(prune && row_topk_ranked<NT>(key, v, k, i, s_key + wbase, s_j + wbase, s_v + wbase, topk_idx, cnt,
                                               vk, vk1))) {
                uint32_t taken;
                row_topk_rounds<NT>(key, v, n, k, taken, vk, vk1);
                int pos = 0;
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const bool bit = (taken >> q) & 1u;
                    const uint32_t mask = __ballot_sync(0xffffffffu, bit);
                    if (bit) {
                        topk_idx[i * k + pos + __popc(mask & lt)] = lane + 32 * q;
                        atomicAdd(&cnt[lane + 32 * q], 1);
                    }
                    pos += __popc(mask);
                }
            }
            if (lane == 0) {
                alpha[i] = qb_threshold(vk, vk1, rule);
                if (vk == vk1) atomicAdd(&nties, 1);
            }
            if (SWEEP) {
                // vk, vk1 are the same in every lane: so is alpha_i
                const float a = qb_threshold(vk, vk1, rule);
                uint32_t inw = 0;
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    if (lane + 32 * q < n) {
                        const uint32_t key = float_key_nz(__fsub_rn(row[lane + 32 * q], a));
                        above[q] += key > hi[q] ? 1u : 0u;
                        inw |= (key >= lo[q] && key <= hi[q]) ? (1u << q) : 0u;
                    }
                }
                if (__any_sync(0xffffffffu, inw != 0)) {
#pragma unroll
                    for (int q = 0; q < NT; ++q) {
                        if ((inw >> q) & 1u) {
                            const int j = lane + 32 * q;
                            const unsigned p = atomicAdd(&npairs, 1u);
                            if (p < (unsigned)qb::kRowPairCap)
                                pairs[p] = make_uint2((uint32_t)j, float_key_nz(__fsub_rn(row[j], a)));
                            else
                                sfull[j] = 1;
                        }
                    }
                }
            }
        }
        __syncthreads();  // every warp is done with the buffer
        if (SWEEP && npairs >= (unsigned)qb::kRowPairCap / 2) sweep_flush(pairs, &npairs, scnt, sbase, sfull, n, sw);
        if (tid == 0) {
            const int64_t tn = t + 2 * (int64_t)gridDim.x;
            if (bulk && tn < ntiles && (tn + 1) * RT <= m) {
                ptx::mbar_expect_tx(&bar[b], tile_bytes);
                ptx::bulk_load(tl, s + tn * tile_floats, tile_bytes, &bar[b]);
                ++issued[b];
            }
        }
    }
    if (abort_flag) {
        // a wait gave up: let this CTA's copies still in flight land before it exits (bounded)
        if (tid == 0) {
            for (int b = 0; b < 2; ++b)
                for (int c = consumed[b]; c < issued[b]; ++c)
                    for (int it = 0; it < (1 << 22) && !ptx::mbar_try_wait(&bar[b], (uint32_t)(c & 1)); ++it) {
                    }
            status[qb::kStError] = 1;
        }
        return;
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
    if (tid == 0 && nties) atomicAdd(&status[tie_slot], nties);
    if (SWEEP) {
        // keys above the windows: lanes -> shared (scnt is free between flushes) -> global
#pragma unroll
        for (int q = 0; q < NT; ++q)
            if (lane + 32 * q < n && above[q]) atomicAdd(&scnt[lane + 32 * q], above[q]);
        __syncthreads();
        for (int j = tid; j < n; j += blockDim.x) {
            if (scnt[j]) atomicAdd(&sw.g_above[j], scnt[j]);
            scnt[j] = 0;
        }
        __syncthreads();
        if (npairs) sweep_flush(pairs, &npairs, scnt, sbase, sfull, n, sw);
    }
}

// ---------------------------------------------------------------------------------------------
// Thread-per-row form of the row pass (used when k + 1 <= the number of column groups).
//
// A warp owns a tile of 32 consecutive rows of s in shared memory (one bulk copy per row into a
// padded row stride, so that 16-byte reads of one column chunk by the 32 threads hit distinct
// banks) and each thread selects for one row:
//   1. group maxima: the row's columns in 32 groups of NT consecutive columns; gm_g = max over
//      the group of v = fp32(s - beta);
//   2. T = the (k+1)-th largest of the 32 group maxima (a sorting network in registers): k + 1
//      distinct elements reach T, so T is a lower bound of the row's (k+1)-th largest v;
//   3. the elements with v >= T' (T' = T, or lower for the window sweep, below) are listed in
//      ascending column order (one byte each), scanning only the groups whose maximum reaches T';
//   4. the listed elements with v >= T are sorted by key (a second network); the k-th and
//      (k+1)-th keys give vk and vk1 (the same values as the ranked selection; only the sign of
//      a zero may differ, and nothing downstream sees it), and the picks are the listed
//      elements with a larger key plus, on a tie at the k-th key, the first ones in column order.
// Window sweep (SWEEP): a key u = fp32(s_ij - alpha_i) can only reach the window [lo_j, hi_j]
// if fp32(s_ij - beta_j) >= T - D, where D = max_j (beta_j - pred(lo_j)) over the columns
// (pred(lo_j): the largest float whose key is below lo_j), because alpha_i >= vk1 >= T:
// fp32(s - a) >= L implies s - a > pred(L), so s - beta_j > alpha_i - D. T' = T - D (rounded
// down) therefore lists every element the sweep can count, and the sweep runs on the list.
// A row whose list overflows kTprCap entries falls back to the warp-per-row code on its tile
// row (ranked selection or rounds, and the full sweep of the row).
namespace qb {
constexpr int kTprWarps = 5;        // warps (32-row tiles) per CTA, one CTA per SM
constexpr int kTprCap = 32;         // listed elements per row
constexpr int kTprPairCap = 3072;   // window pairs buffered per CTA (the rest go straight to the lists)
}  // namespace qb

template <int NT>
__host__ __device__ constexpr int tpr_ld() { return 32 * NT + 4; }  // 32 NT / 4 + 1 is odd: consecutive rows' chunks in distinct banks
template <int NT>
constexpr size_t tpr_dyn_smem() {
    return (size_t)qb::kTprWarps * 32 * tpr_ld<NT>() * sizeof(float) + (size_t)qb::kTprWarps * qb::kTprCap * 32;
}

__device__ __forceinline__ float vmax2(float a, float b) { return fmaxf(a, b); }
__device__ __forceinline__ float vmin2(float a, float b) { return fminf(a, b); }
__device__ __forceinline__ uint32_t vmax2(uint32_t a, uint32_t b) { return max(a, b); }
__device__ __forceinline__ uint32_t vmin2(uint32_t a, uint32_t b) { return min(a, b); }

// Sorts N values held in registers into descending order (bitonic network, N a power of two).
template <typename V, int N>
__device__ __forceinline__ void sort_desc(V (&a)[N]) {
    constexpr int LOG = N == 32 ? 5 : N == 16 ? 4 : N == 8 ? 3 : N == 4 ? 2 : 1;
    static_assert((1 << LOG) == N, "a power of two up to 32");
#pragma unroll
    for (int ls = 1; ls <= LOG; ++ls)
#pragma unroll
        for (int lt = ls - 1; lt >= 0; --lt)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int p = i ^ (1 << lt);
                if (p > i) {
                    const V x = a[i], y = a[p];
                    const V hi = vmax2(x, y), lo = vmin2(x, y);
                    if ((i & (1 << ls)) == 0) { a[i] = hi; a[p] = lo; }
                    else { a[i] = lo; a[p] = hi; }
                }
            }
}

// a[idx & 15] for a 16-entry register array (a tree of selects).
template <typename V>
__device__ __forceinline__ V value_at(const V (&a)[16], int idx) {
    V b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) b[q] = (idx & 8) ? a[q + 8] : a[q];
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = (idx & 4) ? b[q + 4] : b[q];
#pragma unroll
    for (int q = 0; q < 2; ++q) b[q] = (idx & 2) ? b[q + 2] : b[q];
    return (idx & 1) ? b[1] : b[0];
}

// a[idx] for a register array: a tree of selects on the bits of idx (no local-memory copy).
template <typename V>
__device__ __forceinline__ V value_at(const V (&a)[32], int idx) {
    V b[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) b[q] = (idx & 16) ? a[q + 16] : a[q];
#pragma unroll
    for (int q = 0; q < 8; ++q) b[q] = (idx & 8) ? b[q + 8] : b[q];
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = (idx & 4) ? b[q + 4] : b[q];
#pragma unroll
    for (int q = 0; q < 2; ++q) b[q] = (idx & 2) ? b[q + 2] : b[q];
    return (idx & 1) ? b[1] : b[0];
}

// One (column, key) pair inside the window, from the lanes in `mask` (warp-aggregated reservation
// in the CTA buffer; the pairs that do not fit go straight to the column's global list).
__device__ __forceinline__ void tpr_append(bool in, uint32_t j, uint32_t key, uint2* pairs, unsigned* npairs,
                                           const RowSweep& sw) {
    const unsigned full = __activemask();
    const unsigned b = __ballot_sync(full, in);
    if (!b) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(b) - 1;
    unsigned base = 0;
    if (lane == leader) base = atomicAdd(npairs, (unsigned)__popc(b));
    base = __shfl_sync(full, base, leader);
    if (in) {
        const unsigned pos = base + (unsigned)__popc(b & ((1u << lane) - 1u));
        if (pos < (unsigned)qb::kTprPairCap) {
            pairs[pos] = make_uint2(j, key);
        } else {
            const uint32_t g = atomicAdd(&sw.g_ncand[j], 1u);
            if (g < (uint32_t)qb::kGCap) sw.g_cand[(int64_t)j * qb::kGCap + g] = key;
        }
    }
}

template <int NT, bool TRANS, bool SWEEP>
__global__ void __launch_bounds__(qb::kTprWarps * 32, 1)
qb_row_tpr_kernel(const float* __restrict__ s, int64_t m, int n, int k, const float* __restrict__ beta, int rule,
                  float* __restrict__ alpha, int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts,
                  int32_t* __restrict__ status, int tie_slot, int skip_if_done, float* __restrict__ sT, int bulk,
                  RowSweep sw) {
    if (skip_if_done && *(volatile int32_t*)&status[qb::kStQbDone]) return;
    constexpr int W = qb::kTprWarps, LD = tpr_ld<NT>(), NC = 32 * NT, CAP = qb::kTprCap;
    extern __shared__ __align__(128) float tiles[];  // [W][32][LD], then the lists [W][CAP][32] bytes
    unsigned char* lists = reinterpret_cast<unsigned char*>(tiles + (size_t)W * 32 * LD);
    __shared__ __align__(16) float bsh[NC];                        // beta, 0 past n
    __shared__ uint32_t lo_s[SWEEP ? NC : 1], hi_s[SWEEP ? NC : 1];  // the sweep's windows
    __shared__ int cnt[kMaxExperts];
    __shared__ uint32_t above_s[SWEEP ? kMaxExperts : 1];
    __shared__ uint2 pairs[SWEEP ? qb::kTprPairCap : 1];
    __shared__ uint32_t scnt[SWEEP ? kMaxExperts : 1], sbase[SWEEP ? kMaxExperts : 1];
    __shared__ unsigned char sfull[SWEEP ? kMaxExperts : 1];
    __shared__ __align__(8) uint64_t bar[W];
    __shared__ uint32_t f_key[W * 32];
    __shared__ int f_j[W * 32];
    __shared__ float f_v[W * 32];
    __shared__ unsigned npairs;
    __shared__ int nties, abort_flag;
    __shared__ unsigned long long dmax_bits;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned full = 0xffffffffu;
    float* tile = tiles + (size_t)warp * 32 * LD;
    unsigned char* list = lists + (size_t)warp * CAP * 32;

    for (int j = tid; j < NC; j += blockDim.x) {
        bsh[j] = j < n ? beta[j] : 0.f;
        if (SWEEP) {
            uint32_t lo = 0xffffffffu, hi = 0xffffffffu;  // padding columns: no key reaches them
            if (j < n) {
                const uint32_t pk = float_key(beta[j]);
                uint32_t w = sw.win[j] ? sw.win[j] : qb::kWinDefault;
                if (w > qb::kWinSweep) w = qb::kWinSweep;
                lo = pk > w ? pk - w : 0u;
                hi = pk < 0xffffffffu - w ? pk + w : 0xffffffffu;
            }
            lo_s[j] = lo;
            hi_s[j] = hi;
        }
    }
    for (int j = tid; j < kMaxExperts; j += blockDim.x) {
        cnt[j] = 0;
        if (SWEEP) { above_s[j] = 0; scnt[j] = 0; sfull[j] = 0; }
    }
    // tile columns n .. NC - 1 hold -inf for good (the row copies write columns below n only)
    if (n < NC)
        for (int q = tid; q < W * 32 * (NC - n); q += blockDim.x)
            tiles[(q / (NC - n)) * LD + n + q % (NC - n)] = -INFINITY;
    if (tid == 0) { npairs = 0; nties = 0; abort_flag = 0; dmax_bits = 0ull; }
    if (lane == 0) ptx::mbar_init(&bar[warp], 1);
    ptx::fence_barrier_init();
    __syncthreads();
    double dmax = 0.0;
    if (SWEEP) {
        double d = 0.0;
        for (int j = tid; j < n; j += blockDim.x) {
            const uint32_t lo = lo_s[j];
            double dj;
            if (lo <= 0x00800000u) {
                dj = INFINITY;  // the window reaches -inf: every element is listed
            } else {
                uint32_t pk = lo - 1u;
                if (pk == 0x7fffffffu) pk = 0x7ffffffeu;  // below +0 the next float is -denorm_min
                dj = __dsub_ru((double)bsh[j], (double)key_float(pk));
            }
            d = fmax(d, dj);
        }
        atomicMax(&dmax_bits, (unsigned long long)__double_as_longlong(d));  // d >= 0: the bits order like the values
        __syncthreads();
        dmax = __longlong_as_double((long long)dmax_bits);
    }

    const int64_t ntiles = (m + 31) / 32;
    const int64_t nw = (int64_t)gridDim.x * W;
    const int64_t gw = (int64_t)warp * gridDim.x + blockIdx.x;  // tiles b, b + G, ... spread over the CTA's warps
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t used = 0, issued = 0;  // row copies consumed / issued into this warp's tile
    const int ngroups = (n + NT - 1) / NT;
    const uint32_t gvalid = ngroups >= 32 ? 0xffffffffu : ((1u << ngroups) - 1u);

    auto issue = [&](int64_t t) {
        const int64_t i0 = t * 32;
        const int rows = (int)min((int64_t)32, m - i0);
        if (lane == 0) ptx::mbar_expect_tx(&bar[warp], (uint32_t)rows * (uint32_t)n * 4u);
        __syncwarp();
        if (lane < rows) ptx::bulk_load(tile + lane * LD, s + (i0 + lane) * n, (uint32_t)n * 4u, &bar[warp]);
        ++issued;
    };
    if (bulk && gw < ntiles) issue(gw);

    for (int64_t t = gw; t < ntiles; t += nw) {
        const int64_t i0 = t * 32;
        const int rows = (int)min((int64_t)32, m - i0);
        if (bulk) {
            const bool ok = ptx::mbar_wait(&bar[warp], used & 1u, &abort_flag);
            if (!__all_sync(full, ok)) break;
            ++used;
        } else {
            for (int r = 0; r < rows; ++r)
                for (int q = lane; q < n; q += 32) tile[r * LD + q] = s[(i0 + r) * n + q];
            __syncwarp();
        }
        if (__any_sync(full, *(volatile int*)&abort_flag != 0)) break;
        const bool valid = lane < rows;
        const int64_t i = i0 + lane;
        const float* row = tile + lane * LD;

        if (TRANS && valid) {
            for (int c = 0; c < NC / 4; ++c) {
                const float4 sv = *reinterpret_cast<const float4*>(row + 4 * c);
                const float e4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * c + e < n) sT[(int64_t)(4 * c + e) * m + i] = e4[e];
            }
        }

        // 1. group maxima of v = fp32(s - beta)
        float gm[32];
#pragma unroll
        for (int g = 0; g < 32; ++g) gm[g] = -INFINITY;
#pragma unroll
        for (int c = 0; c < NC / 4; ++c) {
            const float4 sv = *reinterpret_cast<const float4*>(row + 4 * c);
            const float4 bv = *reinterpret_cast<const float4*>(bsh + 4 * c);
            const float v0 = __fsub_rn(sv.x, bv.x), v1 = __fsub_rn(sv.y, bv.y), v2 = __fsub_rn(sv.z, bv.z),
                        v3 = __fsub_rn(sv.w, bv.w);
            if constexpr (NT >= 4) {
                gm[4 * c / NT] = fmaxf(gm[4 * c / NT], fmaxf(fmaxf(v0, v1), fmaxf(v2, v3)));
            } else if constexpr (NT == 2) {
                gm[2 * c] = fmaxf(gm[2 * c], fmaxf(v0, v1));
                gm[2 * c + 1] = fmaxf(gm[2 * c + 1], fmaxf(v2, v3));
            } else {
                gm[4 * c] = v0; gm[4 * c + 1] = v1; gm[4 * c + 2] = v2; gm[4 * c + 3] = v3;
            }
        }
        // 2. T and the listing threshold
        float T, Tl;
        uint32_t gbits = 0;
        {
            float srt[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) srt[g] = gm[g];
            sort_desc(srt);
            T = value_at(srt, k);
            Tl = SWEEP ? __double2float_rd(__dsub_rd((double)T, dmax)) : T;
#pragma unroll
            for (int g = 0; g < 32; ++g) gbits |= (gm[g] >= Tl ? 1u : 0u) << g;
            gbits &= gvalid;
        }
        // 3. the listed elements, ascending column
        int nc = 0;
        {
            uint32_t bits = valid ? gbits : 0u;
            while (bits) {
                const int g = __ffs(bits) - 1;
                bits &= bits - 1u;
                const int j0 = g * NT;
                float sv[NT], bv[NT];
                if constexpr (NT >= 4) {
#pragma unroll
                    for (int e = 0; e < NT; e += 4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(row + j0 + e);
                        const float4 b4 = *reinterpret_cast<const float4*>(bsh + j0 + e);
                        sv[e] = a4.x; sv[e + 1] = a4.y; sv[e + 2] = a4.z; sv[e + 3] = a4.w;
                        bv[e] = b4.x; bv[e + 1] = b4.y; bv[e + 2] = b4.z; bv[e + 3] = b4.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < NT; ++e) { sv[e] = row[j0 + e]; bv[e] = bsh[j0 + e]; }
                }
#pragma unroll
                for (int e = 0; e < NT; ++e) {
                    const bool c = (j0 + e < n) && __fsub_rn(sv[e], bv[e]) >= Tl;
                    if (c) {
                        if (nc < CAP) list[nc * 32 + lane] = (unsigned char)(j0 + e);
                        ++nc;
                    }
                }
            }
        }
        const bool ovf = valid && nc > CAP;
        const bool mine = valid && !ovf;
        const int pmax = __reduce_max_sync(full, mine ? nc : 0);
        // 4. keys of the listed elements with v >= T, sorted
        uint32_t kk[CAP];
#pragma unroll
        for (int p = 0; p < CAP; ++p) {
            uint32_t key = 0u;
            if (p < pmax && p < nc && mine) {
                const int j = list[p * 32 + lane];
                const float v = __fsub_rn(row[j], bsh[j]);
                key = v >= T ? float_key_nz(v) : 0u;
            }
            kk[p] = key;
        }
        uint32_t KK = 0, KK1 = 0;
        int A = 0;
        {
            uint32_t srt[CAP];
#pragma unroll
            for (int p = 0; p < CAP; ++p) srt[p] = kk[p];
            sort_desc(srt);
            KK = value_at(srt, k - 1);
            KK1 = value_at(srt, k);
#pragma unroll
            for (int p = 0; p < CAP; ++p) A += srt[p] > KK ? 1 : 0;
        }
        const float vk = key_float(KK), vk1 = key_float(KK1);
        const float a = qb_threshold(vk, vk1, rule);
        if (mine) {
            alpha[i] = a;
            int np = 0, eq = 0;
            const int need_eq = k - A;
#pragma unroll
            for (int p = 0; p < CAP; ++p) {
                if (p < pmax) {
                    const uint32_t key = kk[p];
                    const bool pick = key > KK || (key == KK && eq < need_eq);
                    eq += key == KK ? 1 : 0;
                    if (pick) {
                        const int j = list[p * 32 + lane];
                        topk_idx[i * k + np] = j;
                        atomicAdd(&cnt[j], 1);
                        ++np;
                    }
                }
            }
        }
        {
            const unsigned tb = __ballot_sync(full, mine && vk == vk1);
            if (lane == 0 && tb) atomicAdd(&nties, __popc(tb));
        }
        if (SWEEP) {
            // the sweep on the list: keys above the window counted, keys inside it appended (one
            // reservation in the CTA buffer per warp and tile)
            uint32_t inmask = 0;
            int nin = 0;
            if (mine)
                for (int p = 0; p < nc; ++p) {
                    const int j = list[p * 32 + lane];
                    const uint32_t key = float_key_nz(__fsub_rn(row[j], a));
                    if (key > hi_s[j]) {
                        atomicAdd(&above_s[j], 1u);
                    } else if (key >= lo_s[j]) {
                        inmask |= 1u << p;
                        ++nin;
                    }
                }
            int incl = nin;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(full, incl, o);
                if (lane >= o) incl += y;
            }
            const int total = __shfl_sync(full, incl, 31);
            if (total) {
                unsigned base = 0;
                if (lane == 31) base = atomicAdd(&npairs, (unsigned)total);
                unsigned pos = __shfl_sync(full, base, 31) + (unsigned)(incl - nin);
                while (inmask) {
                    const int p = __ffs(inmask) - 1;
                    inmask &= inmask - 1u;
                    const uint32_t j = list[p * 32 + lane];
                    const uint32_t key = float_key_nz(__fsub_rn(row[j], a));
                    if (pos < (unsigned)qb::kTprPairCap) {
                        pairs[pos] = make_uint2(j, key);
                    } else {
                        const uint32_t g = atomicAdd(&sw.g_ncand[j], 1u);
                        if (g < (uint32_t)qb::kGCap) sw.g_cand[(int64_t)j * qb::kGCap + g] = key;
                    }
                    ++pos;
                }
            }
        }
        // rows whose list overflowed: the warp-per-row code on the tile row
        uint32_t ob = __ballot_sync(full, ovf);
        while (ob) {
            const int r = __ffs(ob) - 1;
            ob &= ob - 1u;
            const int64_t ir = i0 + r;
            const float* rw = tile + r * LD;
            float v[NT];
            uint32_t key[NT];
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const int j = lane + 32 * q;
                const bool ok = j < n;
                v[q] = ok ? __fsub_rn(rw[j], bsh[j]) : 0.f;
                key[q] = ok ? float_key(v[q]) : 0u;
            }
            float wk, wk1;
            if (!(k < 32 && k < n && row_topk_ranked<NT>(key, v, k, ir, f_key + warp * 32, f_j + warp * 32,
                                                          f_v + warp * 32, topk_idx, cnt, wk, wk1))) {
                uint32_t taken;
                row_topk_rounds<NT>(key, v, n, k, taken, wk, wk1);
                int pos = 0;
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const bool bit = (taken >> q) & 1u;
                    const uint32_t mask = __ballot_sync(full, bit);
                    if (bit) {
                        topk_idx[ir * k + pos + __popc(mask & lt)] = lane + 32 * q;
                        atomicAdd(&cnt[lane + 32 * q], 1);
                    }
                    pos += __popc(mask);
                }
            }
            const float wa = qb_threshold(wk, wk1, rule);
            if (lane == 0) {
                alpha[ir] = wa;
                if (wk == wk1) atomicAdd(&nties, 1);
            }
            if (SWEEP) {
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const int j = lane + 32 * q;
                    bool in = false;
                    uint32_t uk = 0;
                    if (j < n) {
                        uk = float_key_nz(__fsub_rn(rw[j], wa));
                        if (uk > hi_s[j]) atomicAdd(&above_s[j], 1u);
                        else in = uk >= lo_s[j];
                    }
                    tpr_append(in, (uint32_t)j, uk, pairs, &npairs, sw);
                }
            }
        }
        __syncwarp();  // every lane is done with the tile
        const int64_t tn = t + nw;
        if (bulk && tn < ntiles) {
            ptx::fence_proxy_async_shared();
            issue(tn);
        }
    }
    __syncthreads();
    if (abort_flag) {
        // a wait gave up: let this warp's copies still in flight land before the CTA exits (bounded)
        if (lane == 0)
            for (uint32_t c = used; c < issued; ++c)
                for (int it = 0; it < (1 << 22) && !ptx::mbar_try_wait(&bar[warp], c & 1u); ++it) {
                }
        if (tid == 0) status[qb::kStError] = 1;
        return;
    }
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
    if (tid == 0 && nties) atomicAdd(&status[tie_slot], nties);
    if (SWEEP) {
        for (int j = tid; j < n; j += blockDim.x)
            if (above_s[j]) atomicAdd(&sw.g_above[j], above_s[j]);
        if (npairs) sweep_flush(pairs, &npairs, scnt, sbase, sfull, n, sw, (unsigned)qb::kTprPairCap);
    }
}

// The same selection without a shared-memory copy of the rows (the passes that write no
// transposed copy): a warp reads its 32 rows from global memory with each lane holding one
// column group of a row (coalesced), forms the group maxima with beta in registers and hands
// them to the row threads through a small shared array; the row threads then read the groups
// that reach T' of their own row again (from L2) and keep the listed elements' scores in their
// shared list. Sixteen warps per SM instead of five: the selection is latency-bound, and the
// rows no longer occupy shared memory.
namespace qb {
constexpr int kTpr2Warps = 16;
}  // namespace qb

constexpr size_t tpr2_dyn_smem() {
    return (size_t)qb::kTpr2Warps * ((32 * 33 + qb::kTprCap * 32) * sizeof(float) + qb::kTprCap * 32);
}

// bsh[g NT .. g NT + NT - 1] (a 16-byte aligned run when NT is a multiple of 4)
template <int NT>
__device__ __forceinline__ void group_betas(const float* bsh, int g, float (&out)[NT]) {
    if constexpr (NT % 4 == 0) {
#pragma unroll
        for (int e = 0; e < NT; e += 4) {
            const float4 q = *reinterpret_cast<const float4*>(bsh + g * NT + e);
            out[e] = q.x; out[e + 1] = q.y; out[e + 2] = q.z; out[e + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < NT; ++e) out[e] = bsh[g * NT + e];
    }
}

// NT consecutive scores from p (the first `valid` of them exist; the rest read as -inf)
template <int NT>
__device__ __forceinline__ void load_group(const float* p, bool vec, int valid, float (&out)[NT]) {
    if (vec && valid >= NT) {
        if constexpr (NT >= 4) {
#pragma unroll
            for (int e = 0; e < NT; e += 4) {
                const float4 q = __ldg(reinterpret_cast<const float4*>(p + e));
                out[e] = q.x; out[e + 1] = q.y; out[e + 2] = q.z; out[e + 3] = q.w;
            }
            return;
        } else if constexpr (NT == 2) {
            const float2 q = __ldg(reinterpret_cast<const float2*>(p));
            out[0] = q.x; out[1] = q.y;
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < NT; ++e) out[e] = e < valid ? __ldg(p + e) : -INFINITY;
}

// SIGN (SignSGD step): also count_j = #{i : fp32(s_ij - alpha_i) > beta_j}. Such an element has
// s_ij - beta_j > alpha_i >= T (fp32(x) > beta_j implies x > beta_j), so v_ij >= T: it is listed.
template <int NT, bool SWEEP, bool SIGN>
__global__ void __launch_bounds__(qb::kTpr2Warps * 32, 1)
qb_row_tpr2_kernel(const float* __restrict__ s, int64_t m, int n, int k, const float* __restrict__ beta, int rule,
                   float* __restrict__ alpha, int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts,
                   int32_t* __restrict__ status, int tie_slot, int skip_if_done, RowSweep sw,
                   int32_t* __restrict__ sign_counts) {
    pdl_wait();  // beta, the status words and the counters come from the previous launches
    if (skip_if_done && *(volatile int32_t*)&status[qb::kStQbDone]) return;
    constexpr int W = qb::kTpr2Warps, NC = 32 * NT, CAP = qb::kTprCap, GS = 33;
    extern __shared__ __align__(16) float dsm[];  // per warp: [32][33] group maxima, [CAP][32] listed scores; then [W][CAP][32] columns
    __shared__ __align__(16) float bsh[NC];
    __shared__ uint32_t lo_s[SWEEP ? NC : 1], hi_s[SWEEP ? NC : 1];
    __shared__ int cnt[kMaxExperts];
    __shared__ uint32_t above_s[(SWEEP || SIGN) ? kMaxExperts : 1];  // keys above the window, or the sign counts
    __shared__ uint2 pairs[SWEEP ? qb::kTprPairCap : 1];
    __shared__ uint32_t scnt[SWEEP ? kMaxExperts : 1], sbase[SWEEP ? kMaxExperts : 1];
    __shared__ unsigned char sfull[SWEEP ? kMaxExperts : 1];
    __shared__ uint32_t f_key[W * 32];
    __shared__ int f_j[W * 32];
    __shared__ float f_v[W * 32];
    __shared__ unsigned npairs;
    __shared__ int nties;
    __shared__ unsigned long long dmax_bits;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned full = 0xffffffffu;
    float* gmx = dsm + (size_t)warp * (32 * GS + CAP * 32);
    float* ls = gmx + 32 * GS;
    unsigned char* lj = reinterpret_cast<unsigned char*>(dsm + (size_t)W * (32 * GS + CAP * 32)) + (size_t)warp * CAP * 32;

    for (int j = tid; j < NC; j += blockDim.x) {
        bsh[j] = j < n ? beta[j] : 0.f;
        if (SWEEP) {
            uint32_t lo = 0xffffffffu, hi = 0xffffffffu;
            if (j < n) {
                const uint32_t pk = float_key(beta[j]);
                uint32_t w = sw.win[j] ? sw.win[j] : qb::kWinDefault;
                if (w > qb::kWinSweep) w = qb::kWinSweep;
                lo = pk > w ? pk - w : 0u;
                hi = pk < 0xffffffffu - w ? pk + w : 0xffffffffu;
            }
            lo_s[j] = lo;
            hi_s[j] = hi;
        }
    }
    for (int j = tid; j < kMaxExperts; j += blockDim.x) {
        cnt[j] = 0;
        if (SWEEP || SIGN) above_s[j] = 0;
        if (SWEEP) { scnt[j] = 0; sfull[j] = 0; }
    }
    if (tid == 0) { npairs = 0; nties = 0; dmax_bits = 0ull; }
    __syncthreads();
    double dmax = 0.0;
    if (SWEEP) {
        double d = 0.0;
        for (int j = tid; j < n; j += blockDim.x) {
            const uint32_t lo = lo_s[j];
            double dj;
            if (lo <= 0x00800000u) {
                dj = INFINITY;
            } else {
                uint32_t pk = lo - 1u;
                if (pk == 0x7fffffffu) pk = 0x7ffffffeu;
                dj = __dsub_ru((double)bsh[j], (double)key_float(pk));
            }
            d = fmax(d, dj);
        }
        atomicMax(&dmax_bits, (unsigned long long)__double_as_longlong(d));
        __syncthreads();
        dmax = __longlong_as_double((long long)dmax_bits);
    }

    const int64_t ntiles = (m + 31) / 32;
    const int64_t nw = (int64_t)gridDim.x * W;
    const int64_t gw = (int64_t)warp * gridDim.x + blockIdx.x;
    const uint32_t lt = (1u << lane) - 1u;
    const int ngroups = (n + NT - 1) / NT;
    const uint32_t gvalid = ngroups >= 32 ? 0xffffffffu : ((1u << ngroups) - 1u);
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15) == 0 && n % 4 == 0;
    // this lane's column group in the coalesced pass, and its beta
    const int gj0 = lane * NT;
    float bl[NT];
#pragma unroll
    for (int e = 0; e < NT; ++e) bl[e] = bsh[gj0 + e];

    for (int64_t t = gw; t < ntiles; t += nw) {
        const int64_t i0 = t * 32;
        const int rows = (int)min((int64_t)32, m - i0);
        // 1. group maxima, 8 rows per batch (lane = column group)
#pragma unroll 1
        for (int r0 = 0; r0 < 32; r0 += 8) {
            float sv[8][NT];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                if (r0 + rr < rows && gj0 < n) {
                    load_group<NT>(s + (i0 + r0 + rr) * n + gj0, vec, n - gj0, sv[rr]);
                } else {
#pragma unroll
                    for (int e = 0; e < NT; ++e) sv[rr][e] = -INFINITY;
                }
            }
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                float g = -INFINITY;
#pragma unroll
                for (int e = 0; e < NT; ++e) g = fmaxf(g, __fsub_rn(sv[rr][e], bl[e]));
                gmx[(r0 + rr) * GS + lane] = g;
            }
        }
        __syncwarp();
        const bool valid = lane < rows;
        const int64_t i = i0 + lane;
        // 2. T and the listing threshold
        float T, Tl;
        uint32_t gbits = 0;
        {
            float srt[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) srt[g] = gmx[lane * GS + g];
            sort_desc(srt);
            T = value_at(srt, k);
            Tl = SWEEP ? __double2float_rd(__dsub_rd((double)T, dmax)) : T;
#pragma unroll
            for (int g = 0; g < 32; ++g) gbits |= (gmx[lane * GS + g] >= Tl ? 1u : 0u) << g;
            gbits &= gvalid;
        }
        // 3. the listed elements of the groups reaching T', two groups' loads in flight
        int nc = 0;
        {
            const float* rowp = s + i * n;
            uint32_t bits = valid ? gbits : 0u;
            while (bits) {
                const int g1 = __ffs(bits) - 1;
                bits &= bits - 1u;
                const int g2 = bits ? __ffs(bits) - 1 : -1;
                if (bits) bits &= bits - 1u;
                float s1[NT], s2[NT];
                load_group<NT>(rowp + g1 * NT, vec, n - g1 * NT, s1);
                if (g2 >= 0) load_group<NT>(rowp + g2 * NT, vec, n - g2 * NT, s2);
                // the group's betas in one piece (bsh holds 32 NT entries, zero past n)
                float b1v[NT], b2v[NT];
                group_betas<NT>(bsh, g1, b1v);
                if (g2 >= 0) group_betas<NT>(bsh, g2, b2v);
#pragma unroll
                for (int e = 0; e < NT; ++e) {
                    const int j = g1 * NT + e;
                    if (j < n && __fsub_rn(s1[e], b1v[e]) >= Tl) {
                        if (nc < CAP) { ls[nc * 32 + lane] = s1[e]; lj[nc * 32 + lane] = (unsigned char)j; }
                        ++nc;
                    }
                }
                if (g2 >= 0) {
#pragma unroll
                    for (int e = 0; e < NT; ++e) {
                        const int j = g2 * NT + e;
                        if (j < n && __fsub_rn(s2[e], b2v[e]) >= Tl) {
                            if (nc < CAP) { ls[nc * 32 + lane] = s2[e]; lj[nc * 32 + lane] = (unsigned char)j; }
                            ++nc;
                        }
                    }
                }
            }
        }
        const bool ovf = valid && nc > CAP;
        const bool mine = valid && !ovf;
        const int pmax = __reduce_max_sync(full, mine ? nc : 0);
        // 4. the k-th and (k+1)-th keys of the listed elements with v >= T
        uint32_t KK = 0, KK1 = 0;
        int A = 0;
        {
            uint32_t kk[CAP];
            // the keys of list slots p < pmax (slots 16 .. CAP - 1 only when some row of the warp has them)
            auto slot_key = [&](int p) {
                uint32_t key = 0u;
                if (p < nc && mine) {
                    const int j = lj[p * 32 + lane];
                    const float v = __fsub_rn(ls[p * 32 + lane], bsh[j]);
                    key = v >= T ? float_key_nz(v) : 0u;
                }
                return key;
            };
#pragma unroll
            for (int p = 0; p < 16; ++p) kk[p] = p < pmax ? slot_key(p) : 0u;
            if (pmax > 16) {
#pragma unroll
                for (int p = 16; p < CAP; ++p) kk[p] = p < pmax ? slot_key(p) : 0u;
            } else {
#pragma unroll
                for (int p = 16; p < CAP; ++p) kk[p] = 0u;
            }
            if (pmax <= 16) {
                // at most 16 listed elements in every row of the warp (then k < 16): a 16-wide network
                uint32_t k16[16];
#pragma unroll
                for (int p = 0; p < 16; ++p) k16[p] = kk[p];
                sort_desc(k16);
                KK = value_at(k16, k - 1);
                KK1 = value_at(k16, k);
#pragma unroll
                for (int p = 0; p < 16; ++p) A += k16[p] > KK ? 1 : 0;
            } else {
                sort_desc(kk);
                KK = value_at(kk, k - 1);
                KK1 = value_at(kk, k);
#pragma unroll
                for (int p = 0; p < CAP; ++p) A += kk[p] > KK ? 1 : 0;
            }
        }
        const float vk = key_float(KK), vk1 = key_float(KK1);
        const float a = qb_threshold(vk, vk1, rule);
        // one pass over the list: the picks, the sign counts, and the sweep's window test of
        // u = fp32(s - alpha_i) (the list positions inside the window in inmask)
        uint32_t inmask = 0;
        int nin = 0;
        if (mine) {
            alpha[i] = a;
            int np = 0, eq = 0;
            const int need_eq = k - A;
            for (int p = 0; p < nc; ++p) {
                const int j = lj[p * 32 + lane];
                const float sv = ls[p * 32 + lane], bj = bsh[j];
                const float v = __fsub_rn(sv, bj);
                const uint32_t key = v >= T ? float_key_nz(v) : 0u;
                const bool pick = key > KK || (key == KK && eq < need_eq);
                eq += key == KK ? 1 : 0;
                if (pick) {
                    topk_idx[i * k + np] = j;
                    atomicAdd(&cnt[j], 1);
                    ++np;
                }
                if (SIGN && key != 0u && __fsub_rn(sv, a) > bj) atomicAdd(&above_s[j], 1u);
                if (SWEEP) {
                    const uint32_t ua = float_key_nz(__fsub_rn(sv, a));
                    if (ua > hi_s[j]) {
                        atomicAdd(&above_s[j], 1u);
                    } else if (ua >= lo_s[j]) {
                        inmask |= 1u << p;
                        ++nin;
                    }
                }
            }
        }
        {
            const unsigned tb = __ballot_sync(full, mine && vk == vk1);
            if (lane == 0 && tb) atomicAdd(&nties, __popc(tb));
        }
        if (SWEEP) {
            int incl = nin;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(full, incl, o);
                if (lane >= o) incl += y;
            }
            const int total = __shfl_sync(full, incl, 31);
            if (total) {
                unsigned base = 0;
                if (lane == 31) base = atomicAdd(&npairs, (unsigned)total);
                unsigned pos = __shfl_sync(full, base, 31) + (unsigned)(incl - nin);
                while (inmask) {
                    const int p = __ffs(inmask) - 1;
                    inmask &= inmask - 1u;
                    const uint32_t j = lj[p * 32 + lane];
                    const uint32_t key = float_key_nz(__fsub_rn(ls[p * 32 + lane], a));
                    if (pos < (unsigned)qb::kTprPairCap) {
                        pairs[pos] = make_uint2(j, key);
                    } else {
                        const uint32_t g = atomicAdd(&sw.g_ncand[j], 1u);
                        if (g < (uint32_t)qb::kGCap) sw.g_cand[(int64_t)j * qb::kGCap + g] = key;
                    }
                    ++pos;
                }
            }
        }
        // rows whose list overflowed: the warp-per-row code, the row read again from global memory
        uint32_t ob = __ballot_sync(full, ovf);
        while (ob) {
            const int r = __ffs(ob) - 1;
            ob &= ob - 1u;
            const int64_t ir = i0 + r;
            const float* rw = s + ir * n;
            float v[NT];
            uint32_t key[NT];
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const int j = lane + 32 * q;
                const bool ok = j < n;
                v[q] = ok ? __fsub_rn(__ldg(rw + j), bsh[j]) : 0.f;
                key[q] = ok ? float_key(v[q]) : 0u;
            }
            float wk, wk1;
            if (!(k < 32 && k < n && row_topk_ranked<NT>(key, v, k, ir, f_key + warp * 32, f_j + warp * 32,
                                                          f_v + warp * 32, topk_idx, cnt, wk, wk1))) {
                uint32_t taken;
                row_topk_rounds<NT>(key, v, n, k, taken, wk, wk1);
                int pos = 0;
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const bool bit = (taken >> q) & 1u;
                    const uint32_t mask = __ballot_sync(full, bit);
                    if (bit) {
                        topk_idx[ir * k + pos + __popc(mask & lt)] = lane + 32 * q;
                        atomicAdd(&cnt[lane + 32 * q], 1);
                    }
                    pos += __popc(mask);
                }
            }
            const float wa = qb_threshold(wk, wk1, rule);
            if (lane == 0) {
                alpha[ir] = wa;
                if (wk == wk1) atomicAdd(&nties, 1);
            }
            if (SIGN) {
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const int j = lane + 32 * q;
                    if (j < n && __fsub_rn(__ldg(rw + j), wa) > bsh[j]) atomicAdd(&above_s[j], 1u);
                }
            }
            if (SWEEP) {
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const int j = lane + 32 * q;
                    bool in = false;
                    uint32_t uk = 0;
                    if (j < n) {
                        uk = float_key_nz(__fsub_rn(__ldg(rw + j), wa));
                        if (uk > hi_s[j]) atomicAdd(&above_s[j], 1u);
                        else in = uk >= lo_s[j];
                    }
                    tpr_append(in, (uint32_t)j, uk, pairs, &npairs, sw);
                }
            }
        }
        __syncwarp();  // the group maxima and lists are rewritten by the next tile
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
    if (tid == 0 && nties) atomicAdd(&status[tie_slot], nties);
    if (SIGN)
        for (int j = tid; j < n; j += blockDim.x)
            if (above_s[j]) atomicAdd(&sign_counts[j], (int)above_s[j]);
    if (SWEEP) {
        for (int j = tid; j < n; j += blockDim.x)
            if (above_s[j]) atomicAdd(&sw.g_above[j], above_s[j]);
        if (npairs) sweep_flush(pairs, &npairs, scnt, sbase, sfull, n, sw, (unsigned)qb::kTprPairCap);
    }
    pdl_trigger();
}

// Block-wide bin selection: scanning bins from the top, the bin where the cumulative count
// reaches `want` (1-based rank). Every thread gets the bin, the rank left inside it and its count.
__device__ __forceinline__ void block_select_bin(const unsigned* hist, int nbins, int64_t want, unsigned* scan,
                                                 int* sel, int64_t* want_left, unsigned* bin_count) {
    const int tid = threadIdx.x, T = blockDim.x;
    const int per = (nbins + T - 1) / T;
    unsigned s = 0;
    for (int u = 0; u < per; ++u) {
        const int b = nbins - 1 - (tid * per + u);
        if (b >= 0) s += hist[b];
    }
    scan[tid] = s;
    __syncthreads();
    for (int o = 1; o < T; o <<= 1) {
        const unsigned add = tid >= o ? scan[tid - o] : 0u;
        __syncthreads();
        scan[tid] += add;
        __syncthreads();
    }
    const int64_t incl = scan[tid], excl = incl - s;
    __shared__ int r_sel;
    __shared__ int64_t r_want;
    __shared__ unsigned r_cnt;
    if (excl < want && want <= incl) {
        int64_t cum = excl;
        for (int u = 0; u < per; ++u) {
            const int b = nbins - 1 - (tid * per + u);
            if (b < 0) break;
            const unsigned h = hist[b];
            if (cum + h >= want) { r_sel = b; r_want = want - cum; r_cnt = h; break; }
            cum += h;
        }
    }
    __syncthreads();
    *sel = r_sel;
    *want_left = r_want;
    *bin_count = r_cnt;
    __syncthreads();
}

// Add 1 to hist[d] for every active lane (shared-memory atomics; lanes on the same bin are
// serialised by the hardware, which costs less than grouping them first).
__device__ __forceinline__ void warp_hist_add(unsigned* hist, bool active, uint32_t d) {
    if (active) atomicAdd(&hist[d], 1u);
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, unsigned* red) {
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t r = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, red[w]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ unsigned block_sum_u32(unsigned v, unsigned* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    unsigned r = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += red[w];
    __syncthreads();
    return r;
}


// Visit every key float_key(fp32(col[i * stride] - alpha[i])) of a column, warp-uniformly (f gets
// ok = false for padding lanes). A contiguous column (stride 1, m a multiple of 4: every column
// of sT starts on a 16-byte boundary) is read with 16-byte loads, kColUnroll of each operand in
// flight per thread; a strided one (a column of row-major s) with 8 scalar loads in flight.
template <typename F>
__device__ __forceinline__ void for_each_col_key(const float* __restrict__ col, int64_t stride,
                                                 const float* __restrict__ alpha, int64_t m, F&& f) {
    const int tid = threadIdx.x, T = blockDim.x;
    if (stride == 1 && (m & 3) == 0) {
        // kColUnroll float4 pairs (column, alpha) per thread in flight before any is used
        constexpr int U = qb::kColUnroll;
        const float4* c4 = reinterpret_cast<const float4*>(col);
        const float4* a4 = reinterpret_cast<const float4*>(alpha);
        const int64_t m4 = m >> 2;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t base = 0; base < m4; base += U * T) {
            float4 c[U], a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t v = base + tid + (int64_t)u * T;
                c[u] = v < m4 ? c4[v] : z;
                a[u] = v < m4 ? a4[v] : z;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const bool ok = base + tid + (int64_t)u * T < m4;
                f(ok, float_key(__fsub_rn(c[u].x, a[u].x)));
                f(ok, float_key(__fsub_rn(c[u].y, a[u].y)));
                f(ok, float_key(__fsub_rn(c[u].z, a[u].z)));
                f(ok, float_key(__fsub_rn(c[u].w, a[u].w)));
            }
        }
    } else {
        constexpr int U = 8;
        for (int64_t base = 0; base < m; base += U * T) {
            float c[U], a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t i = base + tid + (int64_t)u * T;
                c[u] = i < m ? col[i * stride] : 0.f;
                a[u] = i < m ? alpha[i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const bool ok = base + tid + (int64_t)u * T < m;
                f(ok, ok ? float_key(__fsub_rn(c[u], a[u])) : 0u);
            }
        }
    }
}

// Append `key` to the shared list for every lane with `in` (warp-uniform call; one shared
// atomic per warp). Positions past kCandCap are counted but not stored.
__device__ __forceinline__ void warp_append(unsigned* list, unsigned* count, bool in, uint32_t key) {
    const uint32_t bal = __ballot_sync(0xffffffffu, in);
    if (!bal) return;
    const int lane = threadIdx.x & 31;
    unsigned wbase = 0;
    if (lane == 0) wbase = atomicAdd(count, (unsigned)__popc(bal));
    wbase = __shfl_sync(0xffffffffu, wbase, 0);
    const unsigned pos = wbase + __popc(bal & ((1u << lane) - 1u));
    if (in && pos < (unsigned)qb::kCandCap) list[pos] = key;
}

// The want-th largest key (1-based, want <= ncand) of the shared list: three digit passes
// (bits 31..20, 19..8, 7..0). Also gives its multiplicity and the number of list keys above it.
__device__ void select_in_list(const unsigned* list, unsigned ncand, int64_t want, unsigned* hist, unsigned* scan,
                               uint32_t* key_out, unsigned* mult_out, int64_t* greater_out) {
    const int tid = threadIdx.x, T = blockDim.x;
    int s1, s2, s3;
    int64_t w1, w2, w3;
    unsigned c1, c2, c3;
    for (int b = tid; b < 4096; b += T) hist[b] = 0;
    __syncthreads();
    for (unsigned base = 0; base < ncand; base += T) {
        const unsigned c = base + tid;
        const bool ok = c < ncand;
        warp_hist_add(hist, ok, (ok ? list[c] : 0u) >> 20);
    }
    __syncthreads();
    block_select_bin(hist, 4096, want, scan, &s1, &w1, &c1);
    for (int b = tid; b < 4096; b += T) hist[b] = 0;
    __syncthreads();
    for (unsigned base = 0; base < ncand; base += T) {
        const unsigned c = base + tid;
        const uint32_t key = c < ncand ? list[c] : 0u;
        warp_hist_add(hist, c < ncand && (key >> 20) == (uint32_t)s1, (key >> 8) & 0xfffu);
    }
    __syncthreads();
    block_select_bin(hist, 4096, w1, scan, &s2, &w2, &c2);
    const uint32_t pre = ((uint32_t)s1 << 20) | ((uint32_t)s2 << 8);
    for (int b = tid; b < 256; b += T) hist[b] = 0;
    __syncthreads();
    for (unsigned base = 0; base < ncand; base += T) {
        const unsigned c = base + tid;
        const uint32_t key = c < ncand ? list[c] : 0u;
        warp_hist_add(hist, c < ncand && (key & 0xffffff00u) == pre, key & 0xffu);
    }
    __syncthreads();
    block_select_bin(hist, 256, w2, scan, &s3, &w3, &c3);
    *key_out = pre | (uint32_t)s3;
    *mult_out = c3;
    *greater_out = want - w3;
}

// Largest list key strictly below `bound` (0 if none), block-wide.
__device__ __forceinline__ uint32_t list_max_below(const unsigned* list, unsigned ncand, uint32_t bound,
                                                   unsigned* scan) {
    uint32_t best = 0;
    for (unsigned c = threadIdx.x; c < ncand; c += blockDim.x) {
        const uint32_t key = list[c];
        if (key < bound && key > best) best = key;
    }
    return block_max_u32(best, scan);
}

// The want-th and (want+1)-th largest keys (1-based, want + 1 <= ncand) of a short shared list,
// by ranks: a key holds rank r when fewer than r keys are above it and at least r are at or
// above it. One candidate per thread (ncand <= blockDim.x), four list keys per shared load.
__device__ __forceinline__ void rank_select2(const unsigned* list, unsigned ncand, int64_t want, uint32_t* out) {
    const unsigned c = threadIdx.x;
    if (c < ncand) {
        const uint32_t kc = list[c];
        unsigned g = 0, e = 0;
        const unsigned n4 = ncand & ~3u;
        for (unsigned x = 0; x < n4; x += 4) {
            const uint4 q = *reinterpret_cast<const uint4*>(list + x);
            g += (q.x > kc) + (q.y > kc) + (q.z > kc) + (q.w > kc);
            e += (q.x == kc) + (q.y == kc) + (q.z == kc) + (q.w == kc);
        }
        for (unsigned x = n4; x < ncand; ++x) {
            g += list[x] > kc;
            e += list[x] == kc;
        }
        if ((int64_t)g < want && want <= (int64_t)(g + e)) out[0] = kc;
        if ((int64_t)g < want + 1 && want + 1 <= (int64_t)(g + e)) out[1] = kc;
    }
    __syncthreads();
}

// The C-th and (C+1)-th largest keys of fp32(col[i * stride] - alpha[i]) over i < m, by the full
// radix path: a 12-bit digit histogram sweep, a sweep keeping the selected bin's keys (the largest
// key below the bin is tracked), then the low digits over the kept keys (streamed from global
// memory if the bin overflows the shared list). Called by every thread of the block; the keys
// come back in every thread.
__device__ void column_select_full(const float* __restrict__ col, int64_t stride, const float* __restrict__ alpha,
                                   int64_t m, int64_t C, unsigned* hist, unsigned* scan, unsigned* cand,
                                   unsigned* s_ncand_p, uint32_t* akey_out, uint32_t* bkey_out) {
    const int tid = threadIdx.x, T = blockDim.x;
    unsigned& s_ncand = *s_ncand_p;
    unsigned ncand;
    uint32_t akey, bkey;
    // ---- full radix path
    uint32_t below = 0;
    for (int b = tid; b < 4096; b += T) hist[b] = 0;
    __syncthreads();
    for_each_col_key(col, stride, alpha, m, [&](bool ok, uint32_t key) { warp_hist_add(hist, ok, key >> 20); });
    __syncthreads();
    int sel1;
    int64_t want1;
    unsigned cnt1;
    block_select_bin(hist, 4096, C, scan, &sel1, &want1, &cnt1);
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    for_each_col_key(col, stride, alpha, m, [&](bool ok, uint32_t key) {
        const uint32_t d = key >> 20;
        if (ok && d < (uint32_t)sel1 && key > below) below = key;
        warp_append(cand, &s_ncand, ok && d == (uint32_t)sel1, key);
    });
    below = block_max_u32(below, scan);
    ncand = s_ncand;
    if (ncand <= (unsigned)qb::kCandCap) {
        unsigned mult;
        int64_t greater;
        select_in_list(cand, ncand, want1, hist, scan, &akey, &mult, &greater);
        greater += C - want1;
        if (greater + (int64_t)mult >= C + 1) {
            bkey = akey;
        } else {
            const uint32_t best = list_max_below(cand, ncand, akey, scan);
            bkey = best ? best : below;
        }
    } else {
        // the bin overflows the list: its low digits stream from global memory
        int sel2, sel3;
        int64_t want2, want3;
        unsigned cnt2, cnt3;
        for (int b = tid; b < 4096; b += T) hist[b] = 0;
        __syncthreads();
        for_each_col_key(col, stride, alpha, m, [&](bool ok, uint32_t key) {
            warp_hist_add(hist, ok && (key >> 20) == (uint32_t)sel1, (key >> 8) & 0xfffu);
        });
        __syncthreads();
        block_select_bin(hist, 4096, want1, scan, &sel2, &want2, &cnt2);
        const uint32_t pre2 = ((uint32_t)sel1 << 20) | ((uint32_t)sel2 << 8);
        for (int b = tid; b < 256; b += T) hist[b] = 0;
        __syncthreads();
        for_each_col_key(col, stride, alpha, m, [&](bool ok, uint32_t key) {
            warp_hist_add(hist, ok && (key & 0xffffff00u) == pre2, key & 0xffu);
        });
        __syncthreads();
        block_select_bin(hist, 256, want2, scan, &sel3, &want3, &cnt3);
        akey = pre2 | (uint32_t)sel3;
        const int64_t greater = C - want3;
        if (greater + (int64_t)cnt3 >= C + 1) {
            bkey = akey;
        } else {
            uint32_t best = 0;
            for_each_col_key(col, stride, alpha, m, [&](bool ok, uint32_t key) {
                if (ok && (key >> 20) == (uint32_t)sel1 && key < akey && key > best) best = key;
            });
            best = block_max_u32(best, scan);
            bkey = best ? best : below;
        }
    }
    *akey_out = akey;
    *bkey_out = bkey;
}

// Column pass: beta_j = threshold between the C-th and (C+1)-th largest key of column j
// of u = fp32(s - alpha). When both fell inside the window of the row pass's sweep (the usual case once the
// iteration settles) they come from the column's candidate list, copied into shared memory:
// by ranks when the list is short, else by radix digits. Otherwise the full radix path over the
// column: a 12-bit digit histogram sweep, a sweep keeping the selected bin's keys (the largest
// key below the bin is tracked), then the low digits over the kept keys (streamed from global
// memory if the bin overflows the list). The column is read from sT (contiguous) when it
// exists, else from s (stride n). Every path returns the same two keys. Part 1's counters are
// cleared for the next pass. check: nothing to do once kStQbDone is set; otherwise CTA 0
// prepares the next row pass. info (one STEP): CTA 0 also writes the call's info words from the
// row pass's counts.
__global__ void __launch_bounds__(qb::kColThreads)
qb_col_kernel(const float* __restrict__ s, const float* __restrict__ sT, int64_t m, int n, int64_t C,
              const float* __restrict__ alpha, int rule, float* __restrict__ beta, int32_t* __restrict__ counts_next,
              int32_t* __restrict__ status, int iter, int check, uint32_t* __restrict__ win,
              uint32_t* __restrict__ g_above, uint32_t* __restrict__ g_ncand, const uint32_t* __restrict__ g_cand,
              const int32_t* __restrict__ info_counts, int tie_slot, int32_t* __restrict__ info) {
    pdl_wait();  // the row pass's counts, alpha and window lists
    if (info && blockIdx.x == 0 && threadIdx.x < 32) {
        int64_t ex = 0;
        for (int e = threadIdx.x; e < n; e += 32) ex += info_counts[e] > C ? info_counts[e] - C : 0;
        for (int o = 16; o > 0; o >>= 1) ex += __shfl_xor_sync(0xffffffffu, ex, o);
        if (threadIdx.x == 0) {
            info[0] = 1;
            info[1] = status[qb::kStAugments];
            info[2] = (int32_t)ex;
            info[3] = status[tie_slot];
        }
    }
    if (check) {
        if (*(volatile int32_t*)&status[qb::kStQbDone]) return;
        // stop once the row pass just made left every count at C
        int unbalanced = 0;
        for (int e = threadIdx.x; e < n; e += blockDim.x) unbalanced |= info_counts[e] != C;
        if (!__syncthreads_or(unbalanced)) {
            if (blockIdx.x == 0 && threadIdx.x == 0) status[qb::kStQbDone] = 1;
            return;
        }
        if (blockIdx.x == 0) {
            for (int e = threadIdx.x; e < n; e += blockDim.x) counts_next[e] = 0;
            if (threadIdx.x == 0) {
                status[qb::kStIters] = iter + 1;
                status[(iter + 1) % 2 ? qb::kStTies1 : qb::kStTies0] = 0;
            }
        }
    }
    extern __shared__ unsigned col_smem[];
    unsigned* hist = col_smem;                 // 4096
    unsigned* scan = hist + 4096;              // blockDim
    unsigned* cand = scan + qb::kColThreads;   // kCandCap
    __shared__ unsigned s_ncand;
    __shared__ uint32_t s_sel[2];
    const int tid = threadIdx.x, T = blockDim.x;
    const int j = blockIdx.x;
    const float* col = sT ? sT + (int64_t)j * m : s + j;
    const int64_t stride = sT ? 1 : n;

    const uint32_t pk = float_key(beta[j]);
    const unsigned above = __ldcg(&g_above[j]);
    unsigned ncand = __ldcg(&g_ncand[j]);
    // both order statistics inside the window
    const bool hit = ncand <= (unsigned)qb::kGCap && (int64_t)above < C && (int64_t)above + ncand >= C + 1;
    if (hit)
        for (unsigned c = tid; c < ncand; c += T) cand[c] = __ldcg(&g_cand[(int64_t)j * qb::kGCap + c]);
    __syncthreads();
    if (tid == 0) { g_above[j] = 0; g_ncand[j] = 0; }

    uint32_t akey, bkey;
    if (hit && ncand <= (unsigned)T) {
        rank_select2(cand, ncand, C - (int64_t)above, s_sel);
        akey = s_sel[0];
        bkey = s_sel[1];
    } else if (hit) {
        unsigned mult;
        int64_t greater;
        select_in_list(cand, ncand, C - (int64_t)above, hist, scan, &akey, &mult, &greater);
        greater += above;
        bkey = greater + (int64_t)mult >= C + 1 ? akey : list_max_below(cand, ncand, akey, scan);
    } else {
        column_select_full(col, stride, alpha, m, C, hist, scan, cand, &s_ncand, &akey, &bkey);
    }
    if (tid == 0) {
        const float bnew = qb_threshold(key_float(akey), key_float(bkey), rule);
        beta[j] = bnew;
        // next window: centred on the new beta, twice as wide as this move, plus the gap it splits
        const uint32_t nk = float_key(bnew);
        const uint64_t dist = nk > pk ? (uint64_t)(nk - pk) : (uint64_t)(pk - nk);
        uint64_t wn = 2 * dist + (uint64_t)(akey - bkey) + qb::kWinMin;
        if (wn > qb::kWinMax) wn = qb::kWinMax;
        win[j] = (uint32_t)wn;
    }
    pdl_trigger();
}

// The practical QB step on mini-batches ("MoE travelogue 6", Mind the pitfall, closing
// paragraph): beta computed by the formula on each mini-batch of L tokens, then averaged. One CTA
// per (expert j, mini-batch b): the C_b-th and (C_b + 1)-th largest of fp32(s_ij - alpha_i) over
// the mini-batch's tokens, read from sT (contiguous). A mini-batch of at most kCandCap tokens has
// all its keys copied into shared memory and selected there (ranks for at most one key per
// thread, else radix digits); a longer one takes the full radix path over global memory.
__global__ void __launch_bounds__(qb::kColThreads)
qb_col_slice_kernel(const float* __restrict__ sT, int64_t m, int n, int64_t L, int64_t Cb,
                    const float* __restrict__ alpha, int rule, float* __restrict__ beta_parts) {
    extern __shared__ unsigned col_smem[];
    unsigned* hist = col_smem;                 // 4096
    unsigned* scan = hist + 4096;              // blockDim
    unsigned* cand = scan + qb::kColThreads;   // kCandCap
    __shared__ unsigned s_ncand;
    __shared__ uint32_t s_sel[2];
    const int tid = threadIdx.x;
    const int j = blockIdx.x;
    const int64_t b = blockIdx.y;
    const float* col = sT + (int64_t)j * m + b * L;
    const float* a = alpha + b * L;
    uint32_t akey, bkey;
    if (L <= (int64_t)qb::kCandCap) {
        if (tid == 0) s_ncand = 0;
        __syncthreads();
        for_each_col_key(col, 1, a, L, [&](bool ok, uint32_t key) { warp_append(cand, &s_ncand, ok, key); });
        __syncthreads();
        const unsigned ncand = (unsigned)L;
        if (ncand <= (unsigned)blockDim.x) {
            rank_select2(cand, ncand, Cb, s_sel);
            akey = s_sel[0];
            bkey = s_sel[1];
        } else {
            unsigned mult;
            int64_t greater;
            select_in_list(cand, ncand, Cb, hist, scan, &akey, &mult, &greater);
            bkey = greater + (int64_t)mult >= Cb + 1 ? akey : list_max_below(cand, ncand, akey, scan);
        }
    } else {
        column_select_full(col, 1, a, L, Cb, hist, scan, cand, &s_ncand, &akey, &bkey);
    }
    if (tid == 0) beta_parts[b * n + j] = qb_threshold(key_float(akey), key_float(bkey), rule);
}

// beta_j = fp32((sum over b in order of (double) beta_parts[b][j]) / B).
__global__ void qb_beta_mean_kernel(const float* __restrict__ beta_parts, int64_t nb, int n, float* __restrict__ beta) {
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        double acc = 0.0;
        for (int64_t b = 0; b < nb; ++b) acc += (double)beta_parts[b * n + j];
        beta[j] = (float)(acc / (double)nb);
    }
}

namespace qb {
constexpr int kArcThreads = 256;     // 8 warps
constexpr int kArcBatch = 4;         // members per warp step (their loads in flight together)
constexpr int kArcWords = 256;       // bitmap words compacted per pass: at most 8192 members
constexpr int kArcSlices = 8;        // CTAs per row of W, each over 1/8 of the tokens
constexpr int kMemberCap = kArcWords * 32;
constexpr size_t kArcSmem = (size_t)(kArcThreads / 32) * kMaxExperts * (8 + 4) + (size_t)kMemberCap * 4;
}  // namespace qb

// Membership bitmap: bit i of row e is set when token i holds expert e.
__global__ void qb_member_bits_kernel(const int32_t* __restrict__ topk_idx, int64_t m, int k, int64_t words,
                                      uint32_t* __restrict__ mem) {
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= m * k) return;
    const int64_t i = q / k;
    const int e = topk_idx[q];
    atomicOr(&mem[(int64_t)e * words + (i >> 5)], 1u << (i & 31));
}

// Arc costs of the expert graph for the listed rows a = rows[blockIdx.x]:
// W[a][b] = min over tokens i holding a but not b of s_ia - s_ib (fp64), A[a][b] = that token
// (lowest token among equal costs). It builds every row once per SOLVE (later moves update W in
// place: qb_arc_inc_kernel, qb_arc_recompute_kernel). Each row is split over gridDim.y CTAs,
// slice y taking the y-th range of bitmap words (tokens), so the rows spread over the GPU.
// The members of a in the slice come from the bitmap (compacted into shared memory,
// kMemberCap at a time); warp w takes members in batches of kArcBatch, lanes own columns
// b = lane + 32 q; the warps' minima are folded in warp order, and the last slice of the row to
// finish folds the slices' partials in slice order.
template <int NT>
__global__ void __launch_bounds__(qb::kArcThreads, 2)
qb_arc_kernel(const float* __restrict__ s, int64_t m, int n, int k, const int32_t* __restrict__ topk_idx,
              const uint32_t* __restrict__ mem, int64_t words, const int32_t* __restrict__ rows,
              const int32_t* __restrict__ nrows, double* __restrict__ W, int32_t* __restrict__ A,
              const int32_t* __restrict__ status, double* Wp, int32_t* Ap, int32_t* tickets) {
    if (status[qb::kStError] || status[qb::kStDone]) return;
    if ((int)blockIdx.x >= *nrows) return;
    const int S = gridDim.y, slice = blockIdx.y;
    const int64_t per = (words + S - 1) / S;
    const int64_t wbeg = min(words, (int64_t)slice * per), wend = min(words, wbeg + per);
    constexpr int NW = qb::kArcThreads / 32, B = qb::kArcBatch;
    extern __shared__ unsigned char arc_smem[];
    double* bw = reinterpret_cast<double*>(arc_smem);                       // [NW][256]
    int32_t* ba = reinterpret_cast<int32_t*>(bw + NW * kMaxExperts);         // [NW][256]
    int32_t* list = ba + NW * kMaxExperts;                                   // [kMemberCap]
    __shared__ int nlist;
    const int a = rows[blockIdx.x];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t* row = mem + (int64_t)a * words;
    double best[NT];
    int32_t arg[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) { best[q] = INFINITY; arg[q] = 0x7fffffff; }
    for (int64_t w0 = wbeg; w0 < wend; w0 += qb::kArcWords) {
        // compact the members held in the next kArcWords bitmap words (token order is not needed:
        // ties go to the lowest token explicitly)
        if (threadIdx.x == 0) nlist = 0;
        __syncthreads();
        {
            const int64_t wi = w0 + threadIdx.x;
            const uint32_t bits = (threadIdx.x < qb::kArcWords && wi < wend) ? row[wi] : 0u;
            const int c = __popc(bits);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int base = 0;
            if (lane == 31 && incl) base = atomicAdd(&nlist, incl);
            base = __shfl_sync(0xffffffffu, base, 31);
            int pos = base + incl - c;
            uint32_t bb = bits;
            while (bb) {
                const int bit = __ffs(bb) - 1;
                bb &= bb - 1;
                list[pos++] = (int32_t)((wi << 5) + bit);
            }
        }
        __syncthreads();
        const int cnt = nlist;
        for (int p0 = warp * B; p0 < cnt; p0 += NW * B) {
            int32_t id[B];
            float sa[B], sb[B][NT];
            int32_t ex[B];
#pragma unroll
            for (int u = 0; u < B; ++u) {
                id[u] = p0 + u < cnt ? list[p0 + u] : -1;
                const int64_t ti = id[u] >= 0 ? id[u] : 0;
                sa[u] = s[ti * n + a];
                ex[u] = lane < k ? topk_idx[ti * k + lane] : -1;
#pragma unroll
                for (int q = 0; q < NT; ++q) sb[u][q] = (lane + 32 * q < n) ? s[ti * n + lane + 32 * q] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < B; ++u) {
                if (id[u] < 0) continue;  // warp-uniform
                uint32_t in = 0;  // bit q: column lane + 32 q belongs to the member's set (set by its owner lane)
                for (int r = 0; r < k; ++r) {
                    const int e = k <= 32 ? __shfl_sync(0xffffffffu, ex[u], r & 31) : topk_idx[(int64_t)id[u] * k + r];
                    if ((e & 31) == lane) in |= 1u << (e >> 5);
                }
#pragma unroll
                for (int q = 0; q < NT; ++q) {
                    const int b = lane + 32 * q;
                    if (b < n && !((in >> q) & 1u)) {
                        const double c = (double)sa[u] - (double)sb[u][q];
                        if (c < best[q] || (c == best[q] && id[u] < arg[q])) { best[q] = c; arg[q] = id[u]; }
                    }
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < NT; ++q) { bw[warp * kMaxExperts + lane + 32 * q] = best[q]; ba[warp * kMaxExperts + lane + 32 * q] = arg[q]; }
    __syncthreads();
    // fold the warps in order; with one slice that is the row of W, else this slice's partial
    const int64_t pslot = ((int64_t)blockIdx.x * S + slice) * n;
    for (int b = threadIdx.x; b < n; b += blockDim.x) {
        double bb = INFINITY;
        int32_t aa = -1;
        for (int w = 0; w < NW; ++w) {
            const double c = bw[w * kMaxExperts + b];
            const int32_t t = ba[w * kMaxExperts + b];
            if (c < bb || (c == bb && c != INFINITY && t < aa)) { bb = c; aa = t; }
        }
        if (S == 1) {
            W[(int64_t)a * n + b] = bb;
            A[(int64_t)a * n + b] = bb == INFINITY ? -1 : aa;
        } else {
            Wp[pslot + b] = bb;
            Ap[pslot + b] = aa;
        }
    }
    if (S == 1) return;
    // the last slice to finish folds the slices in slice order (token ranges ascend with the slice,
    // so the lowest token among equal costs wins as in one pass) and re-arms the row's ticket
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&tickets[blockIdx.x], 1) == S - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int b = threadIdx.x; b < n; b += blockDim.x) {
        double bb = INFINITY;
        int32_t aa = -1;
        for (int sl = 0; sl < S; ++sl) {
            const int64_t ps = ((int64_t)blockIdx.x * S + sl) * n + b;
            const double c = __ldcg(Wp + ps);
            const int32_t t = __ldcg(Ap + ps);
            if (c < bb || (c == bb && c != INFINITY && t < aa)) { bb = c; aa = t; }
        }
        W[(int64_t)a * n + b] = bb;
        A[(int64_t)a * n + b] = bb == INFINITY ? -1 : aa;
    }
    if (threadIdx.x == 0) tickets[blockIdx.x] = 0;
}

// Compact the indices a < n with flag[a] != 0, in increasing order, into out[] and *count
// (block-wide; threads 0..255 each own one flag, a ballot per warp and a prefix over the warps).
// Ends with a barrier, so out and *count are visible to every thread.
__device__ __forceinline__ void compact_flags(const unsigned char* flag, int n, int32_t* out, int32_t* count,
                                              int* wcount) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool f = tid < n && flag[tid];
    uint32_t bal = 0;
    if (tid < kMaxExperts) {
        bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) wcount[warp] = __popc(bal);
    }
    __syncthreads();
    if (tid < kMaxExperts) {
        int off = 0;
        for (int w = 0; w < warp; ++w) off += wcount[w];
        if (f) out[off + __popc(bal & ((1u << lane) - 1u))] = tid;
        if (tid == kMaxExperts - 1) {
            int tot = 0;
            for (int w = 0; w < kMaxExperts / 32; ++w) tot += wcount[w];
            *count = tot;
        }
    }
    __syncthreads();
}

namespace qb {
constexpr int kRepCtas = 8;       // one cluster of 8 CTAs
constexpr int kRepThreads = 256;  // thread (part 0..7, column 0..31)
constexpr int kRepCols = 32;      // columns of W per CTA (n <= 256)
}  // namespace qb

// One augmentation (one unit of excess) on one 8-CTA cluster. CTA c owns the columns
// b = 32 c .. 32 c + 31 of W, held in its shared memory. Jacobi Bellman-Ford rounds from the
// over-full experts: each round every CTA relaxes its own columns from the experts whose
// distance changed in the previous round (the frontier; the same fixpoint as full rounds), then
// writes its columns' new distances and change flags into the next-round buffers of every CTA
// of the cluster (distributed shared memory) and one cluster barrier ends the round, so every
// CTA holds the same full distance vector. Then the predecessors (lowest a with
// dist[a] + W[a][b] == dist[b] whose distance settled in an earlier round than b's: the value that
// set dist[b] in its last round came from such an a, and with zero-cost cycles several arcs can be
// tight) of each CTA's columns go to CTA 0, whose thread 0 takes the
// nearest under-full expert (lowest index on ties), walks the path and moves each arc's token,
// and CTA 0 lists the rows of W the moves invalidate (the old set of every moved token, plus the
// expert it moved to) for the next arc launch. All decisions that end loops or return are made
// on data every CTA holds identically, so every CTA reaches every cluster barrier.
__global__ void __launch_bounds__(qb::kRepThreads, 1)
qb_repair_step_kernel(int n, int64_t C, int k, const double* __restrict__ W, const int32_t* __restrict__ A,
                      int32_t* __restrict__ counts, int32_t* __restrict__ topk_idx, int32_t* __restrict__ status,
                      int32_t* __restrict__ moves, int32_t* __restrict__ nmoves, uint32_t* __restrict__ mem,
                      int64_t words) {
    extern __shared__ double wsl[];  // [n][32]: this CTA's columns of W
    __shared__ double dist[2][kMaxExperts];
    __shared__ unsigned char chg[2][kMaxExperts];
    __shared__ double part_d[8][qb::kRepCols];
    __shared__ int part_p[8][qb::kRepCols];
    __shared__ int pred[kMaxExperts];
    __shared__ int settle[kMaxExperts];  // the round (1-based) of each expert's last decrease, 0 for the roots
    __shared__ int front[kMaxExperts], nfront, wcount[kMaxExperts / 32];
    __shared__ int any_over;
    const int tid = threadIdx.x, bl = tid & 31, part = tid >> 5;
    const uint32_t crank = ptx::cluster_ctarank();
    const int b = (int)crank * qb::kRepCols + bl;
    const bool own = b < n;
    // status is read by every CTA before any of them can change it (CTA 0 writes it at the end)
    if (status[qb::kStError] || status[qb::kStDone]) return;
    for (int q = tid; q < n * qb::kRepCols; q += blockDim.x) {
        const int a = q / qb::kRepCols, j = (int)crank * qb::kRepCols + (q % qb::kRepCols);
        wsl[q] = j < n ? W[(int64_t)a * n + j] : INFINITY;
    }
    if (tid == 0) any_over = 0;
    __syncthreads();
    for (int e = tid; e < kMaxExperts; e += blockDim.x) {
        const bool over = e < n && counts[e] > C;
        dist[0][e] = over ? 0.0 : INFINITY;
        dist[1][e] = INFINITY;
        chg[0][e] = over ? 1 : 0;
        chg[1][e] = 0;
        pred[e] = -1;
        settle[e] = 0;
        if (over) atomicOr(&any_over, 1);
    }
    __syncthreads();
    if (!any_over) {  // the same counts in every CTA: all return here together
        if (crank == 0 && tid == 0) { status[qb::kStDone] = 1; nmoves[0] = 0; nmoves[1] = 0; }
        return;
    }
    ptx::cluster_sync();  // every CTA's buffers are initialised before any remote write
    int cur = 0;
    bool settled = false;
    int my_settle = 0;  // column b's settle round (the fold threads)
    for (int round = 0; round <= n; ++round) {
        // warp `part` relaxes from the changed experts among 32 part .. 32 part + 31 (a ballot of
        // the change flags, no compaction); the rounds end when no flag is set in any CTA's copy
        // (every CTA holds the same flags)
        const int a0 = part * 32;
        const bool mine = a0 + bl < n && chg[cur][a0 + bl];
        uint32_t fm = __ballot_sync(0xffffffffu, mine);
        if (!__syncthreads_or(mine)) { settled = true; break; }
        double best = INFINITY;
        if (own) {
            while (fm) {
                const int a = a0 + __ffs(fm) - 1;
                fm &= fm - 1;
                const double w = wsl[a * qb::kRepCols + bl];
                if (a != b && w != INFINITY) {
                    const double c = dist[cur][a] + w;
                    if (c < best) best = c;
                }
            }
        }
        part_d[part][bl] = best;
        __syncthreads();
        if (part == 0 && own) {  // fold the 8 partials, then this column into every CTA's next-round buffers
            double nd = dist[cur][b];
            for (int p = 0; p < 8; ++p) nd = fmin(nd, part_d[p][bl]);
            const unsigned char nc = nd != dist[cur][b] ? 1 : 0;
            if (nc) my_settle = round + 1;
            for (int r = 0; r < qb::kRepCtas; ++r) {
                ptx::st_cluster_f64(ptx::mapa_shared(ptx::smem_u32(&dist[cur ^ 1][b]), (uint32_t)r), nd);
                ptx::st_cluster_u8(ptx::mapa_shared(ptx::smem_u32(&chg[cur ^ 1][b]), (uint32_t)r), nc);
            }
        }
        ptx::cluster_sync();
        cur ^= 1;
    }
    if (!settled) {  // still improving after n rounds: a negative cycle, which an optimal start excludes
        if (crank == 0 && tid == 0) {
            status[qb::kStError] = 1;
            record_error(kErrRepair);
            nmoves[0] = 0;
            nmoves[1] = 0;
        }
        return;
    }
    // every CTA learns every column's settle round
    if (part == 0 && own)
        for (int r = 0; r < qb::kRepCtas; ++r)
            ptx::st_cluster_s32(ptx::mapa_shared(ptx::smem_u32(&settle[b]), (uint32_t)r), my_settle);
    ptx::cluster_sync();
    // predecessors of this CTA's columns, over the reachable experts, to CTA 0
    for (int e = tid; e < kMaxExperts; e += blockDim.x) chg[cur ^ 1][e] = (e < n && dist[cur][e] != INFINITY) ? 1 : 0;
    __syncthreads();
    compact_flags(chg[cur ^ 1], n, front, &nfront, wcount);
    const int nr = nfront;
    int pa = 0x7fffffff;
    if (own && dist[cur][b] != INFINITY) {
        const double db = dist[cur][b];
        for (int f = part; f < nr; f += 8) {
            const int a = front[f];
            const double w = wsl[a * qb::kRepCols + bl];
            if (a != b && w != INFINITY && dist[cur][a] + w == db && settle[a] < settle[b] && a < pa) pa = a;
        }
    }
    part_p[part][bl] = pa;
    __syncthreads();
    if (part == 0 && own) {
        int p = 0x7fffffff;
        for (int q = 0; q < 8; ++q) p = min(p, part_p[q][bl]);
        ptx::st_cluster_s32(ptx::mapa_shared(ptx::smem_u32(&pred[b]), 0u), p == 0x7fffffff ? -1 : p);
    }
    ptx::cluster_sync();  // after this, no CTA touches another's shared memory
    if (crank != 0) return;
    const double* dd = dist[cur];
    if (tid == 0) {
        int t = -1;
        for (int e = 0; e < n; ++e)
            if (counts[e] < C && dd[e] != INFINITY && (t < 0 || dd[e] < dd[t])) t = e;
        bool ok = t >= 0;
        int node = t, len = 0;
        int path[kMaxExperts + 1];
        if (ok) {
            path[len++] = node;
            while (pred[node] >= 0 && len <= n) { node = pred[node]; path[len++] = node; }
            ok = len <= n && counts[node] > C;
        }
        int nm = 0;
        for (int p = len - 1; ok && p > 0; --p) {
            const int a = path[p], bb = path[p - 1];
            const int32_t i = A[(int64_t)a * n + bb];
            if (i < 0) { ok = false; break; }
            int32_t* row = topk_idx + (int64_t)i * k;
            int pos = -1;
            bool hasb = false;
            for (int r = 0; r < k; ++r) {
                if (row[r] == a) pos = r;
                if (row[r] == bb) hasb = true;
            }
            if (pos < 0 || hasb) { ok = false; break; }
            mem[(int64_t)a * words + (i >> 5)] &= ~(1u << (i & 31));
            mem[(int64_t)bb * words + (i >> 5)] |= 1u << (i & 31);
            int r = pos;
            row[r] = bb;
            while (r > 0 && row[r - 1] > row[r]) { const int t2 = row[r - 1]; row[r - 1] = row[r]; row[r] = t2; --r; }
            while (r + 1 < k && row[r + 1] < row[r]) { const int t2 = row[r + 1]; row[r + 1] = row[r]; row[r] = t2; ++r; }
            // the move, for the arc update that follows: token i went from a to bb
            moves[3 * nm] = i;
            moves[3 * nm + 1] = a;
            moves[3 * nm + 2] = bb;
            ++nm;
        }
        if (!ok) {
            status[qb::kStError] = 1;
            record_error(kErrRepair);
            nm = 0;
        } else {
            counts[node] -= 1;
            counts[t] += 1;
            status[qb::kStAugments] += 1;
        }
        nmoves[0] = nm;
        nmoves[1] = 0;  // entries queued for recomputation by the next arc update
    }
}

static cudaError_t launch_repair_step(int n, int64_t C, int k, const double* W, const int32_t* A, int32_t* counts,
                                      int32_t* topk_idx, int32_t* status, int32_t* moves, int32_t* nmoves,
                                      uint32_t* mem, int64_t words, cudaStream_t stream) {
    const size_t smem = (size_t)n * qb::kRepCols * sizeof(double);
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(qb_repair_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)((size_t)kMaxExperts * qb::kRepCols * sizeof(double)));
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(qb::kRepCtas);
    cfg.blockDim = dim3(qb::kRepThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = qb::kRepCtas;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qb_repair_step_kernel, n, C, k, W, A, counts, topk_idx, status, moves, nmoves,
                              mem, words);
}

// Arc costs after a repair move, updated in place instead of rebuilding rows. An entry
// W[x][y] is a minimum over the eligible tokens (holding x, not y), taken on (cost, token). A
// move changes the eligibility of its moved tokens only: a token that became eligible enters
// the minimum; a token that stopped being eligible changes the entry only if it was the
// recorded argmin, and those entries are queued for recomputation from the membership
// bitmaps. A minimum over a set that lost a token other than its argmin is unchanged, so the
// result equals the rebuilt rows bit for bit. CTA x takes row x, thread y column y; the moved
// tokens' expert sets after the move come from topk_idx (before it: bb replaced by a).
__global__ void __launch_bounds__(kMaxExperts)
qb_arc_inc_kernel(const float* __restrict__ s, int n, int k, const int32_t* __restrict__ topk_idx,
                  const int32_t* __restrict__ moves, int32_t* __restrict__ nmoves, const int32_t* __restrict__ status,
                  double* __restrict__ W, int32_t* __restrict__ A, int32_t* __restrict__ rec) {
    if (status[qb::kStError] || status[qb::kStDone]) return;
    const int L = nmoves[0];
    if (L <= 0) return;
    __shared__ uint32_t nset[kMaxExperts][kMaxExperts / 32];
    __shared__ int32_t mv[kMaxExperts][3];
    const int tid = threadIdx.x;
    for (int q = tid; q < L * (kMaxExperts / 32); q += blockDim.x) nset[q / (kMaxExperts / 32)][q % (kMaxExperts / 32)] = 0;
    for (int q = tid; q < 3 * L; q += blockDim.x) mv[q / 3][q % 3] = moves[q];
    __syncthreads();
    for (int q = tid; q < L * k; q += blockDim.x) {
        const int p = q / k;
        const int e = topk_idx[(int64_t)mv[p][0] * k + (q - p * k)];
        atomicOr(&nset[p][e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    const int x = blockIdx.x, y = tid;
    if (y >= n || x == y) return;
    const int64_t at = (int64_t)x * n + y;
    double w = W[at];
    int32_t t = A[at];
    bool re = false, changed = false;
    for (int p = 0; p < L; ++p) {
        const int32_t i = mv[p][0];
        const int a = mv[p][1], bb = mv[p][2];
        const bool xn = (nset[p][x >> 5] >> (x & 31)) & 1u, yn = (nset[p][y >> 5] >> (y & 31)) & 1u;
        const bool xo = x == a ? true : (x == bb ? false : xn);
        const bool yo = y == a ? true : (y == bb ? false : yn);
        const bool el_new = xn && !yn, el_old = xo && !yo;
        if (el_old && !el_new) {
            if (t == i) re = true;
        } else if (el_new && !el_old) {
            const double c = (double)s[(int64_t)i * n + x] - (double)s[(int64_t)i * n + y];
            if (c < w || (c == w && i < t)) { w = c; t = i; changed = true; }
        }
    }
    if (re) rec[atomicAdd(&nmoves[1], 1)] = (int32_t)at;
    else if (changed) { W[at] = w; A[at] = t; }
}

// The queued entries, recomputed from the membership bitmaps: W[x][y] = min over tokens in
// mem[x] and not in mem[y] of s_tx - s_ty (fp64, lowest token on ties). One CTA per entry.
__global__ void __launch_bounds__(256)
qb_arc_recompute_kernel(const float* __restrict__ s, int64_t m, int n, const uint32_t* __restrict__ mem,
                        int64_t words, const int32_t* __restrict__ nmoves, const int32_t* __restrict__ rec,
                        const int32_t* __restrict__ status, double* __restrict__ W, int32_t* __restrict__ A) {
    if (status[qb::kStError] || status[qb::kStDone]) return;
    const int nrec = nmoves[1];
    __shared__ double rw[8];
    __shared__ int32_t rt[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = blockIdx.x; e < nrec; e += gridDim.x) {
        const int32_t at = rec[e];
        const int x = at / n, y = at - x * n;
        const uint32_t* mx = mem + (int64_t)x * words;
        const uint32_t* my = mem + (int64_t)y * words;
        double best = INFINITY;
        int32_t arg = 0x7fffffff;
        for (int64_t w0 = 0; w0 < words; w0 += 4 * (int64_t)blockDim.x) {
            uint32_t bits[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t wi = w0 + tid + (int64_t)u * blockDim.x;
                bits[u] = wi < words ? (mx[wi] & ~my[wi]) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t wi = w0 + tid + (int64_t)u * blockDim.x;
                uint32_t b = bits[u];
                while (b) {
                    const int bit = __ffs(b) - 1;
                    b &= b - 1;
                    const int64_t ti = (wi << 5) + bit;
                    if (ti >= m) break;
                    const double c = (double)s[ti * n + x] - (double)s[ti * n + y];
                    if (c < best || (c == best && (int32_t)ti < arg)) { best = c; arg = (int32_t)ti; }
                }
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int32_t oa = __shfl_xor_sync(0xffffffffu, arg, o);
            if (ob < best || (ob == best && oa < arg)) { best = ob; arg = oa; }
        }
        if (lane == 0) { rw[warp] = best; rt[warp] = arg; }
        __syncthreads();
        if (tid == 0) {
            double bw = INFINITY;
            int32_t ba = 0x7fffffff;
            for (int q = 0; q < (int)(blockDim.x >> 5); ++q)
                if (rw[q] < bw || (rw[q] == bw && rt[q] < ba)) { bw = rw[q]; ba = rt[q]; }
            W[at] = bw;
            A[at] = bw == INFINITY ? -1 : ba;
        }
        __syncthreads();
    }
}

__global__ void qb_all_rows_kernel(int n, int32_t* __restrict__ rows, int32_t* __restrict__ nrows) {
    for (int e = threadIdx.x; e < n; e += blockDim.x) rows[e] = e;
    if (threadIdx.x == 0) *nrows = n;
}

__global__ void qb_info_kernel(const int32_t* __restrict__ counts, int n, int64_t C, const int32_t* __restrict__ status,
                               int32_t iters, int tie_slot, int32_t* __restrict__ info) {
    if (threadIdx.x != 0) return;
    int64_t excess = 0;
    for (int e = 0; e < n; ++e) if (counts[e] > C) excess += counts[e] - C;
    info[0] = iters;
    info[1] = status[qb::kStAugments];
    info[2] = (int32_t)excess;
    info[3] = status[tie_slot];
}

struct QBWorkspace {
    float* sT;
    float* alpha;
    int32_t* counts;
    int32_t* status;
    double* W;
    int32_t* A;
    int32_t* rows;
    int32_t* nrows;
    uint32_t* mem;   // [n][ceil(m / 32)] membership bitmap
    uint32_t* win;   // [n] window half-widths of the column pass (0: default)
    double* Wp;      // [n][kArcSlices][n] per-slice partial arc costs
    int32_t* Ap;     // [n][kArcSlices][n] their tokens
    int32_t* arc_tickets;  // [n] slices done per row (re-armed by the folding slice)
    uint32_t* g_above;     // [n] column pass: keys above the window (cleared by the select kernel)
    uint32_t* g_ncand;     // [n] column pass: keys inside the window
    uint32_t* g_cand;      // [n][kGCap] column pass: the keys inside the window
    int32_t* moves;        // [n][3] the last repair move: token, from, to per hop
    int32_t* nmoves;       // [2] hops of the last move, entries queued for recomputation
    int32_t* rec;          // [n * n] queued entries x * n + y
    float* beta_parts;     // [kMaxMiniBatches][n] per-mini-batch beta of the mini-batch step
};

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

static size_t qb_layout(int64_t m, int n, int k, QBWorkspace* w, char* base) {
    (void)k;
    size_t off = 0;
    auto take = [&](size_t bytes) { char* p = base ? base + off : nullptr; off += align256(bytes); return p; };
    char* p;
    p = take(sizeof(float) * (size_t)m * n);            if (w) w->sT = (float*)p;
    p = take(sizeof(float) * (size_t)m);                if (w) w->alpha = (float*)p;
    // the words every call clears, in one block: status, counts (2 n), win (n), g_above (n), g_ncand (n)
    p = take(sizeof(int32_t) * ((size_t)qb::kStWords + 5 * (size_t)n));
    if (w) {
        w->status = (int32_t*)p;
        w->counts = w->status + qb::kStWords;
        w->win = (uint32_t*)(w->counts + 2 * n);
        w->g_above = w->win + n;
        w->g_ncand = w->g_above + n;
    }
    p = take(sizeof(double) * (size_t)n * n);           if (w) w->W = (double*)p;
    p = take(sizeof(int32_t) * (size_t)n * n);          if (w) w->A = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->rows = (int32_t*)p;
    p = take(sizeof(int32_t));                          if (w) w->nrows = (int32_t*)p;
    p = take(sizeof(uint32_t) * (size_t)n * (size_t)((m + 31) / 32)); if (w) w->mem = (uint32_t*)p;
    p = take(sizeof(double) * (size_t)n * qb::kArcSlices * n);  if (w) w->Wp = (double*)p;
    p = take(sizeof(int32_t) * (size_t)n * qb::kArcSlices * n); if (w) w->Ap = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->arc_tickets = (int32_t*)p;
    p = take(sizeof(uint32_t) * (size_t)n * qb::kGCap); if (w) w->g_cand = (uint32_t*)p;
    p = take(sizeof(int32_t) * 3 * (size_t)(n + 1));    if (w) w->moves = (int32_t*)p;
    p = take(sizeof(int32_t) * 2);                      if (w) w->nmoves = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n * n);          if (w) w->rec = (int32_t*)p;
    p = take(sizeof(float) * (size_t)qb::kMaxMiniBatches * n); if (w) w->beta_parts = (float*)p;
    return off;
}

size_t balance_workspace_bytes(int64_t m, int32_t n, int32_t k) { return qb_layout(m, n, k, nullptr, nullptr); }

template <int NT, bool TRANS, bool SWEEP>
static void launch_row_tt(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                          int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip, float* sT,
                          const RowSweep& sw, cudaStream_t stream) {
    const size_t smem = 2 * (size_t)qb::kRowTile * n * sizeof(float);
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(qb_row_kernel<NT, TRANS, SWEEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(2 * (size_t)qb::kRowTile * kMaxExperts * sizeof(float)));
        attr = true;
    }
    // tiles spread evenly: every CTA takes the same number of tiles (the last ones one fewer)
    const int64_t ntiles = (m + qb::kRowTile - 1) / qb::kRowTile;
    const int64_t slots = (int64_t)kNumSMs * 3;
    const int64_t per = (ntiles + slots - 1) / slots;
    int64_t blocks = per > 0 ? (ntiles + per - 1) / per : 1;
    if (blocks < 1) blocks = 1;
    // bulk copies need a 16-byte aligned s (every tile then starts on a 16-byte boundary)
    const int bulk = (reinterpret_cast<uintptr_t>(s) & 15) == 0;
    qb_row_kernel<NT, TRANS, SWEEP><<<(unsigned)blocks, qb::kRowThreads, smem, stream>>>(
        s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, bulk, sw);
}

template <int NT, bool TRANS, bool SWEEP>
static void launch_row_tpr_tt(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                              int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip, float* sT,
                              const RowSweep& sw, cudaStream_t stream) {
    const size_t smem = tpr_dyn_smem<NT>();
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(qb_row_tpr_kernel<NT, TRANS, SWEEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        attr = true;
    }
    const int64_t ntiles = (m + 31) / 32;
    int64_t blocks = (ntiles + qb::kTprWarps - 1) / qb::kTprWarps;
    if (blocks > kNumSMs) blocks = kNumSMs;
    if (blocks < 1) blocks = 1;
    // one bulk copy per row: a 16-byte aligned s and rows of a multiple of 16 bytes
    const int bulk = (reinterpret_cast<uintptr_t>(s) & 15) == 0 && n % 4 == 0;
    qb_row_tpr_kernel<NT, TRANS, SWEEP><<<(unsigned)blocks, qb::kTprWarps * 32, smem, stream>>>(
        s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, bulk, sw);
}

template <int NT, bool SWEEP, bool SIGN>
static void launch_row_tpr2_t(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                              int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip,
                              const RowSweep& sw, int32_t* sign_counts, cudaStream_t stream) {
    const size_t smem = tpr2_dyn_smem();
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(qb_row_tpr2_kernel<NT, SWEEP, SIGN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        attr = true;
    }
    const int64_t ntiles = (m + 31) / 32;
    int64_t blocks = (ntiles + qb::kTpr2Warps - 1) / qb::kTpr2Warps;
    if (blocks > kNumSMs) blocks = kNumSMs;
    if (blocks < 1) blocks = 1;
    // programmatic dependent launch: the pass's prologue overlaps the previous launch's tail
    launch_pdl(qb_row_tpr2_kernel<NT, SWEEP, SIGN>, dim3((unsigned)blocks), dim3(qb::kTpr2Warps * 32), smem, stream,
               s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sw, sign_counts);
}

// Returns true when the launched pass also counted sign_counts (then no separate count is needed).
template <int NT>
static bool launch_row_t(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                         int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip, float* sT,
                         const RowSweep* sw, int32_t* sign_counts, cudaStream_t stream) {
    const RowSweep none{nullptr, nullptr, nullptr, nullptr};
    if (k >= 1 && k + 1 <= (n + NT - 1) / NT) {
        // thread-per-row selection: the (k+1)-th largest of the 32 column-group maxima exists;
        // without a transposed copy to write, the rows are read from global memory
        if (!sT) {
            if (sign_counts) launch_row_tpr2_t<NT, false, true>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, none, sign_counts, stream);
            else if (sw) launch_row_tpr2_t<NT, true, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, *sw, nullptr, stream);
            else launch_row_tpr2_t<NT, false, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, none, nullptr, stream);
            return sign_counts != nullptr;
        }
        if (sw) {
            if (sT) launch_row_tpr_tt<NT, true, true>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, *sw, stream);
            else launch_row_tpr_tt<NT, false, true>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, *sw, stream);
        } else {
            if (sT) launch_row_tpr_tt<NT, true, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, none, stream);
            else launch_row_tpr_tt<NT, false, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, none, stream);
        }
        return false;
    }
    if (sw) {
        if (sT) launch_row_tt<NT, true, true>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, *sw, stream);
        else launch_row_tt<NT, false, true>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, *sw, stream);
    } else {
        if (sT) launch_row_tt<NT, true, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, none, stream);
        else launch_row_tt<NT, false, false>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, none, stream);
    }
    return false;
}

// sT != nullptr: this row pass also writes s transposed into sT (the first pass of a call).
// sw != nullptr: it also runs the column pass's window sweep on its rows.
// sign_counts != nullptr (with sT and sw null): the pass may also count the sign step's
// indicators; the return value says whether it did.
static bool launch_row(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                       int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip, float* sT,
                       const RowSweep* sw, cudaStream_t stream, int32_t* sign_counts = nullptr) {
    if (n <= 32) return launch_row_t<1>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, sw, sign_counts, stream);
    if (n <= 64) return launch_row_t<2>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, sw, sign_counts, stream);
    if (n <= 128) return launch_row_t<4>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, sw, sign_counts, stream);
    return launch_row_t<8>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, sT, sw, sign_counts, stream);
}

// The column pass's select: one CTA per column (the window sweep ran inside the row pass). sT: s
// transposed (SOLVE), read by the select kernel's full path when the window missed; nullptr:
// that path reads the column from s with stride n.
static void launch_col(const float* s, const float* sT, int64_t m, int n, int64_t C, const QBWorkspace& w, int rule,
                       float* beta, const int32_t* counts, int32_t* counts_next, int iter, int check,
                       cudaStream_t stream, int32_t* info = nullptr) {
    launch_pdl(qb_col_kernel, dim3((unsigned)n), dim3(qb::kColThreads), qb::kColSmem, stream, s, sT, m, n, C,
               (const float*)w.alpha, rule, beta, counts_next, w.status, iter, check, w.win, w.g_above, w.g_ncand,
               (const uint32_t*)w.g_cand, counts, (int)qb::kStTies0, info);
}

template <int NT>
static void launch_arc_t(const float* s, int64_t m, int n, int k, const int32_t* topk_idx, const QBWorkspace& w,
                         cudaStream_t stream) {
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(qb_arc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qb::kArcSmem);
        attr = true;
    }
    qb_arc_kernel<NT><<<dim3((unsigned)n, qb::kArcSlices), qb::kArcThreads, qb::kArcSmem, stream>>>(
        s, m, n, k, topk_idx, w.mem, (m + 31) / 32, w.rows, w.nrows, w.W, w.A, w.status, w.Wp, w.Ap,
        w.arc_tickets);
}

static void launch_arc(const float* s, int64_t m, int n, int k, const int32_t* topk_idx, const QBWorkspace& w,
                       cudaStream_t stream) {
    if (n <= 32) launch_arc_t<1>(s, m, n, k, topk_idx, w, stream);
    else if (n <= 64) launch_arc_t<2>(s, m, n, k, topk_idx, w, stream);
    else if (n <= 128) launch_arc_t<4>(s, m, n, k, topk_idx, w, stream);
    else launch_arc_t<8>(s, m, n, k, topk_idx, w, stream);
}

static void launch_arc_update(const float* s, int64_t m, int n, int k, const int32_t* topk_idx, const QBWorkspace& w,
                              cudaStream_t stream) {
    qb_arc_inc_kernel<<<n, kMaxExperts, 0, stream>>>(s, n, k, topk_idx, w.moves, w.nmoves, w.status, w.W, w.A,
                                                     w.rec);
    qb_arc_recompute_kernel<<<kNumSMs * 4, 256, 0, stream>>>(s, m, n, w.mem, (m + 31) / 32, w.nmoves, w.rec,
                                                             w.status, w.W, w.A);
}


// SignSGD on beta: count_j = #{i : fp32(s_ij - alpha_i) > beta_j} over the rows of s (one warp
// per token, lane counters for the columns lane + 32 q, folded per CTA in shared memory).
template <int NT>
__global__ void __launch_bounds__(256)
qb_sign_count_kernel(const float* __restrict__ s, int64_t m, int n, const float* __restrict__ alpha,
                     const float* __restrict__ beta, int32_t* __restrict__ counts) {
    __shared__ int cnt[kMaxExperts];
    __shared__ float sb[kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31;
    for (int j = tid; j < n; j += blockDim.x) { cnt[j] = 0; sb[j] = beta[j]; }
    __syncthreads();
    int c[NT];
#pragma unroll
    for (int q = 0; q < NT; ++q) c[q] = 0;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x / 32) + (tid >> 5); i < m; i += warps) {
        const float a = alpha[i];
#pragma unroll
        for (int q = 0; q < NT; ++q) {
            const int j = lane + 32 * q;
            if (j < n && __fsub_rn(s[i * n + j], a) > sb[j]) ++c[q];
        }
    }
#pragma unroll
    for (int q = 0; q < NT; ++q)
        if (lane + 32 * q < n && c[q]) atomicAdd(&cnt[lane + 32 * q], c[q]);
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
}

__global__ void qb_sign_update_kernel(const int32_t* __restrict__ counts, int n, int64_t C, float gamma,
                                      float* __restrict__ beta) {
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int64_t c = counts[j];
        if (c > C) beta[j] = __fadd_rn(beta[j], gamma);        // gradient C - c < 0
        else if (c < C) beta[j] = __fsub_rn(beta[j], gamma);   // gradient > 0
    }
}

int run_balance_sign_step(const float* s, int64_t m, int n, int k, float* beta, float gamma, int rule,
                          int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream, const char** err) {
    QBWorkspace w;
    qb_layout(m, n, k, &w, static_cast<char*>(workspace));
    const int64_t C = m * k / n;
    cudaError_t ce;
    if ((ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * (qb::kStWords + 2 * n), stream)) != cudaSuccess)
        goto fail;
    {
        int32_t* sc = w.counts + n;  // chi counts, separate from the pick counts
        const bool counted = launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status,
                                        qb::kStTies0, 0, nullptr, nullptr, stream, sc);
        int64_t blocks = (m + 7) / 8;
        if (blocks > (int64_t)kNumSMs * 8) blocks = (int64_t)kNumSMs * 8;
        if (blocks < 1) blocks = 1;
        if (counted) {
        } else if (n <= 32) qb_sign_count_kernel<1><<<(unsigned)blocks, 256, 0, stream>>>(s, m, n, w.alpha, beta, sc);
        else if (n <= 64) qb_sign_count_kernel<2><<<(unsigned)blocks, 256, 0, stream>>>(s, m, n, w.alpha, beta, sc);
        else if (n <= 128) qb_sign_count_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(s, m, n, w.alpha, beta, sc);
        else qb_sign_count_kernel<8><<<(unsigned)blocks, 256, 0, stream>>>(s, m, n, w.alpha, beta, sc);
        qb_sign_update_kernel<<<1, 256, 0, stream>>>(sc, n, C, gamma, beta);
    }
    qb_info_kernel<<<1, 32, 0, stream>>>(w.counts, n, C, w.status, 1, qb::kStTies0, info);
    if ((ce = cudaGetLastError()) != cudaSuccess) goto fail;
    return MOE_OK;
fail:
    *err = cudaGetErrorString(ce);
    return MOE_ERR_CUDA;
}

// The practical QB step with beta averaged over mini-batches of seg_len tokens: the row pass of
// STEP (selection with the old beta; it also writes s transposed), one column select per
// (expert, mini-batch), the fixed-order mean. Fully asynchronous.
int run_balance_step_minibatch(const float* s, int64_t m, int n, int k, float* beta, int rule, int64_t seg_len,
                               int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                               const char** err) {
    QBWorkspace w;
    qb_layout(m, n, k, &w, static_cast<char*>(workspace));
    const int64_t C = m * k / n, nb = m / seg_len, Cb = seg_len * k / n;
    cudaError_t ce;
    static bool attr = false;
    if (!attr) {
        if ((ce = cudaFuncSetAttribute(qb_col_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)qb::kColSmem)) != cudaSuccess)
            goto fail;
        attr = true;
    }
    if ((ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * (qb::kStWords + 2 * n), stream)) != cudaSuccess)
        goto fail;
    launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status, qb::kStTies0, 0, w.sT, nullptr, stream);
    qb_col_slice_kernel<<<dim3((unsigned)n, (unsigned)nb), qb::kColThreads, qb::kColSmem, stream>>>(
        w.sT, m, n, seg_len, Cb, w.alpha, rule, w.beta_parts);
    qb_beta_mean_kernel<<<1, 256, 0, stream>>>(w.beta_parts, nb, n, beta);
    qb_info_kernel<<<1, 32, 0, stream>>>(w.counts, n, C, w.status, 1, qb::kStTies0, info);
    if ((ce = cudaGetLastError()) != cudaSuccess) goto fail;
    return MOE_OK;
fail:
    *err = cudaGetErrorString(ce);
    return MOE_ERR_CUDA;
}

// Returns a moe_status; SOLVE synchronises the stream between phases.
int run_balance_assign(const float* s, int64_t m, int n, int k, float* beta, int mode, int rule, int max_iters,
                       int max_repair, int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                       const char** err) {
    QBWorkspace w;
    qb_layout(m, n, k, &w, static_cast<char*>(workspace));
    const int64_t C = m * k / n;
    const RowSweep sweep{w.win, w.g_above, w.g_ncand, w.g_cand};
    cudaError_t ce;
    static bool col_attr = false;
    if (!col_attr) {
        if ((ce = cudaFuncSetAttribute(qb_col_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)qb::kColSmem)) != cudaSuccess)
            goto cuda_fail;
        col_attr = true;
    }
    // status, counts, windows and the column pass's counters: one block, one clear
    if ((ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * (qb::kStWords + 5 * n), stream)) != cudaSuccess)
        goto cuda_fail;
    if (mode == MOE_QB_STEP) {
        // one pass each; a window miss reads its column from s (no transposed copy)
        launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status, qb::kStTies0, 0, nullptr, &sweep,
                   stream);
        launch_col(s, nullptr, m, n, C, w, rule, beta, w.counts, w.counts + n, 0, 0, stream, info);
        if ((ce = cudaGetLastError()) != cudaSuccess) goto cuda_fail;
        return MOE_OK;
    }
    {
        // QB phase: row pass u uses beta after u updates; column pass u checks row pass u's counts first
        int32_t hstatus[qb::kStWords], hcounts[2 * kMaxExperts];
        for (int u0 = 0; u0 <= max_iters; u0 += qb::kBatch) {
            const int u1 = u0 + qb::kBatch - 1 < max_iters ? u0 + qb::kBatch - 1 : max_iters;
            for (int u = u0; u <= u1; ++u) {
                int32_t* cnt = w.counts + (u % 2) * n;
                // the sweep feeds the column pass that follows (none after the last row pass)
                launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, cnt, w.status,
                           u % 2 ? qb::kStTies1 : qb::kStTies0, 1, u == 0 ? w.sT : nullptr,
                           u < max_iters ? &sweep : nullptr, stream);
                if (u < max_iters)
                    launch_col(s, w.sT, m, n, C, w, rule, beta, cnt, w.counts + ((u + 1) % 2) * n, u, 1, stream);
            }
            if ((ce = cudaGetLastError()) != cudaSuccess) goto cuda_fail;
            if ((ce = cudaMemcpyAsync(hstatus, w.status, sizeof(hstatus), cudaMemcpyDeviceToHost, stream)) !=
                cudaSuccess)
                goto cuda_fail;
            if ((ce = cudaStreamSynchronize(stream)) != cudaSuccess) goto cuda_fail;
            if (hstatus[qb::kStQbDone]) break;
        }
        if ((ce = cudaMemcpyAsync(hcounts, w.counts, sizeof(int32_t) * 2 * n, cudaMemcpyDeviceToHost, stream)) !=
            cudaSuccess)
            goto cuda_fail;
        if ((ce = cudaStreamSynchronize(stream)) != cudaSuccess) goto cuda_fail;
        const int iters = hstatus[qb::kStIters];
        int32_t* final_counts = w.counts + (iters % 2) * n;
        int64_t excess = 0;
        for (int e = 0; e < n; ++e)
            if (hcounts[(iters % 2) * n + e] > C) excess += hcounts[(iters % 2) * n + e] - C;
        // exact finish: one shortest-path move per unit of excess; W is built for every row once,
        // then updated entry by entry after each move
        const int64_t moves = excess < max_repair ? excess : max_repair;
        if (moves > 0) {
            const int64_t words = (m + 31) / 32;
            if ((ce = cudaMemsetAsync(w.mem, 0, sizeof(uint32_t) * (size_t)n * (size_t)words, stream)) != cudaSuccess)
                goto cuda_fail;
            if ((ce = cudaMemsetAsync(w.arc_tickets, 0, sizeof(int32_t) * (size_t)n, stream)) != cudaSuccess)
                goto cuda_fail;
            qb_member_bits_kernel<<<(unsigned)((m * k + 255) / 256), 256, 0, stream>>>(topk_idx, m, k, words, w.mem);
            qb_all_rows_kernel<<<1, 256, 0, stream>>>(n, w.rows, w.nrows);
        }
        for (int64_t a = 0; a < moves; ++a) {
            if (a == 0) launch_arc(s, m, n, k, topk_idx, w, stream);           // every row once
            else launch_arc_update(s, m, n, k, topk_idx, w, stream);          // the entries the last move changed
            if ((ce = launch_repair_step(n, C, k, w.W, w.A, final_counts, topk_idx, w.status, w.moves, w.nmoves,
                                         w.mem, (m + 31) / 32, stream)) != cudaSuccess)
                goto cuda_fail;
        }
        qb_info_kernel<<<1, 32, 0, stream>>>(final_counts, n, C, w.status, iters,
                                             iters % 2 ? qb::kStTies1 : qb::kStTies0, info);
        if ((ce = cudaGetLastError()) != cudaSuccess) goto cuda_fail;
        int32_t hinfo[4];
        if ((ce = cudaMemcpyAsync(hinfo, info, sizeof(hinfo), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
            goto cuda_fail;
        if ((ce = cudaMemcpyAsync(hstatus, w.status, sizeof(hstatus), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
            goto cuda_fail;
        if ((ce = cudaStreamSynchronize(stream)) != cudaSuccess) goto cuda_fail;
        if (hstatus[qb::kStError]) { *err = "balanced-assignment repair found no valid augmenting path"; return MOE_ERR_INTERNAL; }
        if (hinfo[2] != 0) { *err = "max_repair moves did not remove the excess"; return MOE_ERR_NOT_CONVERGED; }
        return MOE_OK;
    }
cuda_fail:
    *err = cudaGetErrorString(ce);
    return MOE_ERR_CUDA;
}

}  // namespace moe
