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
//   qb_row     one warp per token: v = s_i - beta in registers (n/32 values per
//              lane), k + 1 rounds of a warp arg-max give the top-k set, the
//              k-th and (k+1)-th values (alpha) and a tie flag; the set is
//              written in ascending expert order and counted per expert.
//   transpose  s [m, n] -> sT [n, m] once per call, so each column is contiguous.
//   qb_col     one CTA per expert column: exact radix select (four 8-bit
//              digit passes over order-preserving uint32 keys of u) for the
//              C-th largest, then the (C+1)-th from the tie count or one max
//              pass.
//   repair     successive shortest paths on the n-expert graph (exact finish
//              when the QB iterate is not yet balanced): arc a -> b costs
//              W[a][b] = min over tokens i holding a but not b of s_ia - s_ib
//              (fp64, lowest token on ties); one CTA runs Jacobi Bellman-Ford
//              rounds from the over-full experts, picks the nearest under-full
//              expert (lowest index on ties) and moves each arc's argmin
//              token. The number of moves equals the excess, so the host
//              enqueues exactly that many rounds without waiting in between.
#include "common.cuh"

namespace moe {

namespace qb {
constexpr int kRowThreads = 256;
constexpr int kColThreads = 512;  // qb_col_kernel block size (its scan buffer is sized by it)
// status words kept in the workspace
// kStDone: repair finished; kStQbDone: a row pass found every count equal to C (later passes return at once);
// kStIters: beta updates done; kStTies0/1: tie counts of the row passes (ping-pong with the counts buffers)
enum { kStDone = 0, kStAugments = 1, kStError = 2, kStQbDone = 4, kStIters = 5, kStTies0 = 6, kStTies1 = 7,
       kStWords = 8 };
constexpr int kBatch = 16;  // QB iterations enqueued between host checks
}  // namespace qb

__device__ __forceinline__ float qb_threshold(float a, float b, int rule) {
    return rule == MOE_QB_BOUNDARY ? b : __fmul_rn(__fadd_rn(a, b), 0.5f);
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

// Top-(k+1) of one row held by a warp (lane owns j = lane + 32 q). Each round takes the
// best untaken key: lane-local scan (lowest q on ties), then __reduce_max_sync over the
// order-preserving keys and __reduce_min_sync over the candidate indices (lowest j among
// equal keys) -- two warp instructions per round. R rows are interleaved per warp so the
// rounds of independent rows overlap.
template <int NT, int R>
__global__ void __launch_bounds__(qb::kRowThreads)
qb_row_kernel(const float* __restrict__ s, int64_t m, int n, int k, const float* __restrict__ beta, int rule,
              float* __restrict__ alpha, int32_t* __restrict__ topk_idx, int32_t* __restrict__ counts,
              int32_t* __restrict__ status, int tie_slot, int skip_if_done) {
    if (skip_if_done && *(volatile int32_t*)&status[qb::kStQbDone]) return;
    __shared__ float sb[kMaxExperts];
    __shared__ int cnt[kMaxExperts];
    __shared__ int nties;
    const int tid = threadIdx.x, lane = tid & 31;
    for (int j = tid; j < n; j += blockDim.x) { sb[j] = beta[j]; cnt[j] = 0; }
    if (tid == 0) nties = 0;
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    const int64_t warps = (int64_t)gridDim.x * (qb::kRowThreads / 32);
    for (int64_t i0 = ((int64_t)blockIdx.x * (qb::kRowThreads / 32) + (tid >> 5)) * R; i0 < m; i0 += warps * R) {
        float v[R][NT];
        uint32_t key[R][NT], taken[R];
        float vk[R], vk1[R];
#pragma unroll
        for (int u = 0; u < R; ++u) {
            const int64_t i = i0 + u;
            taken[u] = 0;
            vk[u] = vk1[u] = 0.f;
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const int j = lane + 32 * q;
                const bool ok = i < m && j < n;
                v[u][q] = ok ? __fsub_rn(s[i * n + j], sb[j]) : 0.f;
                key[u][q] = ok ? float_key(v[u][q]) : 0u;
            }
        }
        for (int r = 0; r <= k; ++r) {
#pragma unroll
            for (int u = 0; u < R; ++u) {
                uint32_t lb = 0;
                int lq = -1;
                float lv = 0.f;
#pragma unroll
                for (int q = 0; q < NT; ++q)
                    if (!((taken[u] >> q) & 1u) && key[u][q] > lb) { lb = key[u][q]; lq = q; lv = v[u][q]; }
                const uint32_t mx = __reduce_max_sync(0xffffffffu, lb);
                const uint32_t cand = (lq >= 0 && lb == mx) ? (uint32_t)(lq * 32 + lane) : 0xffffffffu;
                const uint32_t wj = __reduce_min_sync(0xffffffffu, cand);
                const float wv = __shfl_sync(0xffffffffu, lv, (int)(wj & 31u));
                if (r < k && wj < (uint32_t)n && (int)(wj & 31u) == lane) taken[u] |= 1u << (wj >> 5);
                if (r == k - 1) vk[u] = wv;
                if (r == k) vk1[u] = wv;
            }
        }
#pragma unroll
        for (int u = 0; u < R; ++u) {
            const int64_t i = i0 + u;
            if (i >= m) break;
            if (lane == 0) {
                alpha[i] = qb_threshold(vk[u], vk1[u], rule);
                if (vk[u] == vk1[u]) atomicAdd(&nties, 1);
            }
            int pos = 0;
#pragma unroll
            for (int q = 0; q < NT; ++q) {
                const bool bit = (taken[u] >> q) & 1u;
                const uint32_t mask = __ballot_sync(0xffffffffu, bit);
                if (bit) {
                    topk_idx[i * k + pos + __popc(mask & lt)] = lane + 32 * q;
                    atomicAdd(&cnt[lane + 32 * q], 1);
                }
                pos += __popc(mask);
            }
        }
    }
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x)
        if (cnt[j]) atomicAdd(&counts[j], cnt[j]);
    if (tid == 0 && nties) atomicAdd(&status[tie_slot], nties);
}

__global__ void transpose_kernel(const float* __restrict__ s, int64_t m, int n, float* __restrict__ sT) {
    __shared__ float tile[32][33];
    const int64_t i0 = (int64_t)blockIdx.x * 32;
    const int j0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int64_t i = i0 + r;
        const int j = j0 + tx;
        tile[r][tx] = (i < m && j < n) ? s[i * n + j] : 0.f;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int j = j0 + r;
        const int64_t i = i0 + tx;
        if (j < n && i < m) sT[(int64_t)j * m + i] = tile[tx][r];
    }
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

// Add 1 to hist[d] for every active lane, one atomic per distinct d in the warp.
__device__ __forceinline__ void warp_hist_add(unsigned* hist, bool active, uint32_t d) {
    const uint32_t grp = __match_any_sync(0xffffffffu, active ? d : 0xffffffffu);
    const int lane = threadIdx.x & 31;
    if (active && (grp & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[d], (unsigned)__popc(grp));
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

namespace qb {
constexpr int kCandCap = 16384;                         // candidate keys kept in shared memory
constexpr size_t kColSmem = 4096 * 4 + kColThreads * 4 + kCandCap * 4;
}  // namespace qb

// beta_j = threshold between the C-th and (C+1)-th largest key of column j of u = fp32(s - alpha).
// Pass 1 (global): histogram of the top 12 key bits. Pass 2 (global): keep the keys of the selected
// bin in shared memory and the largest key below it. Then digits 19..8 and 7..0 over the kept keys.
// If the bin holds more keys than fit, the two remaining digits stream from global memory instead.
__global__ void __launch_bounds__(qb::kColThreads)
qb_col_kernel(const float* __restrict__ sT, int64_t m, int n, int64_t C, const float* __restrict__ alpha, int rule,
              float* __restrict__ beta, const int32_t* __restrict__ counts, int32_t* __restrict__ counts_next,
              int32_t* __restrict__ status, int iter, int check) {
    if (check) {
        // stop once the previous row pass is balanced; otherwise CTA 0 prepares the next row pass
        if (*(volatile int32_t*)&status[qb::kStQbDone]) return;
        __shared__ int balanced;
        if (threadIdx.x == 0) balanced = 1;
        __syncthreads();
        for (int e = threadIdx.x; e < n; e += blockDim.x)
            if (counts[e] != C) balanced = 0;
        __syncthreads();
        if (balanced) {
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
    const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31;
    const int j = blockIdx.x;
    const float* col = sT + (int64_t)j * m;
    auto key_at = [&](int64_t i) { return float_key(__fsub_rn(col[i], alpha[i])); };

    for (int b = tid; b < 4096; b += T) hist[b] = 0;
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    for (int64_t base = 0; base < m; base += T) {
        const int64_t i = base + tid;
        const bool ok = i < m;
        const uint32_t key = ok ? key_at(i) : 0u;
        warp_hist_add(hist, ok, key >> 20);
    }
    __syncthreads();
    int sel1;
    int64_t want1;
    unsigned cnt1;
    block_select_bin(hist, 4096, C, scan, &sel1, &want1, &cnt1);

    uint32_t below = 0;
    for (int64_t base = 0; base < m; base += T) {
        const int64_t i = base + tid;
        const bool ok = i < m;
        const uint32_t key = ok ? key_at(i) : 0u;
        const uint32_t d = key >> 20;
        if (ok && d < (uint32_t)sel1 && key > below) below = key;
        const bool in = ok && d == (uint32_t)sel1;
        const uint32_t bal = __ballot_sync(0xffffffffu, in);
        unsigned wbase = 0;
        if (lane == 0 && bal) wbase = atomicAdd(&s_ncand, (unsigned)__popc(bal));
        wbase = __shfl_sync(0xffffffffu, wbase, 0);
        const unsigned pos = wbase + __popc(bal & ((1u << lane) - 1u));
        if (in && pos < (unsigned)qb::kCandCap) cand[pos] = key;
    }
    below = block_max_u32(below, scan);
    const unsigned ncand = s_ncand;
    const bool kept = ncand <= (unsigned)qb::kCandCap;

    // digits 19..8, then 7..0, within the selected top bin
    int sel2, sel3;
    int64_t want2, want3;
    unsigned cnt2, cnt3;
    for (int b = tid; b < 4096; b += T) hist[b] = 0;
    __syncthreads();
    if (kept) {
        for (unsigned base = 0; base < ncand; base += T) {
            const unsigned c = base + tid;
            const bool ok = c < ncand;
            const uint32_t key = ok ? cand[c] : 0u;
            warp_hist_add(hist, ok, (key >> 8) & 0xfffu);
        }
    } else {
        for (int64_t base = 0; base < m; base += T) {
            const int64_t i = base + tid;
            const uint32_t key = i < m ? key_at(i) : 0u;
            warp_hist_add(hist, i < m && (key >> 20) == (uint32_t)sel1, (key >> 8) & 0xfffu);
        }
    }
    __syncthreads();
    block_select_bin(hist, 4096, want1, scan, &sel2, &want2, &cnt2);
    const uint32_t pre2 = ((uint32_t)sel1 << 20) | ((uint32_t)sel2 << 8);
    for (int b = tid; b < 256; b += T) hist[b] = 0;
    __syncthreads();
    if (kept) {
        for (unsigned base = 0; base < ncand; base += T) {
            const unsigned c = base + tid;
            const uint32_t key = c < ncand ? cand[c] : 0u;
            warp_hist_add(hist, c < ncand && (key & 0xffffff00u) == pre2, key & 0xffu);
        }
    } else {
        for (int64_t base = 0; base < m; base += T) {
            const int64_t i = base + tid;
            const uint32_t key = i < m ? key_at(i) : 0u;
            warp_hist_add(hist, i < m && (key & 0xffffff00u) == pre2, key & 0xffu);
        }
    }
    __syncthreads();
    block_select_bin(hist, 256, want2, scan, &sel3, &want3, &cnt3);
    const uint32_t akey = pre2 | (uint32_t)sel3;
    const int64_t greater = C - want3;
    uint32_t bkey;
    if (greater + (int64_t)cnt3 >= C + 1) {
        bkey = akey;
    } else {
        // the (C+1)-th largest is the largest key below akey: inside the top bin, else below it
        uint32_t best = 0;
        if (kept) {
            for (unsigned c = tid; c < ncand; c += T) {
                const uint32_t key = cand[c];
                if (key < akey && key > best) best = key;
            }
        } else {
            for (int64_t i = tid; i < m; i += T) {
                const uint32_t key = key_at(i);
                if ((key >> 20) == (uint32_t)sel1 && key < akey && key > best) best = key;
            }
        }
        best = block_max_u32(best, scan);
        bkey = best ? best : below;
    }
    if (tid == 0) beta[j] = qb_threshold(key_float(akey), key_float(bkey), rule);
}

namespace qb {
constexpr int kArcThreads = 512;     // 16 warps
constexpr int kArcBatch = 4;         // members per warp step (their loads in flight together)
constexpr int kArcWords = 512;       // bitmap words compacted per pass: at most 16384 members
constexpr int kMemberCap = kArcWords * 32;
constexpr int kStepThreads = 1024;   // 4 threads per expert column in the shortest-path rounds
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
// (lowest token among equal costs). The members of a come from the bitmap (compacted into shared
// memory, kMemberCap at a time); warp w takes members in batches of kArcBatch, lanes own columns
// b = lane + 32 q; the 32 warps' minima are folded in warp order at the end.
template <int NT>
__global__ void __launch_bounds__(qb::kArcThreads, 1)
qb_arc_kernel(const float* __restrict__ s, int64_t m, int n, int k, const int32_t* __restrict__ topk_idx,
              const uint32_t* __restrict__ mem, int64_t words, const int32_t* __restrict__ rows,
              const int32_t* __restrict__ nrows, double* __restrict__ W, int32_t* __restrict__ A,
              const int32_t* __restrict__ status) {
    if (status[qb::kStError] || status[qb::kStDone]) return;
    if ((int)blockIdx.x >= *nrows) return;
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
    for (int64_t w0 = 0; w0 < words; w0 += qb::kArcWords) {
        // compact the members held in the next kArcWords bitmap words (token order is not needed:
        // ties go to the lowest token explicitly)
        if (threadIdx.x == 0) nlist = 0;
        __syncthreads();
        {
            const int64_t wi = w0 + threadIdx.x;
            const uint32_t bits = (threadIdx.x < qb::kArcWords && wi < words) ? row[wi] : 0u;
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
                uint32_t in = 0;  // bit q: column lane + 32 q belongs to the member's set
                for (int r = 0; r < k; ++r) {
                    const int e = k <= 32 ? __shfl_sync(0xffffffffu, ex[u], r & 31) : topk_idx[(int64_t)id[u] * k + r];
#pragma unroll
                    for (int q = 0; q < NT; ++q) in |= (e == lane + 32 * q) ? (1u << q) : 0u;
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
    for (int b = threadIdx.x; b < n; b += blockDim.x) {
        double bb = INFINITY;
        int32_t aa = -1;
        for (int w = 0; w < NW; ++w) {
            const double c = bw[w * kMaxExperts + b];
            const int32_t t = ba[w * kMaxExperts + b];
            if (c < bb || (c == bb && c != INFINITY && t < aa)) { bb = c; aa = t; }
        }
        W[(int64_t)a * n + b] = bb;
        A[(int64_t)a * n + b] = bb == INFINITY ? -1 : aa;
    }
}

// One augmentation (one unit of excess): Jacobi Bellman-Ford rounds from the over-full experts,
// the nearest under-full expert (lowest index on ties), the path by lowest-index predecessors, and
// the moves of each arc's token. Writes the rows of W that the moves invalidate (the old set of
// every moved token, plus the expert it moved to) for the next arc launch.
__global__ void __launch_bounds__(qb::kStepThreads)
qb_repair_step_kernel(int n, int64_t C, int k, const double* __restrict__ W, const int32_t* __restrict__ A,
                      int32_t* __restrict__ counts, int32_t* __restrict__ topk_idx, int32_t* __restrict__ status,
                      int32_t* __restrict__ rows, int32_t* __restrict__ nrows, uint32_t* __restrict__ mem,
                      int64_t words) {
    __shared__ double dist[kMaxExperts], part_d[4][kMaxExperts];
    __shared__ int part_p[4][kMaxExperts], pred[kMaxExperts];
    __shared__ int any_over;
    __shared__ uint32_t touched[kMaxExperts / 32];
    const int tid = threadIdx.x;
    const int b = tid & 255, part = tid >> 8;  // 4 threads per column b, each a quarter of the a range
    if (status[qb::kStError] || status[qb::kStDone]) return;
    if (tid == 0) any_over = 0;
    if (tid < kMaxExperts / 32) touched[tid] = 0;
    __syncthreads();
    if (part == 0 && b < n) {
        const bool over = counts[b] > C;
        dist[b] = over ? 0.0 : INFINITY;
        if (over) atomicOr(&any_over, 1);
    }
    __syncthreads();
    if (!any_over) {
        if (tid == 0) { status[qb::kStDone] = 1; *nrows = 0; }
        return;
    }
    // Jacobi rounds over the frontier: only experts whose distance changed in the previous round
    // can improve another one, so each round reads just their rows of W (same fixpoint as full rounds)
    __shared__ int front[kMaxExperts], nfront;
    __shared__ unsigned char chg[kMaxExperts];
    if (tid < kMaxExperts) chg[tid] = (tid < n && dist[tid] == 0.0) ? 1 : 0;
    __syncthreads();
    bool settled = false;
    for (int round = 0; round <= n; ++round) {
        if (tid == 0) {
            int c = 0;
            for (int a = 0; a < n; ++a)
                if (chg[a]) front[c++] = a;
            nfront = c;
        }
        __syncthreads();
        const int nf = nfront;
        if (nf == 0) { settled = true; break; }
        double bestd = INFINITY;
        if (b < n) {
            // this thread's quarter of the frontier, 8 loads in flight
            for (int f0 = part; f0 < nf; f0 += 4 * 8) {
                double w8[8];
                int a8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int fi = f0 + 4 * u;
                    a8[u] = fi < nf ? front[fi] : -1;
                    w8[u] = a8[u] >= 0 ? W[(int64_t)a8[u] * n + b] : INFINITY;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int aa = a8[u];
                    if (aa >= 0 && aa != b && w8[u] != INFINITY) {
                        const double c = dist[aa] + w8[u];
                        if (c < bestd) bestd = c;
                    }
                }
            }
        }
        part_d[part][b] = bestd;
        __syncthreads();
        if (part == 0) {
            if (b < n) {
                double nd = dist[b];
                for (int p = 0; p < 4; ++p) nd = fmin(nd, part_d[p][b]);
                chg[b] = nd != dist[b];
                part_d[0][b] = nd;
            } else {
                chg[b] = 0;
            }
        }
        __syncthreads();
        if (part == 0 && b < n) dist[b] = part_d[0][b];
        __syncthreads();
    }
    if (!settled) {  // still improving after n rounds: a negative cycle, which an optimal start excludes
        if (tid == 0) { status[qb::kStError] = 1; record_error(kErrRepair); *nrows = 0; }
        return;
    }
    // predecessor: lowest a with dist[a] + W[a][b] == dist[b] (4 threads per column, a quarter each)
    const int qa = (n + 3) / 4, a0 = part * qa, a1 = min(n, a0 + qa);
    int pa = 0x7fffffff;
    if (b < n && dist[b] != INFINITY) {
        for (int a = a0; a < a1; ++a) {
            const double w = W[(int64_t)a * n + b];
            if (a != b && dist[a] != INFINITY && w != INFINITY && dist[a] + w == dist[b]) { pa = a; break; }
        }
    }
    part_p[part][b] = pa;
    __syncthreads();
    if (part == 0 && b < n) {
        int p = 0x7fffffff;
        for (int q = 0; q < 4; ++q) p = min(p, part_p[q][b]);
        pred[b] = p == 0x7fffffff ? -1 : p;
    }
    __syncthreads();
    if (tid == 0) {
        int t = -1;
        for (int e = 0; e < n; ++e)
            if (counts[e] < C && dist[e] != INFINITY && (t < 0 || dist[e] < dist[t])) t = e;
        bool ok = t >= 0;
        int node = t, len = 0;
        int path[kMaxExperts + 1];
        if (ok) {
            path[len++] = node;
            while (pred[node] >= 0 && len <= n) { node = pred[node]; path[len++] = node; }
            ok = len <= n && counts[node] > C;
        }
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
                touched[row[r] >> 5] |= 1u << (row[r] & 31);  // the token's old set
            }
            if (pos < 0 || hasb) { ok = false; break; }
            touched[bb >> 5] |= 1u << (bb & 31);
            mem[(int64_t)a * words + (i >> 5)] &= ~(1u << (i & 31));
            mem[(int64_t)bb * words + (i >> 5)] |= 1u << (i & 31);
            int r = pos;
            row[r] = bb;
            while (r > 0 && row[r - 1] > row[r]) { const int t2 = row[r - 1]; row[r - 1] = row[r]; row[r] = t2; --r; }
            while (r + 1 < k && row[r + 1] < row[r]) { const int t2 = row[r + 1]; row[r + 1] = row[r]; row[r] = t2; ++r; }
        }
        if (!ok) {
            status[qb::kStError] = 1;
            record_error(kErrRepair);
            *nrows = 0;
        } else {
            counts[node] -= 1;
            counts[t] += 1;
            status[qb::kStAugments] += 1;
            int c = 0;
            for (int e = 0; e < n; ++e)
                if ((touched[e >> 5] >> (e & 31)) & 1u) rows[c++] = e;
            *nrows = c;
        }
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
};

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

static size_t qb_layout(int64_t m, int n, int k, QBWorkspace* w, char* base) {
    (void)k;
    size_t off = 0;
    auto take = [&](size_t bytes) { char* p = base ? base + off : nullptr; off += align256(bytes); return p; };
    char* p;
    p = take(sizeof(float) * (size_t)m * n);            if (w) w->sT = (float*)p;
    p = take(sizeof(float) * (size_t)m);                if (w) w->alpha = (float*)p;
    p = take(sizeof(int32_t) * (size_t)2 * n);          if (w) w->counts = (int32_t*)p;
    p = take(sizeof(int32_t) * qb::kStWords);           if (w) w->status = (int32_t*)p;
    p = take(sizeof(double) * (size_t)n * n);           if (w) w->W = (double*)p;
    p = take(sizeof(int32_t) * (size_t)n * n);          if (w) w->A = (int32_t*)p;
    p = take(sizeof(int32_t) * (size_t)n);              if (w) w->rows = (int32_t*)p;
    p = take(sizeof(int32_t));                          if (w) w->nrows = (int32_t*)p;
    p = take(sizeof(uint32_t) * (size_t)n * (size_t)((m + 31) / 32)); if (w) w->mem = (uint32_t*)p;
    return off;
}

size_t balance_workspace_bytes(int64_t m, int32_t n, int32_t k) { return qb_layout(m, n, k, nullptr, nullptr); }

template <int NT>
static void launch_row_t(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                         int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip,
                         cudaStream_t stream) {
    int64_t blocks = (m + 2 * (qb::kRowThreads / 32) - 1) / (2 * (qb::kRowThreads / 32));
    if (blocks > (int64_t)kNumSMs * 8) blocks = (int64_t)kNumSMs * 8;
    if (blocks < 1) blocks = 1;
    qb_row_kernel<NT, 2><<<(unsigned)blocks, qb::kRowThreads, 0, stream>>>(s, m, n, k, beta, rule, alpha, topk_idx,
                                                                           counts, status, tie_slot, skip);
}

static void launch_row(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                       int32_t* topk_idx, int32_t* counts, int32_t* status, int tie_slot, int skip,
                       cudaStream_t stream) {
    if (n <= 32) launch_row_t<1>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, stream);
    else if (n <= 64) launch_row_t<2>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, stream);
    else if (n <= 128) launch_row_t<4>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, stream);
    else launch_row_t<8>(s, m, n, k, beta, rule, alpha, topk_idx, counts, status, tie_slot, skip, stream);
}

template <int NT>
static void launch_arc_t(const float* s, int64_t m, int n, int k, const int32_t* topk_idx, const QBWorkspace& w,
                         cudaStream_t stream) {
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(qb_arc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qb::kArcSmem);
        attr = true;
    }
    qb_arc_kernel<NT><<<n, qb::kArcThreads, qb::kArcSmem, stream>>>(s, m, n, k, topk_idx, w.mem, (m + 31) / 32,
                                                                    w.rows, w.nrows, w.W, w.A, w.status);
}

static void launch_arc(const float* s, int64_t m, int n, int k, const int32_t* topk_idx, const QBWorkspace& w,
                       cudaStream_t stream) {
    if (n <= 32) launch_arc_t<1>(s, m, n, k, topk_idx, w, stream);
    else if (n <= 64) launch_arc_t<2>(s, m, n, k, topk_idx, w, stream);
    else if (n <= 128) launch_arc_t<4>(s, m, n, k, topk_idx, w, stream);
    else launch_arc_t<8>(s, m, n, k, topk_idx, w, stream);
}

// Returns a moe_status; SOLVE synchronises the stream between phases.
int run_balance_assign(const float* s, int64_t m, int n, int k, float* beta, int mode, int rule, int max_iters,
                       int max_repair, int32_t* topk_idx, int32_t* info, void* workspace, cudaStream_t stream,
                       const char** err) {
    QBWorkspace w;
    qb_layout(m, n, k, &w, static_cast<char*>(workspace));
    const int64_t C = m * k / n;
    cudaError_t ce;
    static bool col_attr = false;
    if (!col_attr) {
        if ((ce = cudaFuncSetAttribute(qb_col_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)qb::kColSmem)) != cudaSuccess)
            goto cuda_fail;
        col_attr = true;
    }
    if ((ce = cudaMemsetAsync(w.status, 0, sizeof(int32_t) * qb::kStWords, stream)) != cudaSuccess) goto cuda_fail;
    if ((ce = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * 2 * n, stream)) != cudaSuccess) goto cuda_fail;
    {
        dim3 tb(32, 8), tg((unsigned)((m + 31) / 32), (unsigned)((n + 31) / 32));
        transpose_kernel<<<tg, tb, 0, stream>>>(s, m, n, w.sT);
    }
    if (mode == MOE_QB_STEP) {
        launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, w.counts, w.status, qb::kStTies0, 0, stream);
        qb_col_kernel<<<n, qb::kColThreads, qb::kColSmem, stream>>>(w.sT, m, n, C, w.alpha, rule, beta, w.counts,
                                                                    w.counts + n, w.status, 0, 0);
        qb_info_kernel<<<1, 32, 0, stream>>>(w.counts, n, C, w.status, 1, qb::kStTies0, info);
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
                launch_row(s, m, n, k, beta, rule, w.alpha, topk_idx, cnt, w.status,
                           u % 2 ? qb::kStTies1 : qb::kStTies0, 1, stream);
                if (u < max_iters)
                    qb_col_kernel<<<n, qb::kColThreads, qb::kColSmem, stream>>>(
                        w.sT, m, n, C, w.alpha, rule, beta, cnt, w.counts + ((u + 1) % 2) * n, w.status, u, 1);
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
        // then only the rows a move invalidates are recomputed
        const int64_t moves = excess < max_repair ? excess : max_repair;
        if (moves > 0) {
            const int64_t words = (m + 31) / 32;
            if ((ce = cudaMemsetAsync(w.mem, 0, sizeof(uint32_t) * (size_t)n * (size_t)words, stream)) != cudaSuccess)
                goto cuda_fail;
            qb_member_bits_kernel<<<(unsigned)((m * k + 255) / 256), 256, 0, stream>>>(topk_idx, m, k, words, w.mem);
            qb_all_rows_kernel<<<1, 256, 0, stream>>>(n, w.rows, w.nrows);
        }
        for (int64_t a = 0; a < moves; ++a) {
            launch_arc(s, m, n, k, topk_idx, w, stream);
            qb_repair_step_kernel<<<1, qb::kStepThreads, 0, stream>>>(n, C, k, w.W, w.A, final_counts, topk_idx,
                                                                      w.status, w.rows, w.nrows, w.mem,
                                                                      (m + 31) / 32);
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
