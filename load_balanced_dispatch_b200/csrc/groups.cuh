// groups.cuh -- tile list of a grouped GEMM whose group sizes live on the device.
//
// Expert e owns rows [offsets[e], offsets[e+1]) of the expert-major buffer.
// Each CTA rebuilds, in shared memory, the first tile index of every expert
// (ceil(rows_e / BM) row tiles x ntn column tiles) with one warp: parallel
// loads of the offsets and a warp-wide scan. No host synchronisation needed.
#pragma once

#include "common.cuh"

namespace moe {

struct GroupTable {
    int tile_start[kMaxExperts + 1];  // first tile of expert e; tile_start[n] = total tiles
    int row_start[kMaxExperts + 1];   // first row of expert e (clamped to max_rows); row_start[n] = rows
};

// Called by one full warp.
__device__ __forceinline__ void build_group_table(const int32_t* __restrict__ offsets, int n, int ntn, int bm,
                                                  int64_t max_rows, GroupTable& g) {
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) / 32;  // <= 8
    int cnt[8], rs[8];
    int lsum = 0;
    bool clamped = false;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        cnt[q] = 0;
        rs[q] = 0;
        const int e = lane * per + q;
        if (q < per && e < n) {
            int64_t r0 = offsets[e], r1 = offsets[e + 1];
            if (r1 > max_rows) { r1 = max_rows; clamped = true; }
            if (r0 > r1) r0 = r1;
            rs[q] = (int)r0;
            cnt[q] = (int)((r1 - r0 + bm - 1) / bm) * ntn;
            lsum += cnt[q];
        }
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - lsum;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int e = lane * per + q;
        if (q < per && e < n) {
            g.tile_start[e] = run;
            g.row_start[e] = rs[q];
            run += cnt[q];
        }
    }
    if (lane == 31) {
        g.tile_start[n] = incl;
        int64_t rend = offsets[n];
        if (rend > max_rows) { rend = max_rows; clamped = true; }
        g.row_start[n] = (int)rend;
    }
    if (clamped) record_error(kErrRowOverflow);
}

// Largest e in [0, n) with tile_start[e] <= tile.
__device__ __forceinline__ int group_of_tile(const GroupTable& g, int n, int tile) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (g.tile_start[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

}  // namespace moe
