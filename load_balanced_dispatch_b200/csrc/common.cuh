// common.cuh -- helpers shared by the kernels of the MoE-layer library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kNumSMs = 148;

// Device error word (one per device): kernels record the first condition they
// detect and skip the offending access; moe_sync_status() reads and clears it.
enum : int {
    kErrNone = 0,
    kErrExpertIndex = 1,   // expert id outside [0, n)
    kErrRowOverflow = 2,   // more kept rows than the caller's buffer holds
    kErrTokenIndex = 3,    // src_token outside [0, m)
    kErrPipelineTimeout = 4,  // a bounded pipeline wait gave up
    kErrRepair = 5,        // balanced-assignment repair found no valid path
    kErrTotals = 6,        // a routed-count total is not a non-negative integer
};
__device__ int g_error = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_error, 0, code); }

// ---- warp helpers ---------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// (key, index) ordering: larger key first, equal keys -> lower index first.
__device__ __forceinline__ bool ranks_before(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}
// Warp-wide best (key, index); every lane receives the winner.
__device__ __forceinline__ void warp_best(float& key, int& idx) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ok = __shfl_xor_sync(0xffffffffu, key, o);
        int oi = __shfl_xor_sync(0xffffffffu, idx, o);
        if (ranks_before(ok, oi, key, idx)) { key = ok; idx = oi; }
    }
}

// ---- element loads / stores -----------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// 16-byte vector of T: 4 fp32 or 8 bf16, unpacked to fp32.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void load(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* out) {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* in) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

__device__ __forceinline__ float round_to_bf16(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// Programmatic dependent launch. A kernel started with launch_pdl may begin while its predecessor
// in the stream is still running: it calls pdl_wait() before it reads or writes any global memory
// (pdl_wait returns once the predecessor grid has completed and its writes are visible), and
// pdl_trigger() to let its own successor start early the same way. For a kernel launched without
// the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
