// capacity_static.cu -- capacity slots without caller-provided scratch.
//
// moe_capacity_slots needs a small device workspace (per-chunk expert
// histograms and prefixes). Some callers cannot hand one over: code bound
// through a fixed foreign-function signature that carries only the inputs and
// outputs, or a host framework that owns all device memory and forbids its
// plugins to call cudaMalloc (which may also synchronise the device, something
// latency-critical serving loops avoid). For them, moe_capacity_slots_static
// runs the same kernels on scratch that lives in a fixed-size array compiled
// into this library, so the call allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its 1 MiB until the process exits. Host code may not pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so the
// first call on each device looks up the array's device address with
// cudaGetSymbolAddress while that device is current, checks the result, and
// caches it per device for later calls.
#include <mutex>

#include "common.cuh"

namespace moe {

size_t capacity_workspace_bytes(int64_t m, int32_t k, int32_t n, int64_t seg_len);

constexpr size_t kStaticCapacityScratchBytes = size_t(1) << 20;  // 1 MiB
constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) int32_t g_capacity_scratch[kStaticCapacityScratchBytes / sizeof(int32_t)];

// Device address of g_capacity_scratch on the current device (set up once per device).
static cudaError_t static_capacity_scratch(void** out) {
    static std::mutex mu;
    static void* addr[kMaxStaticDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxStaticDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_capacity_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace moe

extern "C" moe_status moe_capacity_slots_static(const int32_t* topk_idx, int64_t m, int32_t k, int32_t n,
                                                int32_t capacity, int64_t seg_len, int32_t* slot, int32_t* dest_row,
                                                int32_t* src_token, int32_t* expert_offsets, int32_t* routed_count,
                                                int32_t* kept_count, moe_stream_t stream) {
    // Invalid arguments are rejected first, so they never reach the one-time address lookup below.
    const moe_status st = capacity_args_ok(topk_idx, m, k, n, capacity, seg_len, slot, dest_row, src_token,
                                           expert_offsets, routed_count, kept_count);
    if (st != MOE_OK) return st;
    const size_t need = moe::capacity_workspace_bytes(m, k, n, seg_len);
    if (need > moe::kStaticCapacityScratchBytes)
        return fail(MOE_ERR_WORKSPACE,
                    "moe_capacity_slots_static: this problem needs %zu bytes of scratch, more than the fixed "
                    "%zu-byte array; call moe_capacity_slots with a workspace instead",
                    need, moe::kStaticCapacityScratchBytes);
    // The scratch address is per device: the stream must belong to the current device.
    int cur = 0, sdev = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e == cudaSuccess) e = cudaStreamGetDevice(stream, &sdev);
    if (e != cudaSuccess)
        return fail(MOE_ERR_CUDA, "moe_capacity_slots_static: device of the stream: %s", cudaGetErrorString(e));
    if (sdev != cur)
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_capacity_slots_static: the stream belongs to device %d but device %d is current", sdev, cur);
    void* scratch = nullptr;
    e = moe::static_capacity_scratch(&scratch);
    if (e != cudaSuccess)
        return fail(MOE_ERR_CUDA, "moe_capacity_slots_static: device address of the scratch array: %s",
                    cudaGetErrorString(e));
    // Same kernels as moe_capacity_slots; the scratch is fully written before it is read.
    return moe_capacity_slots(topk_idx, m, k, n, capacity, seg_len, slot, dest_row, src_token, expert_offsets,
                              routed_count, kept_count, scratch, moe::kStaticCapacityScratchBytes, stream);
}
