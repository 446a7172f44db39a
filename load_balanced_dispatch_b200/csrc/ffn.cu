// ffn.cu -- expert FFN entry: selects the kernel for the dtype.
#include "common.cuh"

namespace moe {

cudaError_t launch_ffn_simt(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2,
                            const void* b2, const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows,
                            void* ybuf, void* hbuf, cudaStream_t stream);

cudaError_t launch_ffn_tc(const void* xbuf, const void* w1, const void* b1, const void* w2, const void* b2,
                          const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                          cudaStream_t stream);

// bf16: tcgen05 tensor-core grouped GEMMs; fp32: fp32 FMA grouped GEMMs.
cudaError_t launch_ffn(const void* xbuf, moe_dtype dt, const void* w1, const void* b1, const void* w2, const void* b2,
                       const int32_t* offsets, int n, int d, int d_ff, int64_t max_rows, void* ybuf, void* hbuf,
                       cudaStream_t stream) {
    if (dt == MOE_BF16) return launch_ffn_tc(xbuf, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, stream);
    return launch_ffn_simt(xbuf, dt, w1, b1, w2, b2, offsets, n, d, d_ff, max_rows, ybuf, hbuf, stream);
}

}  // namespace moe
