// bl_gemm_tc.cu -- prefill tensor-core path (tcgen05 kind::i8); see below.
#include "bl_internal.cuh"

namespace bl {

bool gemm_tc_supported(int64_t, int64_t, int64_t) { return false; }

cudaError_t launch_gemm_tc(const int8_t*, const float*, const uint8_t*, const float*, int64_t, int64_t,
                           int64_t, void*, bl_dtype, int32_t*, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace bl
