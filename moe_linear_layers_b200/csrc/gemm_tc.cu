// tcgen05 tensor-core GEMM for W4A16 and W4A8 (in progress).
#include "q4_common.cuh"

int q4_gemm_tc_launch(const void*, const float*, int32_t, const q4_weight*, void*, int32_t, int32_t*, bool,
                      int32_t*, cudaStream_t)
{
    return Q4_ERR_UNSUPPORTED;
}
