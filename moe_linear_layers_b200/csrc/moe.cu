// Top-k routed MoE layer with INT4 SwiGLU experts (in progress).
#include "q4_common.cuh"

extern "C" size_t moe_q4_workspace_size(int32_t, int32_t, int32_t, int32_t, int32_t) { return 0; }

extern "C" int moe_q4_forward(const uint16_t*, int32_t, int32_t, const float*, const float*, int32_t, int32_t,
                              const q4_weight*, int32_t, void*, int32_t, int32_t*, float*, int32_t*, int32_t*,
                              int32_t*, void*, size_t, int32_t*, void*)
{
    return Q4_ERR_UNSUPPORTED;
}
