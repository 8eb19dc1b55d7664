// Per-token INT8 activation quantization (act_quant_per_token).
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §3.1: per-token amax, scale = amax/127,
// round half to even, clamp to [-128, 127].  The division by the scale is IEEE fp32; a token whose
// amax is 0 gets scale 0 and all-zero codes.
//
// HBM-bound (2 B read + 1 B written per element): one CTA per token, 16-byte loads, a block-wide
// max, then a second pass over the (cache-resident) row that writes 8 codes per 8-byte store.
#include "q4_common.cuh"

namespace {

__global__ void __launch_bounds__(256) act_quant_kernel(const uint16_t* __restrict__ x, int k,
                                                        int8_t* __restrict__ xq, float* __restrict__ scale_a,
                                                        int32_t* status)
{
    __shared__ float red[8];
    const int64_t row = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * k);
    const int n8 = k / 8;
    float amax = 0.0f;
    bool finite = true;
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
        const uint4 v = __ldg(xr + i);
        const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float a = __uint_as_float(e[j] << 16), b = __uint_as_float(e[j] & 0xFFFF0000u);
            finite &= isfinite(a) && isfinite(b);
            amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
        }
    }
    if (!finite) q4_set_status(status, Q4_ERR_NONFINITE);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax;
    __syncthreads();
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; i++) m = fmaxf(m, red[i]);
    const float s = m / 127.0f;
    if (threadIdx.x == 0) scale_a[row] = s;
    uint2* out = reinterpret_cast<uint2*>(xq + row * k);
    for (int i = threadIdx.x; i < n8; i += blockDim.x) {
        const uint4 v = __ldg(xr + i);
        const uint32_t e[4] = {v.x, v.y, v.z, v.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float a = __uint_as_float(e[j] << 16), b = __uint_as_float(e[j] & 0xFFFF0000u);
            const int qa = s == 0.0f ? 0 : (int)fminf(fmaxf(rintf(a / s), -128.0f), 127.0f);
            const int qb = s == 0.0f ? 0 : (int)fminf(fmaxf(rintf(b / s), -128.0f), 127.0f);
            packed[j / 2] |= ((uint32_t)(qa & 0xFF) | ((uint32_t)(qb & 0xFF) << 8)) << (16 * (j & 1));
        }
        out[i] = make_uint2(packed[0], packed[1]);
    }
}

}  // namespace

extern "C" int act_quant_per_token(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                                   int32_t* dev_status, void* stream)
{
    if (!x || !xq || !scale_a) return Q4_ERR_NULL;
    if (m < 0 || k <= 0 || k % 8) return Q4_ERR_SHAPE;
    if (!q4_aligned16(x) || !q4_aligned16(xq) || ((uintptr_t)scale_a & 3u)) return Q4_ERR_ALIGN;
    if (m == 0) return Q4_OK;
    act_quant_kernel<<<m, 256, 0, (cudaStream_t)stream>>>(x, k, xq, scale_a, dev_status);
    return q4_launch_status();
}
