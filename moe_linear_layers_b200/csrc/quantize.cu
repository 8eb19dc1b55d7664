// RTN group quantization + nibble packing (q4_quantize_pack).
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.3 (offline INT4 quantization keeping
// scale and zero point) and §2.1 (4-bit storage); "从FP32到INT4：大语言模型量化压缩实战指南" §1.3
// (each group computes its own range; a zero point only for the asymmetric form).
//
// HBM-bound: 4 B read per element, 0.5 B (+ 2-4 B per group) written.  Each thread owns 8
// consecutive elements (two 16-byte loads, one 4-byte packed store); a group of G elements is G/8
// consecutive lanes of one warp, reduced with xor shuffles inside that lane segment.
#include "q4_common.cuh"

namespace {

template <int G, bool SYM>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const float* __restrict__ w, int64_t total8,
                                                            uint32_t* __restrict__ packed,
                                                            __half* __restrict__ scales,
                                                            __half* __restrict__ zeros, int32_t* status)
{
    constexpr int TPG = G / 8;  // lanes per group; 32 % TPG == 0 so groups never straddle warps
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32) * 32; base < total8;
         base += warps_total * 32) {
        const int64_t t = base + lane;
        const bool valid = t < total8;  // total8 is a multiple of TPG: invalid lanes are whole groups
        float v[8];
        if (valid) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(w) + 2 * t);
            const float4 b = __ldg(reinterpret_cast<const float4*>(w) + 2 * t + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) v[i] = 0.0f;
        }
        bool finite = true;
#pragma unroll
        for (int i = 0; i < 8; i++) finite &= isfinite(v[i]);

        int codes[8];
        float S;
        __half s16, z16 = __float2half_rn(0.0f);
        if constexpr (SYM) {
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int off = TPG / 2; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            s16 = __float2half_rn(amax / 7.0f);
            S = __half2float(s16);
#pragma unroll
            for (int i = 0; i < 8; i++)
                codes[i] = S == 0.0f ? 0 : (int)fminf(fmaxf(rintf(v[i] / S), -8.0f), 7.0f);
        } else {
            float mn = 0.0f, mx = 0.0f;  // the range always includes 0
#pragma unroll
            for (int i = 0; i < 8; i++) { mn = fminf(mn, v[i]); mx = fmaxf(mx, v[i]); }
#pragma unroll
            for (int off = TPG / 2; off >= 1; off >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            }
            s16 = __float2half_rn((mx - mn) / 15.0f);
            S = __half2float(s16);
            if (S == 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; i++) codes[i] = 0;
            } else {
                const float z = fminf(fmaxf(rintf(-mn / S), 0.0f), 15.0f);
                z16 = __float2half_rn(z);
#pragma unroll
                for (int i = 0; i < 8; i++) codes[i] = (int)fminf(fmaxf(rintf(v[i] / S) + z, 0.0f), 15.0f);
            }
        }
        if (!valid) continue;
        if (!finite || !isfinite(S)) q4_set_status(status, Q4_ERR_NONFINITE);
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; i++) word |= (uint32_t)(codes[i] & 0xF) << (4 * i);
        packed[t] = word;
        if ((lane % TPG) == 0) {
            scales[t / TPG] = s16;
            if constexpr (!SYM) zeros[t / TPG] = z16;
        }
    }
}

}  // namespace

extern "C" int q4_quantize_pack(const float* w, int32_t n, int32_t k, int32_t group, int32_t symmetric,
                                uint8_t* packed, uint16_t* scales, uint16_t* zeros, int32_t* dev_status,
                                void* stream)
{
    if (n < 0 || k <= 0 || (group != 32 && group != 64 && group != 128 && group != 256) || k % group) return Q4_ERR_SHAPE;
    if (n == 0) return Q4_OK;   // no rows: the four arrays hold nothing and may be NULL
    if (!w || !packed || !scales || (!symmetric && !zeros)) return Q4_ERR_NULL;
    if (!q4_aligned16(w) || !q4_aligned16(packed) || !q4_aligned16(scales) || (!symmetric && !q4_aligned16(zeros)))
        return Q4_ERR_ALIGN;
    const int64_t total8 = (int64_t)n * k / 8;
    const int64_t warps = (total8 + 31) / 32;
    const int64_t blocks = std::min<int64_t>((warps + 7) / 8, (int64_t)q4_num_sms() * 16);
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* pk = reinterpret_cast<uint32_t*>(packed);
    __half* sc = reinterpret_cast<__half*>(scales);
    __half* zr = reinterpret_cast<__half*>(zeros);
    if (group == 256) {
        if (symmetric) quantize_pack_kernel<256, true><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
        else quantize_pack_kernel<256, false><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
    } else if (group == 128) {
        if (symmetric) quantize_pack_kernel<128, true><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
        else quantize_pack_kernel<128, false><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
    } else if (group == 64) {
        if (symmetric) quantize_pack_kernel<64, true><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
        else quantize_pack_kernel<64, false><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
    } else {
        if (symmetric) quantize_pack_kernel<32, true><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
        else quantize_pack_kernel<32, false><<<(int)blocks, 256, 0, s>>>(w, total8, pk, sc, zr, dev_status);
    }
    return q4_launch_status();
}
