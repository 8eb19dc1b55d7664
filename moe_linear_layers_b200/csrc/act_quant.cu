// Per-token INT8 activation quantization (act_quant_per_token).
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §3.1: per-token amax, scale = amax/127,
// round half to even, clamp to [-128, 127].  The division by the scale is IEEE fp32; a token whose
// amax is 0 gets scale 0 and all-zero codes.  Inputs are bf16 (the layer inputs) or fp16 (the MoE's
// intermediate activations h); both widen to fp32 exactly.
//
// HBM-bound (2 B read + 1 B written per element): one warp per token for rows up to 1024 values, one
// CTA per token beyond; the row held in registers between the max pass and the coding pass (one read
// of x), 16-byte loads and 8-byte stores.  The quotient
// x / s is formed without a division per element: with r = RN(1/s), t = RN(x*r), e = x - s*t exact by
// FMA, q = RN(t + e*r) is the correctly rounded quotient RN(x/s) (Markstein's theorem for round to
// nearest; every residual that can decide a rounding stays a normal float when s >= 2^-100), so the codes
// equal those of an IEEE division bit for bit.  Rows with a smaller scale take the division itself.
#include "q4_common.cuh"

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int code8(float x, float s, float r, bool exact_div)
{
    float q;
    if (exact_div) {
        q = x / s;
    } else {
        const float t = x * r;
        const float e = fmaf(-s, t, x);
        q = fmaf(e, r, t);
    }
    return (int)fminf(fmaxf(rintf(q), -128.0f), 127.0f);
}

// low / high 16-bit value of a word as fp32
template <bool F16> __device__ __forceinline__ float lo16(uint32_t w)
{
    if constexpr (F16) return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
    return __uint_as_float(w << 16);
}
template <bool F16> __device__ __forceinline__ float hi16(uint32_t w)
{
    if constexpr (F16) return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    return __uint_as_float(w & 0xFFFF0000u);
}

// codes of one 16-byte word (8 values) as 8 bytes
template <bool F16>
__device__ __forceinline__ uint2 code_word(const uint4& v, float s, float r, bool exact_div)
{
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const int qa = code8(lo16<F16>(e[j]), s, r, exact_div);
        const int qb = code8(hi16<F16>(e[j]), s, r, exact_div);
        packed[j / 2] |= ((uint32_t)(qa & 0xFF) | ((uint32_t)(qb & 0xFF) << 8)) << (16 * (j & 1));
    }
    return make_uint2(packed[0], packed[1]);
}

// per-halfword max of bf16 / fp16 magnitudes (for both formats the integer order of the magnitude bits
// is the order of the values, NaN aside) and a flag for an all-ones exponent (inf or NaN) in the word
template <bool F16>
__device__ __forceinline__ uint32_t word_amax(const uint4& v, uint32_t& bad)
{
    constexpr uint32_t expo = F16 ? 0x7C007C00u : 0x7F807F80u;     // exponent field of both halves
    constexpr uint32_t one = F16 ? 0x04000400u : 0x00800080u;      // its lowest bit
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    uint32_t a = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        a = __vmaxu2(a, e[j] & 0x7FFF7FFFu);
        bad |= ((e[j] & expo) + one) & 0x80008000u;
    }
    return a;
}

// The kernels are launched as programmatic dependents (launch_pdl): a kernel lets the next one on the
// stream launch at once, and reads x and writes its outputs only after the previous kernel's completion.
__device__ __forceinline__ void pdl_start()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <typename... P, typename... A>
int launch_pdl(void (*kern)(P...), int grid, int block, cudaStream_t s, A... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return q4_cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

// W = 16-byte words per thread kept in registers (k <= 8 * kThreads * W); W = 0: any k, two passes.
template <int W, bool F16>
__global__ void __launch_bounds__(kThreads) act_quant_kernel(const uint16_t* __restrict__ x, int k,
                                                             int8_t* __restrict__ xq, float* __restrict__ scale_a,
                                                             int32_t* status)
{
    __shared__ uint32_t red[kThreads / 32];
    pdl_start();
    const int64_t row = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * k);
    uint2* out = reinterpret_cast<uint2*>(xq + row * k);
    const int n8 = k / 8;
    uint32_t a = 0, bad = 0;
    uint4 v[W > 0 ? W : 1];
    if constexpr (W > 0) {
#pragma unroll
        for (int i = 0; i < W; i++) {
            const int w = i * kThreads + threadIdx.x;
            v[i] = w < n8 ? __ldg(xr + w) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < W; i++) a = __vmaxu2(a, word_amax<F16>(v[i], bad));
    } else {
        for (int w = threadIdx.x; w < n8; w += kThreads) a = __vmaxu2(a, word_amax<F16>(__ldg(xr + w), bad));
    }
    if (bad) q4_set_status(status, Q4_ERR_NONFINITE);
    a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = a;
    __syncthreads();
    uint32_t mb = 0;
#pragma unroll
    for (int i = 0; i < kThreads / 32; i++) mb = max(mb, red[i]);
    const float m = F16 ? __half2float(__ushort_as_half((unsigned short)mb)) : __uint_as_float(mb << 16);
    const float s = m / 127.0f;
    if (threadIdx.x == 0) scale_a[row] = s;
    const bool exact_div = !(s >= 0x1p-100f);           // tiny (or zero / NaN) scale: divide directly
    const float r = exact_div ? 0.0f : 1.0f / s;
    if constexpr (W > 0) {
#pragma unroll
        for (int i = 0; i < W; i++) {
            const int w = i * kThreads + threadIdx.x;
            if (w < n8) out[w] = s == 0.0f ? make_uint2(0u, 0u) : code_word<F16>(v[i], s, r, exact_div);
        }
    } else {
        for (int w = threadIdx.x; w < n8; w += kThreads)
            out[w] = s == 0.0f ? make_uint2(0u, 0u) : code_word<F16>(__ldg(xr + w), s, r, exact_div);
    }
}

// Rows of at most 8 * 32 * W values: one warp per row (8 rows per CTA), the row in registers, the amax
// reduced with shuffles only -- short rows (the MoE's h rows of 1024 values) would leave most of a
// 256-thread CTA idle and pay a block barrier per row.  (Rows of 2048 measured faster with a CTA each:
// 10.7 against 12.3 us for 4096 rows.)
template <int W, bool F16>
__global__ void __launch_bounds__(256) act_quant_warp_kernel(const uint16_t* __restrict__ x, int m, int k,
                                                             int8_t* __restrict__ xq, float* __restrict__ scale_a,
                                                             int32_t* status)
{
    pdl_start();
    const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= m) return;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * k);
    uint2* out = reinterpret_cast<uint2*>(xq + row * k);
    const int n8 = k / 8;
    uint32_t a = 0, bad = 0;
    uint4 v[W];
#pragma unroll
    for (int i = 0; i < W; i++) {
        const int w = i * 32 + lane;
        v[i] = w < n8 ? __ldg(xr + w) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < W; i++) a = __vmaxu2(a, word_amax<F16>(v[i], bad));
    if (bad) q4_set_status(status, Q4_ERR_NONFINITE);
    a = max(a & 0xFFFFu, a >> 16);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = max(a, __shfl_xor_sync(0xffffffffu, a, off));
    const float mx = F16 ? __half2float(__ushort_as_half((unsigned short)a)) : __uint_as_float(a << 16);
    const float s = mx / 127.0f;
    if (lane == 0) scale_a[row] = s;
    const bool exact_div = !(s >= 0x1p-100f);
    const float r = exact_div ? 0.0f : 1.0f / s;
#pragma unroll
    for (int i = 0; i < W; i++) {
        const int w = i * 32 + lane;
        if (w < n8) out[w] = s == 0.0f ? make_uint2(0u, 0u) : code_word<F16>(v[i], s, r, exact_div);
    }
}

template <bool F16>
int act_quant_launch(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a, int32_t* dev_status,
                     cudaStream_t s)
{
    if (m < 0 || k <= 0 || k % 8) return Q4_ERR_SHAPE;
    if (m == 0) return Q4_OK;                 // no rows: x, xq, scale_a may be NULL
    if (!x || !xq || !scale_a) return Q4_ERR_NULL;
    if (!q4_aligned16(x) || !q4_aligned16(xq) || ((uintptr_t)scale_a & 3u)) return Q4_ERR_ALIGN;
    const int n8 = k / 8;
    const int wgrid = (m + 7) / 8;
    if (n8 <= 32 * 2) return launch_pdl(act_quant_warp_kernel<2, F16>, wgrid, 256, s, x, m, k, xq, scale_a, dev_status);
    if (n8 <= 32 * 4) return launch_pdl(act_quant_warp_kernel<4, F16>, wgrid, 256, s, x, m, k, xq, scale_a, dev_status);
    if (n8 <= kThreads) return launch_pdl(act_quant_kernel<1, F16>, m, kThreads, s, x, k, xq, scale_a, dev_status);
    if (n8 <= 2 * kThreads) return launch_pdl(act_quant_kernel<2, F16>, m, kThreads, s, x, k, xq, scale_a, dev_status);
    if (n8 <= 4 * kThreads) return launch_pdl(act_quant_kernel<4, F16>, m, kThreads, s, x, k, xq, scale_a, dev_status);
    if (n8 <= 8 * kThreads) return launch_pdl(act_quant_kernel<8, F16>, m, kThreads, s, x, k, xq, scale_a, dev_status);
    return launch_pdl(act_quant_kernel<0, F16>, m, kThreads, s, x, k, xq, scale_a, dev_status);
}

}  // namespace

int q4_act_quant_rows(const uint16_t* x, bool f16, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                      int32_t* dev_status, cudaStream_t s)
{
    return f16 ? act_quant_launch<true>(x, m, k, xq, scale_a, dev_status, s)
               : act_quant_launch<false>(x, m, k, xq, scale_a, dev_status, s);
}

extern "C" int act_quant_per_token(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                                   int32_t* dev_status, void* stream)
{
    return act_quant_launch<false>(x, m, k, xq, scale_a, dev_status, (cudaStream_t)stream);
}

extern "C" int act_quant_per_token_f16(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                                       int32_t* dev_status, void* stream)
{
    return act_quant_launch<true>(x, m, k, xq, scale_a, dev_status, (cudaStream_t)stream);
}
