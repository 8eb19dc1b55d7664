// Device helpers shared by the W4A16 GEMV kernels (gemv.cu: one launch per problem group; gemv_chain.cu:
// a chain of dependent stages in one launch): bulk copies into shared memory, the integer dot product of
// packed INT4 codes with int16 activations, and the per-block power-of-two scaling of x.
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored before the
// multiply) and §1 (small batch: memory bound).
#pragma once

#include "q4_common.cuh"
#include "tc_ptx.cuh"

namespace gemv {

// Codes -> bytes: (u & mask) ^ key keeps the low (or high) nibble of every byte of a packed word; for
// symmetric codes the key flips bit 3 of each nibble (two's complement -> offset binary: code + 8).
template <bool SYM> struct Keys;
template <> struct Keys<true> {
    static constexpr uint32_t lo = 0x08080808u, hi = 0x80808080u, zero = 8;
};
template <> struct Keys<false> {
    static constexpr uint32_t lo = 0u, hi = 0u, zero = 0;
};


// Bring a byte range into L2 (coherent: it cannot observe stale data).  Needs 16-byte alignment.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_l2_range(const void* lo_, const void* hi_)
{
    const uintptr_t a = ((uintptr_t)lo_ + 15) & ~(uintptr_t)15, b = (uintptr_t)hi_ & ~(uintptr_t)15;
    for (uintptr_t q = a; q < b; q += 65536) prefetch_l2((const void*)q, (uint32_t)min((uintptr_t)65536, b - q));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)) : "memory");
}


__device__ __forceinline__ uint4 lds128(const void* p)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(tc::smem_u32(p)));
    return v;
}

__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The 8 codes of one 32-bit word against the int16 x of that word, exactly, in int32: the low nibbles
// (codes 0, 2, 4, 6) as bytes into acc1, the high nibbles in place (16 * code) into acc16.
// X = {(x0,x2), (x4,x6), (x1,x3), (x5,x7)} as int16 pairs.
template <bool SYM>
__device__ __forceinline__ void word_dot(uint32_t u, const uint4& X, int& acc1, int& acc16)
{
    const uint32_t lo = lop3_and_xor(u, 0x0F0F0F0Fu, Keys<SYM>::lo);
    const uint32_t hi = lop3_and_xor(u, 0xF0F0F0F0u, Keys<SYM>::hi);
    acc1 = dp2a_lo(X.x, lo, acc1);
    acc1 = dp2a_hi(X.y, lo, acc1);
    acc16 = dp2a_lo(X.z, hi, acc16);
    acc16 = dp2a_hi(X.w, hi, acc16);
}

// Power-of-two scale 2^e of a 64-value block with max|x| * 2^e in [2^14, 2^15) (bf16 bits of the max
// magnitude in, e clamped so that 2^e and 2^-e are normal floats), and its inverse.
__device__ __forceinline__ float2 block_scale(uint32_t amax_bits)
{
    const int ex = (int)((amax_bits >> 7) & 0xFFu);
    if (amax_bits == 0 || ex == 0xFF) return make_float2(1.0f, 1.0f);
    const int e = min(126, max(-126, 141 - ex));
    return make_float2(__uint_as_float((uint32_t)(127 + e) << 23), __uint_as_float((uint32_t)(127 - e) << 23));
}

// x of one word (8 bf16 values) -> int16 rne(x * scale), in the pair order word_dot consumes.  Adding
// 1.5 * 2^23 rounds to an integer that sits in the low mantissa bits.
__device__ __forceinline__ uint4 x_ints(const uint4& v, float scale)
{
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    constexpr float kMagic = 12582912.0f;
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        b[2 * i] = __float_as_uint(fmaf(__uint_as_float(e[i] << 16), scale, kMagic));
        b[2 * i + 1] = __float_as_uint(fmaf(__uint_as_float(e[i] & 0xFFFF0000u), scale, kMagic));
    }
    uint4 o;
    o.x = prmt(b[0], b[2], 0x5410u);
    o.y = prmt(b[4], b[6], 0x5410u);
    o.z = prmt(b[1], b[3], 0x5410u);
    o.w = prmt(b[5], b[7], 0x5410u);
    return o;
}

// Fused SwiGLU input (the dense FFN's down projection): x = silu(g) * u = g / (1 + e^-g) * u in fp32,
// staged like bf16 x but from fp32 values, with the block scale one binade lower (max * 2^e in
// [2^13, 2^14)) so that rounding an fp32 value can never reach 2^15.
__device__ __forceinline__ uint4 x_ints_f32(const float (&h)[8], float scale)
{
    constexpr float kMagic = 12582912.0f;
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; i++) b[i] = __float_as_uint(fmaf(h[i], scale, kMagic));
    uint4 o;
    o.x = prmt(b[0], b[2], 0x5410u);
    o.y = prmt(b[4], b[6], 0x5410u);
    o.z = prmt(b[1], b[3], 0x5410u);
    o.w = prmt(b[5], b[7], 0x5410u);
    return o;
}

__device__ __forceinline__ float2 block_scale_f32(uint32_t amax_bits)
{
    const int ex = (int)((amax_bits >> 23) & 0xFFu);
    if (amax_bits == 0 || ex == 0xFF) return make_float2(1.0f, 1.0f);
    const int e = min(126, max(-126, 140 - ex));
    return make_float2(__uint_as_float((uint32_t)(127 + e) << 23), __uint_as_float((uint32_t)(127 - e) << 23));
}

// Per-halfword max of the bf16 magnitudes of a word (integer order = magnitude order for non-NaN),
// and a flag for an all-ones exponent (inf or NaN) in any of its 8 values.
__device__ __forceinline__ uint32_t bf16_mag_max(const uint4& v, uint32_t& bad)
{
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    uint32_t a = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        a = __vmaxu2(a, e[i] & 0x7FFF7FFFu);
        bad |= ((e[i] & 0x7F807F80u) + 0x00800080u) & 0x80008000u;   // carry into bit 15 iff exponent all ones
    }
    return a;
}

// Dot product of one weight row (in the stage) with the lane's 64 x values, per activation row:
// sum_k (c_k - z) xi_k = sum_k c_k xi_k - z * sum_k xi_k, exact in int32, then one conversion and the
// group scale times the block's inverse x scale.
template <bool SYM, int MT>
__device__ __forceinline__ void row_dot(const uint8_t* wrow, const __half* srow, const __half* zrow, int gl,
                                        const uint4 (&X)[MT][8], const float (&inv_xs)[MT], const int (&xsum)[MT],
                                        float (&part)[MT])
{
    const float sc = __half2float(srow[gl]);
    int z = Keys<SYM>::zero;
    if constexpr (!SYM) z = (int)(__half_as_ushort(__hadd(zrow[gl], __float2half_rn(1024.0f))) & 0x3FFu);
    const uint4 w0 = lds128(wrow), w1 = lds128(wrow + 16);
#pragma unroll
    for (int mm = 0; mm < MT; mm++) {
        int a1 = 0, a16 = 0, c1 = 0, c16 = 0;
        word_dot<SYM>(w0.x, X[mm][0], a1, a16);
        word_dot<SYM>(w0.y, X[mm][1], c1, c16);
        word_dot<SYM>(w0.z, X[mm][2], a1, a16);
        word_dot<SYM>(w0.w, X[mm][3], c1, c16);
        word_dot<SYM>(w1.x, X[mm][4], a1, a16);
        word_dot<SYM>(w1.y, X[mm][5], c1, c16);
        word_dot<SYM>(w1.z, X[mm][6], a1, a16);
        word_dot<SYM>(w1.w, X[mm][7], c1, c16);
        const int t = (a1 + c1) + ((a16 + c16) >> 4) - z * xsum[mm];   // a16, c16: multiples of 16
        part[mm] = (float)t * (sc * inv_xs[mm]);
    }
}

// y[o] of a buffer of n values (the debug build checks o against n)
__device__ __forceinline__ void store_y(void* y, int64_t o, float v, int out_bf16, int64_t n, int32_t* status)
{
    if (!q4_in_bounds(o, n, status)) return;
    if (out_bf16) reinterpret_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(y)[o] = v;
}

}  // namespace gemv
