// W4A16 GEMV for small m (decode): y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[m][k].
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a
// 16-bit type before the multiply) and §1 (small model, small batch: memory bound).
//
// Design (HBM-bound; the packed weights are streamed once):
//  * a warp walks weight rows; lane l owns 16-byte chunks (32 codes) at fixed k positions, so its
//    slice of x stays in registers (m == 1) or is read from shared memory (m > 1) for every row;
//  * loads are 128-bit ld.global.nc, coalesced (a warp reads 512 contiguous bytes of a row), with
//    the next row block prefetched while the current one is computed;
//  * dequant in registers: one LOP3 turns two nibbles into an fp16x2 "1024 + code" (the exponent
//    of 1024 makes the code the low mantissa bits); an HSUB2 of (1024 + zero) leaves the exact
//    integer (code - zero) in fp16; nibbles 1, 3, 5, 7 of a word are used in place (16 * code) and
//    accumulate separately, scaled by 1/16 once per chunk;
//  * products accumulate in fp16x2 over one chunk (8 per half) and then in fp32, scaled by the
//    group scale once per chunk; x is pre-scaled by a power of two so |x| < 2 (exact), which keeps
//    every fp16 partial far from overflow;
//  * rows that need more than 64 chunks (k > 2048) are split over a team of 2..8 warps, reduced
//    through shared memory.
#include "q4_common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct GemvParams {
    const uint16_t* x;
    const uint8_t* packed;
    const __half* scales;
    const __half* zeros;
    void* y;
    int32_t* status;
    int m, n, k, group, out_bf16;
};

// Nibble -> fp16x2 magic: (u & mask) ^ key, key = 0x6400 (1024.0) in both halves, plus the sign
// flip 8 of symmetric codes (two's complement -> offset binary: c + 8 = nibble ^ 8).
template <bool SYM> struct Keys;
template <> struct Keys<true> {
    static constexpr uint32_t k1 = 0x64006400u ^ 0x00080008u, k16 = 0x64006400u ^ 0x00800080u;
};
template <> struct Keys<false> {
    static constexpr uint32_t k1 = 0x64006400u, k16 = 0x64006400u;
};

// Power-of-two prescale p with max|x| * p in [1, 2): exact, and every fp16 partial stays small.
__device__ __forceinline__ float prescale_for(float amax)
{
    if (!(amax > 0.0f) || !isfinite(amax)) return 1.0f;
    int e;
    frexpf(amax, &e);  // amax = f * 2^e, f in [0.5, 1)
    return ldexpf(1.0f, 1 - e);
}

// Block-wide max of |x| over one token row; also flags non-finite values.
__device__ float block_amax(const uint16_t* xr, int k, int32_t* status, float* red)
{
    float a = 0.0f;
    bool finite = true;
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
        float v = bf16_bits_to_float(xr[i]);
        finite &= isfinite(v);
        a = fmaxf(a, fabsf(v));
    }
    if (!finite) q4_set_status(status, Q4_ERR_NONFINITE);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = a;
    __syncthreads();
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < kWarps; i++) r = fmaxf(r, red[i]);
    return r;
}

// One chunk (32 codes) against the x pairs of that chunk; returns the fp32 dot product of
// (code - zero) and the pre-scaled x (not yet multiplied by the group scale).
template <bool SYM>
__device__ __forceinline__ float chunk_dot(const uint4& wv, __half2 bias1, __half2 bias16, const __half2 (&X)[16])
{
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
    __half2 acc1 = __float2half2_rn(0.0f), acc16 = __float2half2_rn(0.0f);
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint32_t u = words[w], u8 = u >> 8;
        const __half2 d0 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x000F000Fu, Keys<SYM>::k1)), bias1);
        const __half2 d1 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x00F000F0u, Keys<SYM>::k16)), bias16);
        const __half2 d2 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x000F000Fu, Keys<SYM>::k1)), bias1);
        const __half2 d3 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x00F000F0u, Keys<SYM>::k16)), bias16);
        acc1 = __hfma2(d0, X[4 * w + 0], acc1);
        acc16 = __hfma2(d1, X[4 * w + 1], acc16);
        acc1 = __hfma2(d2, X[4 * w + 2], acc1);
        acc16 = __hfma2(d3, X[4 * w + 3], acc16);
    }
    const float2 f1 = __half22float2(acc1), f16 = __half22float2(acc16);
    return (f1.x + f1.y) + 0.0625f * (f16.x + f16.y);
}

// x pairs of one chunk in the order chunk_dot consumes them: for word w,
// X[4w+0] = (x[8w], x[8w+4]), X[4w+1] = (x[8w+1], x[8w+5]), X[4w+2] = (x[8w+2], x[8w+6]),
// X[4w+3] = (x[8w+3], x[8w+7]); each value times the power-of-two prescale p.
__device__ __forceinline__ void load_x_chunk(const uint16_t* xc, float p, __half2 (&X)[16])
{
    const uint4* v = reinterpret_cast<const uint4*>(xc);
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint4 q = __ldg(v + w);
        const uint32_t e[4] = {q.x, q.y, q.z, q.w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            f[2 * i] = __uint_as_float(e[i] << 16) * p;
            f[2 * i + 1] = __uint_as_float(e[i] & 0xFFFF0000u) * p;
        }
#pragma unroll
        for (int j = 0; j < 4; j++) X[4 * w + j] = __floats2half2_rn(f[j], f[j + 4]);
    }
}

// Programmatic dependent launch: let the next kernel on the stream start launching, and wait for the
// previous one (its writes become visible) only before reading data it may produce.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bring a contiguous byte range into L2 (a hint: it neither reads into registers nor can it observe
// stale data, L2 being the device's point of coherence).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

template <int KSPLIT, int J, int ROWS, bool SYM>
__global__ void __launch_bounds__(kThreads, 2) w4a16_gemv_m1_kernel(GemvParams p)
{
    constexpr int TEAMS = kWarps / KSPLIT;
    __shared__ float red[kWarps * ROWS];
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int team = warp / KSPLIT, wit = warp % KSPLIT;
    const int C = p.k / 32, ng = p.k / p.group, cpg = p.group / 32;
    const int64_t rowbytes = p.k / 2;
    const int rows_per_cta = TEAMS * ROWS;
    const int64_t stride = (int64_t)gridDim.x * rows_per_cta;

    pdl_launch_dependents();
    // The weights do not depend on the previous kernel: start pulling this CTA's rows into L2 now.
    if (threadIdx.x == 0) {
        for (int64_t rb = (int64_t)blockIdx.x * rows_per_cta; rb < p.n; rb += stride) {
            const int64_t rows = min((int64_t)rows_per_cta, (int64_t)p.n - rb);
            prefetch_l2(p.packed + rb * rowbytes, (uint32_t)(rows * rowbytes));
        }
    }
    pdl_wait();

    int cidx[J];
    bool cval[J];
    uint4 xraw[J][4];
    float amax = 0.0f;
    bool finite = true;
#pragma unroll
    for (int j = 0; j < J; j++) {
        cidx[j] = wit * 32 * J + 32 * j + lane;
        cval[j] = cidx[j] < C;
#pragma unroll
        for (int w = 0; w < 4; w++) {
            xraw[j][w] = cval[j] ? __ldg(reinterpret_cast<const uint4*>(p.x + 32 * cidx[j]) + w) : make_uint4(0, 0, 0, 0);
            const uint32_t e[4] = {xraw[j][w].x, xraw[j][w].y, xraw[j][w].z, xraw[j][w].w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float a = __uint_as_float(e[i] << 16), b = __uint_as_float(e[i] & 0xFFFF0000u);
                finite &= isfinite(a) && isfinite(b);
                amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
            }
        }
    }
    if (!finite) q4_set_status(p.status, Q4_ERR_NONFINITE);
    // every team covers the whole row of x, so the block max over all warps is max|x|
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kWarps; i++) amax = fmaxf(amax, red[i]);
    __syncthreads();
    const float ps = prescale_for(amax);
    const float inv_ps = 1.0f / ps;

    __half2 X[J][16];
#pragma unroll
    for (int j = 0; j < J; j++) {
#pragma unroll
        for (int w = 0; w < 4; w++) {
            const uint32_t e[4] = {xraw[j][w].x, xraw[j][w].y, xraw[j][w].z, xraw[j][w].w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                f[2 * i] = __uint_as_float(e[i] << 16) * ps;
                f[2 * i + 1] = __uint_as_float(e[i] & 0xFFFF0000u) * ps;
            }
#pragma unroll
            for (int q = 0; q < 4; q++) X[j][4 * w + q] = __floats2half2_rn(f[q], f[q + 4]);
        }
    }

    // Row block in flight: the next block is fetched into (nw, ns, nz) while (cw, cs, cz) is used.
    uint4 cw[ROWS][J], nw[ROWS][J];
    __half cs[ROWS][J], ns[ROWS][J], cz[ROWS][J], nz[ROWS][J];
    auto fetch = [&](uint4 (&wv)[ROWS][J], __half (&sc)[ROWS][J], __half (&zc)[ROWS][J], int64_t rb) {
#pragma unroll
        for (int rr = 0; rr < ROWS; rr++) {
            const int64_t r = rb + team * ROWS + rr;
#pragma unroll
            for (int j = 0; j < J; j++) {
                if (r < p.n && cval[j]) {
                    wv[rr][j] = ldg_nc_v4(p.packed + r * rowbytes + (int64_t)cidx[j] * 16);
                    const int64_t gi = r * ng + cidx[j] / cpg;
                    sc[rr][j] = p.scales[gi];
                    zc[rr][j] = SYM ? __float2half_rn(8.0f) : p.zeros[gi];
                } else {
                    wv[rr][j] = make_uint4(0, 0, 0, 0);
                    sc[rr][j] = __float2half_rn(0.0f);
                    zc[rr][j] = __float2half_rn(0.0f);
                }
            }
        }
    };

    int64_t rb = (int64_t)blockIdx.x * rows_per_cta;
    if (rb < p.n) fetch(cw, cs, cz, rb);
    for (; rb < p.n; rb += stride) {
        if (rb + stride < p.n) fetch(nw, ns, nz, rb + stride);
        float part[ROWS];
#pragma unroll
        for (int rr = 0; rr < ROWS; rr++) {
            part[rr] = 0.0f;
#pragma unroll
            for (int j = 0; j < J; j++) {
                __half2 b1, b16;
                if constexpr (SYM) {
                    b1 = __float2half2_rn(1032.0f);
                    b16 = __float2half2_rn(1152.0f);
                } else {
                    const __half z = cz[rr][j];
                    b1 = __half2half2(__hadd(z, __float2half_rn(1024.0f)));
                    b16 = __half2half2(__hfma(z, __float2half_rn(16.0f), __float2half_rn(1024.0f)));
                }
                part[rr] += __half2float(cs[rr][j]) * chunk_dot<SYM>(cw[rr][j], b1, b16, X[j]);
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) part[rr] += __shfl_xor_sync(0xffffffffu, part[rr], off);
        }
        if constexpr (KSPLIT == 1) {
            if (lane < ROWS) {
                float v = part[0];
#pragma unroll
                for (int rr = 1; rr < ROWS; rr++) if (lane == rr) v = part[rr];
                const int64_t r = rb + team * ROWS + lane;
                if (r < p.n) {
                    v *= inv_ps;
                    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[r] = __float2bfloat16_rn(v);
                    else reinterpret_cast<float*>(p.y)[r] = v;
                }
            }
        } else {
            if (lane == 0) {
#pragma unroll
                for (int rr = 0; rr < ROWS; rr++) red[warp * ROWS + rr] = part[rr];
            }
            __syncthreads();
            if (wit == 0 && lane < ROWS) {
                float v = 0.0f;
#pragma unroll
                for (int t = 0; t < KSPLIT; t++) v += red[(team * KSPLIT + t) * ROWS + lane];
                const int64_t r = rb + team * ROWS + lane;
                if (r < p.n) {
                    v *= inv_ps;
                    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[r] = __float2bfloat16_rn(v);
                    else reinterpret_cast<float*>(p.y)[r] = v;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int rr = 0; rr < ROWS; rr++)
#pragma unroll
            for (int j = 0; j < J; j++) { cw[rr][j] = nw[rr][j]; cs[rr][j] = ns[rr][j]; cz[rr][j] = nz[rr][j]; }
    }
}

// m in 2..4: the dequantized pairs of a chunk are reused for every token; x pairs come from shared
// memory laid out [m][word][chunk] (16 bytes each) so that a warp's reads are conflict-free.
template <int KSPLIT, int J, int MT, bool SYM>
__global__ void __launch_bounds__(kThreads, 1) w4a16_gemv_small_m_kernel(GemvParams p)
{
    constexpr int TEAMS = kWarps / KSPLIT;
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ float red[kWarps * MT];
    __shared__ float pscale[MT];
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int team = warp / KSPLIT, wit = warp % KSPLIT;
    const int C = p.k / 32, ng = p.k / p.group, cpg = p.group / 32;
    const int64_t rowbytes = p.k / 2;
    uint4* xs = reinterpret_cast<uint4*>(smem);  // [MT][4][C] of 4 half2

    for (int mm = 0; mm < MT; mm++) {
        const float amax = block_amax(p.x + (int64_t)mm * p.k, p.k, p.status, red);
        if (threadIdx.x == 0) pscale[mm] = prescale_for(amax);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < MT * C; idx += blockDim.x) {
        const int mm = idx / C, c = idx % C;
        __half2 X[16];
        load_x_chunk(p.x + (int64_t)mm * p.k + 32 * c, pscale[mm], X);
#pragma unroll
        for (int w = 0; w < 4; w++) {
            uint4 v;
            v.x = h2_as_u32(X[4 * w]); v.y = h2_as_u32(X[4 * w + 1]);
            v.z = h2_as_u32(X[4 * w + 2]); v.w = h2_as_u32(X[4 * w + 3]);
            xs[((int64_t)mm * 4 + w) * C + c] = v;
        }
    }
    __syncthreads();

    for (int64_t rb = (int64_t)blockIdx.x * TEAMS; rb < p.n; rb += (int64_t)gridDim.x * TEAMS) {
        const int64_t r = rb + team;
        float part[MT];
#pragma unroll
        for (int mm = 0; mm < MT; mm++) part[mm] = 0.0f;
        uint4 wv[J];
        __half scv[J], zcv[J];
#pragma unroll
        for (int j = 0; j < J; j++) {
            const int c = wit * 32 * J + 32 * j + lane;
            if (r < p.n && c < C) {
                wv[j] = ldg_nc_v4(p.packed + r * rowbytes + (int64_t)c * 16);
                scv[j] = p.scales[r * ng + c / cpg];
                zcv[j] = SYM ? __float2half_rn(8.0f) : p.zeros[r * ng + c / cpg];
            } else {
                wv[j] = make_uint4(0, 0, 0, 0);
                scv[j] = __float2half_rn(0.0f);
                zcv[j] = __float2half_rn(0.0f);
            }
        }
#pragma unroll
        for (int j = 0; j < J; j++) {
            const int c = wit * 32 * J + 32 * j + lane;
            if (c >= C) continue;
            const __half2 b1 = __half2half2(__hadd(zcv[j], __float2half_rn(1024.0f)));
            const __half2 b16 = __half2half2(__hfma(zcv[j], __float2half_rn(16.0f), __float2half_rn(1024.0f)));
            const uint32_t words[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
            __half2 acc1[MT], acc16[MT];
#pragma unroll
            for (int mm = 0; mm < MT; mm++) { acc1[mm] = __float2half2_rn(0.0f); acc16[mm] = acc1[mm]; }
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const uint32_t u = words[w], u8 = u >> 8;
                const __half2 d0 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x000F000Fu, Keys<SYM>::k1)), b1);
                const __half2 d1 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x00F000F0u, Keys<SYM>::k16)), b16);
                const __half2 d2 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x000F000Fu, Keys<SYM>::k1)), b1);
                const __half2 d3 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x00F000F0u, Keys<SYM>::k16)), b16);
#pragma unroll
                for (int mm = 0; mm < MT; mm++) {
                    const uint4 xv = xs[((int64_t)mm * 4 + w) * C + c];
                    acc1[mm] = __hfma2(d0, u32_as_h2(xv.x), acc1[mm]);
                    acc16[mm] = __hfma2(d1, u32_as_h2(xv.y), acc16[mm]);
                    acc1[mm] = __hfma2(d2, u32_as_h2(xv.z), acc1[mm]);
                    acc16[mm] = __hfma2(d3, u32_as_h2(xv.w), acc16[mm]);
                }
            }
            const float s = __half2float(scv[j]);
#pragma unroll
            for (int mm = 0; mm < MT; mm++) {
                const float2 f1 = __half22float2(acc1[mm]), f16 = __half22float2(acc16[mm]);
                part[mm] += s * ((f1.x + f1.y) + 0.0625f * (f16.x + f16.y));
            }
        }
#pragma unroll
        for (int mm = 0; mm < MT; mm++)
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) part[mm] += __shfl_xor_sync(0xffffffffu, part[mm], off);
        if (lane == 0) {
#pragma unroll
            for (int mm = 0; mm < MT; mm++) red[warp * MT + mm] = part[mm];
        }
        __syncthreads();
        if (wit == 0 && lane < MT && r < p.n) {
            float v = 0.0f;
            for (int t = 0; t < KSPLIT; t++) v += red[(team * KSPLIT + t) * MT + lane];
            v /= pscale[lane];
            const int64_t o = (int64_t)lane * p.n + r;
            if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
            else reinterpret_cast<float*>(p.y)[o] = v;
        }
        __syncthreads();
    }
}

// Launched with programmatic stream serialization: the kernel may begin (and prefetch weights into
// L2) while the previous kernel on the stream drains; it reads x only after griddepcontrol.wait.
template <int KSPLIT, int J, int ROWS>
int launch_m1(const GemvParams& p, int symmetric, int grid, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = symmetric ? cudaLaunchKernelEx(&cfg, w4a16_gemv_m1_kernel<KSPLIT, J, ROWS, true>, p)
                              : cudaLaunchKernelEx(&cfg, w4a16_gemv_m1_kernel<KSPLIT, J, ROWS, false>, p);
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

template <int KSPLIT, int J>
int launch_m1_rows(const GemvParams& p, int symmetric, cudaStream_t s)
{
    constexpr int TEAMS = kWarps / KSPLIT;
    const int64_t target = (int64_t)q4_num_sms() * 2;  // two resident CTAs per SM
    auto ctas = [&](int rows) { return ((int64_t)p.n + TEAMS * rows - 1) / (TEAMS * rows); };
    // four rows in flight only with one chunk per lane (two chunks x four rows exceed 128 registers)
    if constexpr (J == 1)
        if (ctas(4) >= target) return launch_m1<KSPLIT, J, 4>(p, symmetric, (int)std::min<int64_t>(ctas(4), target), s);
    if (ctas(2) >= target) return launch_m1<KSPLIT, J, 2>(p, symmetric, (int)std::min<int64_t>(ctas(2), target), s);
    return launch_m1<KSPLIT, J, 1>(p, symmetric, (int)std::min<int64_t>(ctas(1), target), s);
}

template <int KSPLIT, int J, int MT>
int launch_small(const GemvParams& p, int symmetric, cudaStream_t s)
{
    constexpr int TEAMS = kWarps / KSPLIT;
    const size_t smem = (size_t)MT * p.k * 2;
    const int grid = (int)std::min<int64_t>(((int64_t)p.n + TEAMS - 1) / TEAMS, (int64_t)q4_num_sms());
    auto kern = symmetric ? w4a16_gemv_small_m_kernel<KSPLIT, J, MT, true> : w4a16_gemv_small_m_kernel<KSPLIT, J, MT, false>;
    if (smem > 200 * 1024) return Q4_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return Q4_ERR_CUDA;
    kern<<<grid, kThreads, smem, s>>>(p);
    return q4_launch_status();
}

template <int KSPLIT, int J>
int launch_small_m(const GemvParams& p, int symmetric, cudaStream_t s)
{
    switch (p.m) {
        case 2: return launch_small<KSPLIT, J, 2>(p, symmetric, s);
        case 3: return launch_small<KSPLIT, J, 3>(p, symmetric, s);
        default: return launch_small<KSPLIT, J, 4>(p, symmetric, s);
    }
}

template <int J>
int dispatch_ksplit(const GemvParams& p, int symmetric, int ksplit, cudaStream_t s)
{
    if (p.m == 1) {
        switch (ksplit) {
            case 1: return launch_m1_rows<1, J>(p, symmetric, s);
            case 2: return launch_m1_rows<2, J>(p, symmetric, s);
            case 4: return launch_m1_rows<4, J>(p, symmetric, s);
            default: return launch_m1_rows<8, J>(p, symmetric, s);
        }
    }
    switch (ksplit) {
        case 1: return launch_small_m<1, J>(p, symmetric, s);
        case 2: return launch_small_m<2, J>(p, symmetric, s);
        case 4: return launch_small_m<4, J>(p, symmetric, s);
        default: return launch_small_m<8, J>(p, symmetric, s);
    }
}

}  // namespace

// Host entry used by q4_linear_w4a16 for m <= 4.  Requires k % 32 == 0 and k <= 16384.
int q4_gemv_w4a16_launch(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                         int32_t* dev_status, cudaStream_t stream)
{
    if (w->k % 32 || w->k > 16384 || m < 1 || m > 4) return Q4_ERR_UNSUPPORTED;
    GemvParams p;
    p.x = x;
    p.packed = w->packed;
    p.scales = reinterpret_cast<const __half*>(w->scales);
    p.zeros = reinterpret_cast<const __half*>(w->zeros);
    p.y = y;
    p.status = dev_status;
    p.m = m;
    p.n = w->n;
    p.k = w->k;
    p.group = w->group;
    p.out_bf16 = out_dtype == Q4_OUT_BF16;
    const int C = w->k / 32;
    const int J = C >= 64 ? 2 : 1;
    int ksplit = 1;
    while (ksplit * 32 * J < C) ksplit *= 2;
    if (ksplit > 8) return Q4_ERR_UNSUPPORTED;
    return J == 2 ? dispatch_ksplit<2>(p, w->symmetric, ksplit, stream)
                  : dispatch_ksplit<1>(p, w->symmetric, ksplit, stream);
}
