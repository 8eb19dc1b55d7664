// W4A16 GEMV for small m (decode): y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[m][k].
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a
// 16-bit type before the multiply) and §1 (small model, small batch: memory bound).
//
// HBM-bound design (the packed weights are streamed exactly once):
//  * persistent CTAs, one per SM, each owning a contiguous block of weight rows;
//  * a producer thread streams the block through a 5-stage shared-memory ring with cp.async.bulk
//    (16 KB per stage: whole rows are contiguous in memory), completion tracked by mbarriers, so
//    ~80 KB per SM are in flight without any register-held loads;
//  * programmatic dependent launch: the CTA pulls its rows into L2 (a coherent prefetch) before it
//    waits for the previous kernel on the stream, so consecutive GEMVs keep HBM busy across the
//    kernel boundary; x (which the previous kernel may produce) is read only after the wait;
//  * x is converted once per CTA into fp16 pairs (power-of-two prescale so max|x| < 2, exact) and
//    held in registers by the lanes that use it;
//  * in-register dequant: one LOP3 turns two nibbles into fp16x2 "1024 + code"; an HSUB2 of
//    (1024 + zero) leaves the exact integer (code - zero); nibbles 1, 3, 5, 7 of a word are used in
//    place (16 * code) and accumulate separately (scaled by 1/16 once per chunk); products accumulate
//    in fp16x2 over one 32-code chunk (8 products per half) and then in fp32 times the group scale;
//  * lanes split a row into 16-byte chunks (coalesced, bank-conflict-free shared reads); rows longer
//    than 2048 codes are split over 2..8 warps and combined through shared memory.
#include "q4_common.cuh"
#include "tc_ptx.cuh"

namespace {

constexpr int kComputeWarps = 16;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;      // + one producer warp
constexpr int kStageBytes = 16384;
constexpr int kStages = 5;
constexpr int kScaleBytes = 16384;                  // the CTA's scales (+ zeros) in shared memory
constexpr int kMaxM = 4;

struct GemvParams {
    const uint16_t* x;
    const uint8_t* packed;
    const __half* scales;
    const __half* zeros;
    void* y;
    int32_t* status;
    int m, n, k, group, out_bf16;
    int rows_per_cta;    // contiguous weight rows per CTA
    int rows_per_stage;  // rows per 16 KB stage
};

// Nibble -> fp16x2 magic: (u & mask) ^ key, key = 0x6400 (1024.0) in both halves, plus the flip of
// bit 3 of symmetric codes (two's complement -> offset binary: code + 8 = nibble ^ 8).
template <bool SYM> struct Keys;
template <> struct Keys<true> {
    static constexpr uint32_t k1 = 0x64006400u ^ 0x00080008u, k16 = 0x64006400u ^ 0x00800080u;
};
template <> struct Keys<false> {
    static constexpr uint32_t k1 = 0x64006400u, k16 = 0x64006400u;
};

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bring a byte range into L2 (coherent: it cannot observe stale data).  Needs 16-byte alignment.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_l2_range(const uint8_t* lo, const uint8_t* hi)
{
    const uintptr_t a = ((uintptr_t)lo + 15) & ~(uintptr_t)15, b = (uintptr_t)hi & ~(uintptr_t)15;
    for (uintptr_t q = a; q < b; q += 65536) prefetch_l2((const void*)q, (uint32_t)min((uintptr_t)65536, b - q));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory"); }

__device__ __forceinline__ uint4 lds128(const void* p)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(tc::smem_u32(p)));
    return v;
}

// Power-of-two prescale p with max|x| * p in [1, 2): exact, and every fp16 partial stays small.
__device__ __forceinline__ float prescale_for(float amax)
{
    if (!(amax > 0.0f) || !isfinite(amax)) return 1.0f;
    int e;
    frexpf(amax, &e);  // amax = f * 2^e, f in [0.5, 1)
    return ldexpf(1.0f, 1 - e);
}

// The 8 codes of one 32-bit word against the x pairs of that word.
// X = {(x0,x4), (x1,x5), (x2,x6), (x3,x7)} as half2 bit patterns.
template <bool SYM>
__device__ __forceinline__ void word_dot(uint32_t u, __half2 b1, __half2 b16, const uint4& X, __half2& acc1,
                                         __half2& acc16)
{
    const uint32_t u8 = u >> 8;
    const __half2 d0 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x000F000Fu, Keys<SYM>::k1)), b1);
    const __half2 d1 = __hsub2(u32_as_h2(lop3_and_xor(u, 0x00F000F0u, Keys<SYM>::k16)), b16);
    const __half2 d2 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x000F000Fu, Keys<SYM>::k1)), b1);
    const __half2 d3 = __hsub2(u32_as_h2(lop3_and_xor(u8, 0x00F000F0u, Keys<SYM>::k16)), b16);
    acc1 = __hfma2(d0, u32_as_h2(X.x), acc1);
    acc16 = __hfma2(d1, u32_as_h2(X.y), acc16);
    acc1 = __hfma2(d2, u32_as_h2(X.z), acc1);
    acc16 = __hfma2(d3, u32_as_h2(X.w), acc16);
}

__device__ __forceinline__ float fold(__half2 acc1, __half2 acc16)
{
    const float2 f = __half22float2(__hfma2(acc16, __float2half2_rn(0.0625f), acc1));
    return f.x + f.y;
}

template <int KSPLIT, int J, int MT, bool SYM>
__global__ void __launch_bounds__(kThreads, 1) w4a16_gemv_kernel(GemvParams p)
{
    constexpr int TEAMS = kComputeWarps / KSPLIT;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* stages = smem;                                                   // kStages x kStageBytes
    uint4* xs = reinterpret_cast<uint4*>(smem + kStages * kStageBytes);       // [MT][4][C] x pairs
    const int C = p.k / 32, ng = p.k / p.group, cpg = p.group / 32;
    __half* ssc = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(xs) + (size_t)MT * p.k * 2);
    __half* szr = ssc + p.rows_per_cta * ng;
    float* red = reinterpret_cast<float*>(smem + kStages * kStageBytes + (size_t)MT * p.k * 2 + kScaleBytes);
    float* pscale = red + 2 * 16 * kMaxM;
    uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * 16 * kMaxM + 8 * kMaxM);
    uint64_t* empty = full + kStages;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int64_t rowbytes = p.k / 2;
    const int r0 = blockIdx.x * p.rows_per_cta;
    const int r1 = min(p.n, r0 + p.rows_per_cta);
    const int nstages = (r1 - r0 + p.rows_per_stage - 1) / p.rows_per_stage;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], kComputeWarps); }
        tc::fence_mbar_init();
    }
    if (warp == kComputeWarps && lane == 0 && r0 < r1) {
        // weights do not depend on the previous kernel: start pulling them into L2 now
        prefetch_l2_range(p.packed + (int64_t)r0 * rowbytes, p.packed + (int64_t)r1 * rowbytes);
        prefetch_l2_range(reinterpret_cast<const uint8_t*>(p.scales + (int64_t)r0 * ng),
                          reinterpret_cast<const uint8_t*>(p.scales + (int64_t)r1 * ng));
        if constexpr (!SYM)
            prefetch_l2_range(reinterpret_cast<const uint8_t*>(p.zeros + (int64_t)r0 * ng),
                              reinterpret_cast<const uint8_t*>(p.zeros + (int64_t)r1 * ng));
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            for (int st = 0; st < nstages; st++) {
                const int s = st % kStages;
                if (!tc::mbar_wait(&empty[s], ((st / kStages) & 1) ^ 1, p.status, nullptr)) break;
                const int rs = r0 + st * p.rows_per_stage;
                const uint32_t bytes = (uint32_t)(min(p.rows_per_stage, r1 - rs) * rowbytes);
                tc::mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s(stages + s * kStageBytes, p.packed + (int64_t)rs * rowbytes, bytes, &full[s]);
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- compute warps
    // x -> fp16 pairs with a power-of-two prescale per token; the CTA's scales and zeros -> smem
    for (int mm = 0; mm < MT; mm++) {
        const uint4* xr = reinterpret_cast<const uint4*>(p.x + (int64_t)mm * p.k);
        float amax = 0.0f;
        bool finite = true;
        for (int u = threadIdx.x; u < p.k / 8; u += kComputeThreads) {
            const uint4 v = __ldg(xr + u);
            const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float a = __uint_as_float(e[i] << 16), b = __uint_as_float(e[i] & 0xFFFF0000u);
                finite &= isfinite(a) && isfinite(b);
                amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
            }
        }
        if (!finite) q4_set_status(p.status, Q4_ERR_NONFINITE);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) red[warp] = amax;
        compute_bar();
        if (threadIdx.x == 0) {
            float a = 0.0f;
            for (int i = 0; i < kComputeWarps; i++) a = fmaxf(a, red[i]);
            pscale[mm] = prescale_for(a);
        }
        compute_bar();
        const float ps = pscale[mm];
        for (int u = threadIdx.x; u < p.k / 8; u += kComputeThreads) {
            const uint4 v = __ldg(xr + u);
            const uint32_t e[4] = {v.x, v.y, v.z, v.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                f[2 * i] = __uint_as_float(e[i] << 16) * ps;
                f[2 * i + 1] = __uint_as_float(e[i] & 0xFFFF0000u) * ps;
            }
            uint4 o;
            o.x = h2_as_u32(__floats2half2_rn(f[0], f[4]));
            o.y = h2_as_u32(__floats2half2_rn(f[1], f[5]));
            o.z = h2_as_u32(__floats2half2_rn(f[2], f[6]));
            o.w = h2_as_u32(__floats2half2_rn(f[3], f[7]));
            xs[((int64_t)mm * 4 + (u & 3)) * C + (u >> 2)] = o;   // word u&3 of chunk u>>2
        }
    }
    for (int i = threadIdx.x; i < (r1 - r0) * ng; i += kComputeThreads) {
        ssc[i] = p.scales[(int64_t)r0 * ng + i];
        if constexpr (!SYM) szr[i] = p.zeros[(int64_t)r0 * ng + i];
    }
    compute_bar();

    const int team = warp / KSPLIT, ks = warp % KSPLIT;
    int cidx[J];
    uint4 X[J][4];
#pragma unroll
    for (int j = 0; j < J; j++) {
        cidx[j] = ks * 32 * J + 32 * j + lane;
#pragma unroll
        for (int w = 0; w < 4; w++)
            X[j][w] = (MT == 1 && cidx[j] < C) ? xs[(int64_t)w * C + cidx[j]] : make_uint4(0, 0, 0, 0);
    }

    for (int st = 0; st < nstages; st++) {
        const int s = st % kStages;
        const int rs = r0 + st * p.rows_per_stage;
        const int rows_here = min(p.rows_per_stage, r1 - rs);
        if (!tc::mbar_wait(&full[s], (st / kStages) & 1, p.status, nullptr)) break;
        const uint8_t* sbase = stages + s * kStageBytes;
        float* redb = red + (st & 1) * 16 * kMaxM;
        for (int rr = team; rr < rows_here; rr += TEAMS) {
            const int row = rs + rr;
            const int lrow = row - r0;
            float part[MT];
#pragma unroll
            for (int mm = 0; mm < MT; mm++) part[mm] = 0.0f;
#pragma unroll
            for (int j = 0; j < J; j++) {
                const int c = cidx[j];
                if (c < C) {
                    const uint4 wv = lds128(sbase + rr * rowbytes + c * 16);
                    const int gidx = lrow * ng + c / cpg;
                    const float sc = __half2float(ssc[gidx]);
                    __half2 b1, b16;
                    if constexpr (SYM) {
                        b1 = __float2half2_rn(1032.0f);
                        b16 = __float2half2_rn(1152.0f);
                    } else {
                        const __half z = szr[gidx];
                        b1 = __half2half2(__hadd(z, __float2half_rn(1024.0f)));
                        b16 = __half2half2(__hfma(z, __float2half_rn(16.0f), __float2half_rn(1024.0f)));
                    }
                    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                    for (int mm = 0; mm < MT; mm++) {
                        __half2 acc1 = __float2half2_rn(0.0f), acc16 = __float2half2_rn(0.0f);
#pragma unroll
                        for (int w = 0; w < 4; w++) {
                            const uint4 xv = MT == 1 ? X[j][w] : xs[((int64_t)mm * 4 + w) * C + c];
                            word_dot<SYM>(words[w], b1, b16, xv, acc1, acc16);
                        }
                        part[mm] += sc * fold(acc1, acc16);
                    }
                }
            }
#pragma unroll
            for (int mm = 0; mm < MT; mm++) {
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) part[mm] += __shfl_xor_sync(0xffffffffu, part[mm], off);
            }
            if constexpr (KSPLIT == 1) {
                if (lane < MT) {
                    float v = part[0];
#pragma unroll
                    for (int mm = 1; mm < MT; mm++) if (lane == mm) v = part[mm];
                    v /= pscale[lane];
                    const int64_t o = (int64_t)lane * p.n + row;
                    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
                    else reinterpret_cast<float*>(p.y)[o] = v;
                }
            } else {
                // rows_per_stage == TEAMS here: one row per team per stage
                if (lane < MT) {
                    float v = part[0];
#pragma unroll
                    for (int mm = 1; mm < MT; mm++) if (lane == mm) v = part[mm];
                    redb[(team * KSPLIT + ks) * MT + lane] = v;
                }
            }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[s]);
        if constexpr (KSPLIT > 1) {
            compute_bar();
            if (ks == 0 && team < rows_here && lane < MT) {
                float v = 0.0f;
#pragma unroll
                for (int t = 0; t < KSPLIT; t++) v += redb[(team * KSPLIT + t) * MT + lane];
                v /= pscale[lane];
                const int64_t o = (int64_t)lane * p.n + (rs + team);
                if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
                else reinterpret_cast<float*>(p.y)[o] = v;
            }
        }
    }
}

template <int KSPLIT, int J, int MT>
int launch(const GemvParams& p, int symmetric, int grid, cudaStream_t s)
{
    const size_t smem = (size_t)kStages * kStageBytes + (size_t)MT * p.k * 2 + kScaleBytes +
                        (2 * 16 * kMaxM + 8 * kMaxM) * sizeof(float) + 2 * kStages * sizeof(uint64_t);
    if (smem > 227 * 1024) return Q4_ERR_UNSUPPORTED;
    auto kern = symmetric ? w4a16_gemv_kernel<KSPLIT, J, MT, true> : w4a16_gemv_kernel<KSPLIT, J, MT, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return Q4_ERR_CUDA;
    // Programmatic stream serialization: the kernel may start (and prefetch its weights into L2) while
    // the previous kernel on the stream drains; it reads x only after griddepcontrol.wait.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p) == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

template <int KSPLIT, int J>
int launch_m(const GemvParams& p, int symmetric, int grid, cudaStream_t s)
{
    switch (p.m) {
        case 1: return launch<KSPLIT, J, 1>(p, symmetric, grid, s);
        case 2: return launch<KSPLIT, J, 2>(p, symmetric, grid, s);
        case 3: return launch<KSPLIT, J, 3>(p, symmetric, grid, s);
        default: return launch<KSPLIT, J, 4>(p, symmetric, grid, s);
    }
}

template <int J>
int launch_ksplit(const GemvParams& p, int symmetric, int ksplit, int grid, cudaStream_t s)
{
    switch (ksplit) {
        case 1: return launch_m<1, J>(p, symmetric, grid, s);
        case 2: return launch_m<2, J>(p, symmetric, grid, s);
        case 4: return launch_m<4, J>(p, symmetric, grid, s);
        default: return launch_m<8, J>(p, symmetric, grid, s);
    }
}

}  // namespace

// Host entry used by q4_linear_w4a16 for m <= 4.  Requires k % 32 == 0 and k <= 16384.
int q4_gemv_w4a16_launch(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                         int32_t* dev_status, cudaStream_t stream)
{
    if (w->k % 32 || w->k > 16384 || m < 1 || m > kMaxM) return Q4_ERR_UNSUPPORTED;
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
    int ksplit = 1;
    while (ksplit * 64 < C) ksplit *= 2;                     // at most two chunks per lane
    if (ksplit > 8) return Q4_ERR_UNSUPPORTED;
    const int J = (C + 32 * ksplit - 1) / (32 * ksplit);
    const int teams = kComputeWarps / ksplit;
    const int rowbytes = w->k / 2;
    int rps = kStageBytes / rowbytes;
    if (ksplit > 1) rps = teams;                             // one row per team per stage
    const int ng = w->k / w->group;
    const int sbytes_row = ng * 2 * (w->symmetric ? 1 : 2);
    const int sms = q4_num_sms();
    int rpc = (w->n + sms - 1) / sms;
    rpc = std::max(1, std::min(rpc, kScaleBytes / sbytes_row));
    p.rows_per_cta = rpc;
    p.rows_per_stage = std::max(1, rps);
    const int grid = (w->n + rpc - 1) / rpc;
    return J == 2 ? launch_ksplit<2>(p, w->symmetric, ksplit, grid, stream)
                  : launch_ksplit<1>(p, w->symmetric, ksplit, grid, stream);
}
