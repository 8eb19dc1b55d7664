// W4A16 GEMV for small m (decode): y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[m][k],
// for one weight matrix or a group of independent ones in a single launch.
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a
// 16-bit type before the multiply) and §1 (small model, small batch: memory bound).
//
// HBM-bound design (the packed weights are streamed exactly once):
//  * each CTA owns a contiguous block of weight rows of one problem; a producer thread streams the
//    block (packed rows, and their scales and zeros, all contiguous in memory) through a 4-stage
//    shared-memory ring with cp.async.bulk, completion tracked by mbarriers;
//  * programmatic dependent launch: the CTA pulls its rows into L2 (a coherent prefetch) before it
//    waits for the previous kernel on the stream, so consecutive launches keep HBM busy across the
//    kernel boundary; x (which the previous kernel may produce) is read only after the wait;
//  * small CTAs (8 compute warps + 1 producer, few registers, ~70 KB shared memory) so that the next
//    launch's CTAs can be resident, and prefetching, while this launch finishes;
//  * every lane converts its own 64 values of x to fp16 pairs with its own power-of-two prescale
//    (max |x| * p in [1, 2): exact), so no block-wide reduction precedes the weight stream;
//  * in-register dequant: one LOP3 turns two nibbles into fp16x2 "1024 + code"; an HSUB2 of
//    (1024 + zero) leaves the exact integer (code - zero); nibbles 1, 3, 5, 7 of a word are used in
//    place (16 * code) and accumulate separately (scaled by 1/16 once per group); products accumulate
//    in fp16x2 over the lane's 2 chunks of one group (16 products per half), then in fp32 times the
//    group scale; a lane's two 16-byte chunks are adjacent, so they share one group and one scale;
//  * rows longer than 2048 codes are split over 2..8 warps and combined through shared memory.
#include "q4_common.cuh"
#include "tc_ptx.cuh"

namespace {

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;      // + one producer warp
constexpr int kWeightStage = 16384;                 // packed bytes per stage
constexpr int kStages = 4;
constexpr int kMaxM = 4;
constexpr int kMaxProblems = 8;

struct Problem {
    const uint16_t* x;       // [m][k] bf16
    const uint8_t* packed;   // [n][k/2]
    const __half* scales;    // [n][k/group]
    const __half* zeros;     // [n][k/group] or null
    void* y;                 // [m][n]
    int n;
    int cta_begin;           // first CTA of this problem
};

struct GemvParams {
    Problem prob[kMaxProblems];
    int count;
    int m, k, group, out_bf16;
    int rows_per_cta;        // contiguous weight rows per CTA
    int rows_per_stage;
    int stage_bytes;         // weights + scales (+ zeros) of one stage, 16-byte multiple
    int bulk_scales;         // scales/zeros travel in the stages (16-byte aligned rows of scales)
    int32_t* status;
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

// x pairs of one word (8 bf16 values e[0..3]) with prescale p, in the order word_dot consumes them.
__device__ __forceinline__ uint4 x_pairs(const uint4& v, float p)
{
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        f[2 * i] = __uint_as_float(e[i] << 16) * p;
        f[2 * i + 1] = __uint_as_float(e[i] & 0xFFFF0000u) * p;
    }
    uint4 o;
    o.x = h2_as_u32(__floats2half2_rn(f[0], f[4]));
    o.y = h2_as_u32(__floats2half2_rn(f[1], f[5]));
    o.z = h2_as_u32(__floats2half2_rn(f[2], f[6]));
    o.w = h2_as_u32(__floats2half2_rn(f[3], f[7]));
    return o;
}

__device__ __forceinline__ float bf16_amax(const uint4& v, bool& finite)
{
    const uint32_t e[4] = {v.x, v.y, v.z, v.w};
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float lo = __uint_as_float(e[i] << 16), hi = __uint_as_float(e[i] & 0xFFFF0000u);
        finite &= isfinite(lo) && isfinite(hi);
        a = fmaxf(a, fmaxf(fabsf(lo), fabsf(hi)));
    }
    return a;
}

template <int KSPLIT, int J, int MT, bool SYM>
__global__ void __launch_bounds__(kThreads, 2) w4a16_gemv_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int TEAMS = kComputeWarps / KSPLIT;
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kStages;
    float* red = reinterpret_cast<float*>(empty + kStages);          // [2][TEAMS][KSPLIT][MT]
    uint8_t* stages = smem + 1024;

    // this CTA's problem and rows
    int pi = 0;
    while (pi + 1 < p.count && (int)blockIdx.x >= p.prob[pi + 1].cta_begin) pi++;
    const Problem& P = p.prob[pi];
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int ng = p.k / p.group, cpg = p.group / 32, C = p.k / 32;
    const int64_t rowbytes = p.k / 2;
    const int r0 = ((int)blockIdx.x - P.cta_begin) * p.rows_per_cta;
    const int r1 = min(P.n, r0 + p.rows_per_cta);
    const int nstages = (r1 - r0 + p.rows_per_stage - 1) / p.rows_per_stage;
    const int wbytes = p.rows_per_stage * (int)rowbytes;            // weight part of a stage
    const int sbytes = p.rows_per_stage * ng * 2;                   // scale part of a stage

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], kComputeWarps); }
        tc::fence_mbar_init();
    }
    if (warp == kComputeWarps && lane == 0 && r0 < r1) {
        // weights do not depend on the previous kernel: start pulling them into L2 now
        prefetch_l2_range(P.packed + (int64_t)r0 * rowbytes, P.packed + (int64_t)r1 * rowbytes);
        prefetch_l2_range(P.scales + (int64_t)r0 * ng, P.scales + (int64_t)r1 * ng);
        if constexpr (!SYM) prefetch_l2_range(P.zeros + (int64_t)r0 * ng, P.zeros + (int64_t)r1 * ng);
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
                const int rows = min(p.rows_per_stage, r1 - rs);
                uint8_t* dst = stages + s * p.stage_bytes;
                uint32_t bytes = (uint32_t)(rows * rowbytes);
                if (p.bulk_scales) bytes += (uint32_t)(rows * ng * 2 * (SYM ? 1 : 2));
                tc::mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s(dst, P.packed + (int64_t)rs * rowbytes, (uint32_t)(rows * rowbytes), &full[s]);
                if (p.bulk_scales) {
                    bulk_g2s(dst + wbytes, P.scales + (int64_t)rs * ng, (uint32_t)(rows * ng * 2), &full[s]);
                    if constexpr (!SYM)
                        bulk_g2s(dst + wbytes + sbytes, P.zeros + (int64_t)rs * ng, (uint32_t)(rows * ng * 2), &full[s]);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- compute warps
    const int team = warp / KSPLIT, ks = warp % KSPLIT;
    const int c0 = ks * 32 * J + J * lane;          // the lane's first chunk (J adjacent chunks)
    const bool cvalid = c0 < C;
    const int gl = c0 / cpg;                        // their group (J <= cpg, c0 % J == 0)

    // x of the lane's chunks -> fp16 pairs with the lane's own power-of-two prescale
    uint4 X[MT][J][4];
    float inv_ps[MT];
#pragma unroll
    for (int mm = 0; mm < MT; mm++) {
        uint4 raw[J][4];
        float amax = 0.0f;
        bool finite = true;
#pragma unroll
        for (int j = 0; j < J; j++)
#pragma unroll
            for (int w = 0; w < 4; w++) {
                raw[j][w] = cvalid ? __ldg(reinterpret_cast<const uint4*>(P.x + (int64_t)mm * p.k + 32 * (c0 + j)) + w)
                                   : make_uint4(0, 0, 0, 0);
                amax = fmaxf(amax, bf16_amax(raw[j][w], finite));
            }
        if (!finite) q4_set_status(p.status, Q4_ERR_NONFINITE);
        const float ps = prescale_for(amax);
        inv_ps[mm] = 1.0f / ps;
#pragma unroll
        for (int j = 0; j < J; j++)
#pragma unroll
            for (int w = 0; w < 4; w++) X[mm][j][w] = x_pairs(raw[j][w], ps);
    }

    for (int st = 0; st < nstages; st++) {
        const int s = st % kStages;
        const int rs = r0 + st * p.rows_per_stage;
        const int rows_here = min(p.rows_per_stage, r1 - rs);
        if (!tc::mbar_wait(&full[s], (st / kStages) & 1, p.status, nullptr)) break;
        const uint8_t* sb = stages + s * p.stage_bytes;
        const __half* ssc = reinterpret_cast<const __half*>(sb + wbytes);
        const __half* szr = reinterpret_cast<const __half*>(sb + wbytes + sbytes);
        float* redb = red + (st & 1) * TEAMS * KSPLIT * MT;
        for (int rr = team; rr < rows_here; rr += TEAMS) {
            const int row = rs + rr;
            float part[MT];
#pragma unroll
            for (int mm = 0; mm < MT; mm++) part[mm] = 0.0f;
            if (cvalid) {
                float sc;
                __half z;
                if (p.bulk_scales) {
                    sc = __half2float(ssc[rr * ng + gl]);
                    z = SYM ? __float2half_rn(8.0f) : szr[rr * ng + gl];
                } else {
                    sc = __half2float(P.scales[(int64_t)row * ng + gl]);
                    z = SYM ? __float2half_rn(8.0f) : P.zeros[(int64_t)row * ng + gl];
                }
                const __half2 b1 = __half2half2(__hadd(z, __float2half_rn(1024.0f)));
                const __half2 b16 = __half2half2(__hfma(z, __float2half_rn(16.0f), __float2half_rn(1024.0f)));
                uint4 wv[J];
#pragma unroll
                for (int j = 0; j < J; j++) wv[j] = lds128(sb + rr * rowbytes + (c0 + j) * 16);
#pragma unroll
                for (int mm = 0; mm < MT; mm++) {
                    __half2 acc1 = __float2half2_rn(0.0f), acc16 = __float2half2_rn(0.0f);
#pragma unroll
                    for (int j = 0; j < J; j++) {
                        word_dot<SYM>(wv[j].x, b1, b16, X[mm][j][0], acc1, acc16);
                        word_dot<SYM>(wv[j].y, b1, b16, X[mm][j][1], acc1, acc16);
                        word_dot<SYM>(wv[j].z, b1, b16, X[mm][j][2], acc1, acc16);
                        word_dot<SYM>(wv[j].w, b1, b16, X[mm][j][3], acc1, acc16);
                    }
                    const float2 f = __half22float2(__hfma2(acc16, __float2half2_rn(0.0625f), acc1));
                    part[mm] = sc * (f.x + f.y) * inv_ps[mm];
                }
            }
#pragma unroll
            for (int mm = 0; mm < MT; mm++) {
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) part[mm] += __shfl_xor_sync(0xffffffffu, part[mm], off);
            }
            if (lane < MT) {
                float v = part[0];
#pragma unroll
                for (int mm = 1; mm < MT; mm++) if (lane == mm) v = part[mm];
                if constexpr (KSPLIT == 1) {
                    const int64_t o = (int64_t)lane * P.n + row;
                    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v);
                    else reinterpret_cast<float*>(P.y)[o] = v;
                } else {
                    redb[(team * KSPLIT + ks) * MT + lane] = v;   // one row per team per stage
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
                const int64_t o = (int64_t)lane * P.n + (rs + team);
                if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v);
                else reinterpret_cast<float*>(P.y)[o] = v;
            }
        }
    }
}

template <int KSPLIT, int J, int MT>
int launch(const GemvParams& p, int symmetric, int grid, cudaStream_t s)
{
    const size_t smem = 1024 + (size_t)kStages * p.stage_bytes;
    if (smem > 227 * 1024) return Q4_ERR_UNSUPPORTED;
    auto kern = symmetric ? w4a16_gemv_kernel<KSPLIT, J, MT, true> : w4a16_gemv_kernel<KSPLIT, J, MT, false>;
    if (const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))
        return q4_cuda_status(e);
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
    return q4_cuda_status(cudaLaunchKernelEx(&cfg, kern, p));
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

// Host entry used by q4_linear_w4a16 (count == 1) and q4_linear_w4a16_grouped: m <= 4, and every
// problem with the same k (a multiple of 64, at most 16384), group and symmetry.
int q4_gemv_w4a16_launch_group(int count, const uint16_t* const* x, int32_t m, const q4_weight* w, void* const* y,
                               int32_t out_dtype, int32_t* dev_status, cudaStream_t stream)
{
    if (count < 1 || count > kMaxProblems || m < 1 || m > kMaxM) return Q4_ERR_UNSUPPORTED;
    const int k = w[0].k, group = w[0].group, sym = w[0].symmetric;
    if (k % 64 || k > 16384) return Q4_ERR_UNSUPPORTED;
    for (int i = 1; i < count; i++)
        if (w[i].k != k || w[i].group != group || w[i].symmetric != sym) return Q4_ERR_UNSUPPORTED;
    GemvParams p = {};
    p.count = count;
    p.m = m;
    p.k = k;
    p.group = group;
    p.out_bf16 = out_dtype == Q4_OUT_BF16;
    p.status = dev_status;
    const int C = k / 32;
    const int J = 2;                                   // two adjacent chunks (64 codes) per lane
    int ksplit = 1;
    while (ksplit * 32 * J < C) ksplit *= 2;
    if (ksplit > 8) return Q4_ERR_UNSUPPORTED;
    const int teams = kComputeWarps / ksplit;
    const int rowbytes = k / 2;
    const int ng = k / group;
    int rps = ksplit > 1 ? teams : std::max(1, kWeightStage / rowbytes);
    p.rows_per_stage = rps;
    p.bulk_scales = (ng * 2) % 16 == 0;
    p.stage_bytes = rps * rowbytes + (p.bulk_scales ? rps * ng * 2 * (sym ? 1 : 2) : 0);
    p.stage_bytes = (p.stage_bytes + 15) & ~15;
    // rows per CTA: about two CTAs per SM over the whole group, whole stages where possible
    int64_t rows_total = 0;
    for (int i = 0; i < count; i++) rows_total += w[i].n;
    const int64_t target_ctas = 2LL * q4_num_sms();
    int rpc = (int)std::max<int64_t>(1, (rows_total + target_ctas - 1) / target_ctas);
    if (rpc > rps) rpc = (rpc + rps - 1) / rps * rps;
    p.rows_per_cta = rpc;
    int ctas = 0;
    for (int i = 0; i < count; i++) {
        Problem& P = p.prob[i];
        P.x = x[i];
        P.packed = w[i].packed;
        P.scales = reinterpret_cast<const __half*>(w[i].scales);
        P.zeros = reinterpret_cast<const __half*>(w[i].zeros);
        P.y = y[i];
        P.n = w[i].n;
        P.cta_begin = ctas;
        ctas += (w[i].n + rpc - 1) / rpc;
    }
    if (ctas == 0) return Q4_OK;
    return launch_ksplit<2>(p, sym, ksplit, ctas, stream);
}
