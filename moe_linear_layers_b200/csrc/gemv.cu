// W4A16 GEMV for small m (decode): y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[m][k],
// for one weight matrix or a group of independent ones in a single launch.
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a
// 16-bit type before the multiply) and §1 (small model, small batch: memory bound).
//
// HBM-bound design (the packed weights are streamed exactly once):
//  * each CTA owns a contiguous block of weight rows of one problem; a producer thread streams the
//    block (packed rows, and their scales and zeros, all contiguous in memory) through a shared-memory
//    ring with cp.async.bulk, completion tracked by mbarriers;
//  * programmatic dependent launch, weights first: the weights never depend on the previous kernel on
//    the stream, so the producer fills the whole ring (and pulls the rest of the CTA's rows into L2)
//    BEFORE anything waits for that kernel.  CTAs are small enough that the next launch's CTAs are
//    resident, filling their rings, while this launch computes: HBM stays busy across the chain of
//    dependent launches of a decode step.  Only the compute warps wait, and only they read x and
//    write y;
//  * after the wait, x is converted once per CTA: each thread turns one 16-byte word (8 values) into
//    int16 with the power-of-two scale of its 64-value block (max |x| * 2^e in [2^14, 2^15): every
//    bf16 value is kept to 2^-15 of the block maximum), staged in shared memory (XOR-swizzled); every
//    lane then loads its 64 values and takes their integer sum with DP2A against ones.  (Loading a
//    lane's 64 contiguous values straight from global memory instead is uncoalesced and slower;)
//  * integer dot products: a LOP3 spreads the low (high) nibbles of a packed word over four bytes and
//    two DP2A instructions multiply them with int16 x pairs into an int32 accumulator, so a row's
//    dot product with the lane's 64 x values (one group) is exact; the zero point comes out as
//    z * sum(x) in the same integers, and one conversion and one multiply by (group scale * 2^-e)
//    give the lane's fp32 share.  (DP2A sustains about twice the code rate of an fp16 dequant-and-HFMA2
//    loop on this GPU, which alone would barely keep up with HBM;)
//  * a warp handles two rows at a time; their lane sums are reduced together (one exchange, then a
//    4-step butterfly), so a row costs half the shuffles;
//  * rows longer than 2048 codes are split over 2..8 warps; their partial sums meet in shared memory
//    once, at the end of the CTA.
#include "gemv_common.cuh"

#ifndef Q4_GEMV_STAGES
#define Q4_GEMV_STAGES 6
#endif
#ifndef Q4_GEMV_CTAS_PER_SM
#define Q4_GEMV_CTAS_PER_SM 1
#endif
#ifndef Q4_GEMV_MIN_BLOCKS
#define Q4_GEMV_MIN_BLOCKS 2
#endif

namespace {

using namespace gemv;

constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;
constexpr int kThreads = kComputeThreads + 32;      // + one producer warp
constexpr int kWeightStage = 16384;                 // packed bytes per stage
constexpr int kStages = Q4_GEMV_STAGES;
constexpr int kMaxM = 4;
constexpr int kMaxProblems = 8;
constexpr int kLaneK = 64;                          // k values per lane: two adjacent 16-byte chunks
constexpr int kWarpK = 32 * kLaneK;                 // 2048
constexpr int kRedBytesMax = 16384;                 // split-k partial sums per CTA

struct Problem {
    const uint16_t* x;       // [m][k] bf16 (unused when g is set)
    const float* g;          // fused SwiGLU input: x = silu(g) * u, fp32 [m][k] each (or null)
    const float* u;
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
    int xs_off, ips_off, red_off, ring_off;   // shared-memory carve, bytes
    int32_t* status;
};

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kComputeThreads) : "memory"); }

template <int MT>
__device__ __forceinline__ void stage_swiglu(const float* g, const float* u, int k, int nw, uint4* xs, float* xinv,
                                             int32_t* status)
{
    bool bad = false;
#pragma unroll
    for (int mm = 0; mm < MT; mm++) {
        const float4* gr = reinterpret_cast<const float4*>(g + (int64_t)mm * k);
        const float4* ur = reinterpret_cast<const float4*>(u + (int64_t)mm * k);
        for (int i = 0; i * kComputeThreads < nw; i++) {   // uniform; nw % 8 == 0 keeps blocks together
            const int w = i * kComputeThreads + threadIdx.x;
            float h[8];
            uint32_t a = 0;
            if (w < nw) {
                const float4 g0 = __ldg(gr + 2 * w), g1 = __ldg(gr + 2 * w + 1);
                const float4 u0 = __ldg(ur + 2 * w), u1 = __ldg(ur + 2 * w + 1);
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    h[j] = gv[j] * __frcp_rn(1.0f + __expf(-gv[j])) * uv[j];
                    bad |= !isfinite(h[j]);
                    a = max(a, __float_as_uint(h[j]) & 0x7FFFFFFFu);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 8; j++) h[j] = 0.0f;
            }
            a = max(a, __shfl_xor_sync(0xffffffffu, a, 1));
            a = max(a, __shfl_xor_sync(0xffffffffu, a, 2));
            a = max(a, __shfl_xor_sync(0xffffffffu, a, 4));
            const float2 sc = block_scale_f32(a);
            if (w < nw) {
                const int L = w >> 3, j = w & 7;
                xs[mm * nw + (L << 3) + (j ^ (L & 7))] = x_ints_f32(h, sc.x);
                if (j == 0) xinv[mm * (nw / 8) + L] = sc.y;
            }
        }
    }
    if (bad) q4_set_status(status, Q4_ERR_NONFINITE);
}

template <int KSPLIT, int MT, bool SYM, bool SWIGLU>
__global__ void __launch_bounds__(kThreads, MT == 1 ? Q4_GEMV_MIN_BLOCKS : 2) w4a16_gemv_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int TEAMS = kComputeWarps / KSPLIT;
    constexpr bool PAIR = MT <= 2;                  // two rows per warp iteration
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint32_t* consumed = reinterpret_cast<uint32_t*>(full + kStages);   // [kComputeWarps] stages finished per warp
    uint4* xs = reinterpret_cast<uint4*>(smem + p.xs_off);      // [MT][k/8] int16 x pairs, swizzled
    float* xinv = reinterpret_cast<float*>(smem + p.ips_off);   // [MT][k/64] 2^-e of each block
    float* red = reinterpret_cast<float*>(smem + p.red_off);    // [rows_per_cta][KSPLIT][MT]
    uint8_t* ring = smem + p.ring_off;

    // this CTA's problem and rows
    int pi = 0;
    while (pi + 1 < p.count && (int)blockIdx.x >= p.prob[pi + 1].cta_begin) pi++;
    const Problem& P = p.prob[pi];
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int ng = p.k / p.group, C = p.k / 32, nw = p.k / 8;
    const int64_t rowbytes = p.k / 2;
    const int rps = p.rows_per_stage;
    const int r0 = ((int)blockIdx.x - P.cta_begin) * p.rows_per_cta;
    const int r1 = min(P.n, r0 + p.rows_per_cta);
    const int nstages = (r1 - r0 + rps - 1) / rps;
    const int wbytes = rps * (int)rowbytes;                     // weight part of a stage
    const int sbytes = rps * ng * 2;                            // scale part of a stage

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) tc::mbar_init(&full[i], 1);
        for (int i = 0; i < kComputeWarps; i++) consumed[i] = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kComputeWarps) {
        // ------------------------------------------------------------------ producer (never waits for
        // the previous kernel: it reads only weights)
        if (lane == 0 && nstages > 0) {
            auto issue = [&](int st) {
                const int s = st % kStages;
                const int rs = r0 + st * rps;
                const int rows = min(rps, r1 - rs);
                uint8_t* dst = ring + s * p.stage_bytes;
                uint32_t bytes = (uint32_t)(rows * rowbytes);
                if (p.bulk_scales) bytes += (uint32_t)(rows * ng * 2 * (SYM ? 1 : 2));
                tc::mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s(dst, P.packed + (int64_t)rs * rowbytes, (uint32_t)(rows * rowbytes), &full[s]);
                if (p.bulk_scales) {
                    bulk_g2s(dst + wbytes, P.scales + (int64_t)rs * ng, (uint32_t)(rows * ng * 2), &full[s]);
                    if constexpr (!SYM)
                        bulk_g2s(dst + wbytes + sbytes, P.zeros + (int64_t)rs * ng, (uint32_t)(rows * ng * 2), &full[s]);
                }
            };
            const int pre = min(nstages, kStages);
            for (int st = 0; st < pre; st++) issue(st);
            // x too: an L2 prefetch is coherent, so it is safe before the wait and shortens the read after it
            if constexpr (SWIGLU) {
                prefetch_l2(P.g, (uint32_t)(p.m * p.k * 4));
                prefetch_l2(P.u, (uint32_t)(p.m * p.k * 4));
            } else {
                prefetch_l2(P.x, (uint32_t)(p.m * p.k * 2));
            }
            if (nstages > kStages) {
                const int rl = r0 + kStages * rps;
                prefetch_l2_range(P.packed + (int64_t)rl * rowbytes, P.packed + (int64_t)r1 * rowbytes);
                if (p.bulk_scales) {
                    prefetch_l2_range(P.scales + (int64_t)rl * ng, P.scales + (int64_t)r1 * ng);
                    if constexpr (!SYM) prefetch_l2_range(P.zeros + (int64_t)rl * ng, P.zeros + (int64_t)r1 * ng);
                }
            }
            // beyond the first fill the producer polls the compute warps' counters with plain loads: an
            // mbarrier wait would also wait for this thread's own bulk copies in flight
            for (int st = kStages; st < nstages; st++) {
                if (!tc::poll_counters<kComputeWarps>(consumed, st - kStages + 1, p.status, nullptr)) break;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(st);
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- compute warps
    pdl_wait();   // x (and the y buffer) may belong to the previous kernel on the stream

    // x -> int16 with the power-of-two scale of its 64-value block: one 16-byte word (8 values) per
    // thread and pass (coalesced), all loads issued first and the passes independent of one another;
    // the 8 threads of a block share its scale.  Word w of block L is staged at 8L + ((w % 8) ^ (L % 8)):
    // conflict-free lane loads.
    if constexpr (SWIGLU) {
        stage_swiglu<MT>(P.g, P.u, p.k, nw, xs, xinv, p.status);
    } else {
        constexpr int kMaxPasses = 16384 / 8 / kComputeThreads;
        uint32_t bad = 0;
#pragma unroll
        for (int mm = 0; mm < MT; mm++) {
            const uint4* xrow = reinterpret_cast<const uint4*>(P.x + (int64_t)mm * p.k);
            uint4 raw[kMaxPasses];
#pragma unroll
            for (int i = 0; i < kMaxPasses; i++) {
                const int w = i * kComputeThreads + threadIdx.x;
                raw[i] = w < nw ? __ldg(xrow + w) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < kMaxPasses; i++) {
                if (i * kComputeThreads < nw) {   // uniform; nw % 8 == 0 keeps blocks of 8 threads together
                    const int w = i * kComputeThreads + threadIdx.x;
                    uint32_t a = bf16_mag_max(raw[i], bad);
                    a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 1));
                    a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 2));
                    a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 4));
                    const float2 sc = block_scale(max(a & 0xFFFFu, a >> 16));
                    if (w < nw) {
                        const int L = w >> 3, j = w & 7;
                        xs[mm * nw + (L << 3) + (j ^ (L & 7))] = x_ints(raw[i], sc.x);
                        if (j == 0) xinv[mm * (nw / 8) + L] = sc.y;
                    }
                }
            }
        }
        if (bad) q4_set_status(p.status, Q4_ERR_NONFINITE);
    }
    compute_bar();

    const int team = warp / KSPLIT, ks = warp % KSPLIT;
    const int L = ks * 32 + lane;                   // the lane's 64-value block of k
    const int c0 = 2 * L;                           // its first 16-byte chunk
    const bool cvalid = c0 < C;
    const int gl = L * kLaneK / p.group;            // its group
    uint4 X[MT][8];
    float inv_xs[MT];
    int xsum[MT];
#pragma unroll
    for (int mm = 0; mm < MT; mm++) {
#pragma unroll
        for (int i = 0; i < 8; i++)
            X[mm][i] = cvalid ? xs[mm * nw + (L << 3) + (i ^ (L & 7))] : make_uint4(0, 0, 0, 0);
        inv_xs[mm] = cvalid ? xinv[mm * (nw / 8) + L] : 0.0f;
        // the lane's integer sum of x, for the zero point: DP2A against ones, four chains
        int s4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            s4[0] = dp2a_lo(X[mm][i].x, 0x01010101u, s4[0]);
            s4[1] = dp2a_lo(X[mm][i].y, 0x01010101u, s4[1]);
            s4[2] = dp2a_lo(X[mm][i].z, 0x01010101u, s4[2]);
            s4[3] = dp2a_lo(X[mm][i].w, 0x01010101u, s4[3]);
        }
        xsum[mm] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
    }

    for (int st = 0; st < nstages; st++) {
        const int s = st % kStages;
        const int rs = r0 + st * rps;
        const int rows_here = min(rps, r1 - rs);
        if (!tc::mbar_wait(&full[s], (st / kStages) & 1, p.status, nullptr)) break;
        const uint8_t* sb = ring + s * p.stage_bytes;
        for (int ra = team; ra < rows_here; ra += (PAIR ? 2 : 1) * TEAMS) {
            const int rb = ra + TEAMS;
            const bool hasb = PAIR && rb < rows_here;
            float pa[MT], pb[MT];
#pragma unroll
            for (int mm = 0; mm < MT; mm++) pa[mm] = pb[mm] = 0.0f;
            if (cvalid) {
                const __half* sa = p.bulk_scales ? reinterpret_cast<const __half*>(sb + wbytes) + ra * ng
                                                 : P.scales + (int64_t)(rs + ra) * ng;
                const __half* za = p.bulk_scales ? reinterpret_cast<const __half*>(sb + wbytes + sbytes) + ra * ng
                                                 : P.zeros + (int64_t)(rs + ra) * ng;
                row_dot<SYM, MT>(sb + ra * rowbytes + c0 * 16, sa, za, gl, X, inv_xs, xsum, pa);
                if (hasb) {
                    const int d = (rb - ra) * ng;
                    row_dot<SYM, MT>(sb + rb * rowbytes + c0 * 16, sa + d, SYM ? za : za + d, gl, X, inv_xs, xsum, pb);
                }
            }
            if constexpr (PAIR) {
                // lanes 0-15 end with row a, lanes 16-31 with row b
                const bool hi = lane & 16;
#pragma unroll
                for (int mm = 0; mm < MT; mm++) {
                    float v = hi ? pb[mm] : pa[mm];
                    v += __shfl_xor_sync(0xffffffffu, hi ? pa[mm] : pb[mm], 16);
#pragma unroll
                    for (int off = 8; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    pa[mm] = v;
                }
                if ((lane & 15) == 0 && (!hi || hasb)) {
                    const int rr = hi ? rb : ra;
#pragma unroll
                    for (int mm = 0; mm < MT; mm++) {
                        if constexpr (KSPLIT == 1)
                            store_y(P.y, (int64_t)mm * P.n + rs + rr, pa[mm], p.out_bf16, (int64_t)p.m * P.n, p.status);
                        else red[((rs - r0 + rr) * KSPLIT + ks) * MT + mm] = pa[mm];
                    }
                }
            } else {
#pragma unroll
                for (int mm = 0; mm < MT; mm++)
#pragma unroll
                    for (int off = 16; off >= 1; off >>= 1) pa[mm] += __shfl_xor_sync(0xffffffffu, pa[mm], off);
                if (lane < MT) {
                    float v = pa[0];
#pragma unroll
                    for (int mm = 1; mm < MT; mm++) if (lane == mm) v = pa[mm];
                    if constexpr (KSPLIT == 1)
                        store_y(P.y, (int64_t)lane * P.n + rs + ra, v, p.out_bf16, (int64_t)p.m * P.n, p.status);
                    else red[((rs - r0 + ra) * KSPLIT + ks) * MT + lane] = v;
                }
            }
        }
        __syncwarp();
        if (lane == 0) tc::sts_publish(&consumed[warp], st + 1);   // this warp is done with the stage
    }

    if constexpr (KSPLIT > 1) {
        compute_bar();
        const int rows = r1 - r0;
        for (int i = threadIdx.x; i < rows * MT; i += kComputeThreads) {
            const int rr = i / MT, mm = i % MT;
            float v = 0.0f;
#pragma unroll
            for (int t = 0; t < KSPLIT; t++) v += red[(rr * KSPLIT + t) * MT + mm];
            store_y(P.y, (int64_t)mm * P.n + r0 + rr, v, p.out_bf16, (int64_t)p.m * P.n, p.status);
        }
    }
}

template <int KSPLIT, int MT>
int launch(const GemvParams& p, int symmetric, bool swiglu, int grid, size_t smem, cudaStream_t s)
{
    auto kern = swiglu ? (symmetric ? w4a16_gemv_kernel<KSPLIT, MT, true, true> : w4a16_gemv_kernel<KSPLIT, MT, false, true>)
                       : (symmetric ? w4a16_gemv_kernel<KSPLIT, MT, true, false> : w4a16_gemv_kernel<KSPLIT, MT, false, false>);
    // the shared-memory opt-in is set once per device and instantiation (it does not affect occupancy)
    static uint64_t opted[4] = {0, 0, 0, 0};
    const int slot = (symmetric ? 1 : 0) + (swiglu ? 2 : 0);
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(opted[slot] & bit)) {
        if (const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024))
            return q4_cuda_status(e);
        opted[slot] |= bit;
    }
    // Programmatic stream serialization: the kernel may start, and fill its weight ring, while the
    // previous kernel on the stream runs; x is read only after griddepcontrol.wait.
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

template <int KSPLIT>
int launch_m(const GemvParams& p, int symmetric, bool swiglu, int grid, size_t smem, cudaStream_t s)
{
    switch (p.m) {
        case 1: return launch<KSPLIT, 1>(p, symmetric, swiglu, grid, smem, s);
        case 2: return launch<KSPLIT, 2>(p, symmetric, swiglu, grid, smem, s);
        case 3: return launch<KSPLIT, 3>(p, symmetric, swiglu, grid, smem, s);
        default: return launch<KSPLIT, 4>(p, symmetric, swiglu, grid, smem, s);
    }
}

}  // namespace

// Host entry used by q4_linear_w4a16 (count == 1) and q4_linear_w4a16_grouped: m <= 4, and every
// problem with the same k (a multiple of 64, at most 16384), group and symmetry.
// g, u (nullable, both or neither): the problems' inputs are silu(g[i]) * u[i] instead of x[i].
int q4_gemv_w4a16_launch_group(int count, const uint16_t* const* x, int32_t m, const q4_weight* w, void* const* y,
                               int32_t out_dtype, int32_t* dev_status, cudaStream_t stream,
                               const float* const* g, const float* const* u)
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
    int ksplit = 1;
    while (ksplit * kWarpK < k) ksplit *= 2;
    if (ksplit > 8) return Q4_ERR_UNSUPPORTED;
    const int rowbytes = k / 2;
    const int ng = k / group;
    const int rps = std::max(1, kWeightStage / rowbytes);
    p.rows_per_stage = rps;
    p.bulk_scales = (ng * 2) % 16 == 0;
    p.stage_bytes = rps * rowbytes + (p.bulk_scales ? rps * ng * 2 * (sym ? 1 : 2) : 0);
    p.stage_bytes = (p.stage_bytes + 15) & ~15;
    // rows per CTA: a fixed number of CTAs per SM over the whole group
    int64_t rows_total = 0;
    for (int i = 0; i < count; i++) rows_total += w[i].n;
    const int64_t target_ctas = (int64_t)Q4_GEMV_CTAS_PER_SM * q4_num_sms();
    // (balanced over the SMs: a CTA's last stage may be partial)
    int rpc = (int)std::max<int64_t>(1, (rows_total + target_ctas - 1) / target_ctas);
    if (ksplit > 1) rpc = std::min(rpc, std::max(rps, kRedBytesMax / (ksplit * m * 4)));
    p.rows_per_cta = rpc;
    // shared memory: barriers | int16 x | per-block inverse scale | split-k partials | weight ring
    p.xs_off = 128;
    p.ips_off = p.xs_off + m * k * 2;
    p.red_off = p.ips_off + m * (k / 64) * 4;
    const int red_bytes = ksplit > 1 ? rpc * ksplit * m * 4 : 0;
    p.ring_off = (p.red_off + red_bytes + 127) & ~127;
    const size_t smem = (size_t)p.ring_off + (size_t)kStages * p.stage_bytes;
    if (smem > 227 * 1024) return Q4_ERR_UNSUPPORTED;
    int ctas = 0;
    for (int i = 0; i < count; i++) {
        Problem& P = p.prob[i];
        P.x = x ? x[i] : nullptr;
        P.g = g ? g[i] : nullptr;
        P.u = u ? u[i] : nullptr;
        P.packed = w[i].packed;
        P.scales = reinterpret_cast<const __half*>(w[i].scales);
        P.zeros = reinterpret_cast<const __half*>(w[i].zeros);
        P.y = y[i];
        P.n = w[i].n;
        P.cta_begin = ctas;
        ctas += (w[i].n + rpc - 1) / rpc;
    }
    if (ctas == 0) return Q4_OK;
    switch (ksplit) {
        case 1: return launch_m<1>(p, sym, g != nullptr, ctas, smem, stream);
        case 2: return launch_m<2>(p, sym, g != nullptr, ctas, smem, stream);
        case 4: return launch_m<4>(p, sym, g != nullptr, ctas, smem, stream);
        default: return launch_m<8>(p, sym, g != nullptr, ctas, smem, stream);
    }
}
