// W4A16 GEMV chain at m = 1: a sequence of DEPENDENT stages of GEMVs (a decode step: per layer [q,k,v],
// o, [gate,up], down) in ONE persistent launch.
//
// Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored before the
// multiply) and §1 (small model, small batch: memory bound).  Every stage computes, for each of its
// problems, y[n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x[k] exactly as q4_linear_w4a16's
// GEMV does (x per 64-value block as int16 with a power-of-two scale, exact int32 dot products); the
// chain only changes WHEN work may start.
//
// Why one launch: a decode step is a chain of dependent GEMVs, and a launch per stage pays the launch-to-
// launch dependency latency (about 2 us on this GPU) 64 times per step, which alone caps a 64-stage step
// far below HBM bandwidth.  Here the dependency is a counter per stage in global memory:
//  * one CTA per SM (cooperative launch: every CTA is resident), 16 compute warps and a producer warp;
//  * each stage's weight rows are split over the CTAs, each problem of the stage getting CTAs in proportion
//    to its rows, so that a CTA serves one problem (stages one x) per stage;
//  * the producer streams the CTA's rows of every stage, in stage order, through a shared-memory ring
//    with cp.async.bulk (evict-first in L2, so that activations and outputs stay cached).  It never waits
//    for the dependency: weights do not depend on it.  Nor does it wait on an mbarrier for a free slot:
//    on this GPU a thread's mbarrier wait also waits for that thread's own bulk copies in flight, which
//    would leave one chunk in flight per HBM round trip; the compute warps publish the chunks they have
//    finished in per-warp shared-memory counters, which the producer polls with plain loads;
//  * a prefetch warp pulls the rows of the next ~1.3 layers (and their x) into L2, paced by the same
//    counters, so that HBM keeps streaming while the compute warps wait at stage boundaries;
//  * the compute warps of stage s wait until every CTA has finished stage s-1 (one thread polls the
//    stage's arrival counter with acquire loads, bounded in time), then read x -- which may be an output of
//    an earlier stage -- and reduce the rows already waiting in the ring; they then publish their own
//    arrival (block barrier, fence, atomic add).  The last CTA to arrive at the final stage resets the
//    counters, so the next call finds them zero.
//  * A stage input may also be the SwiGLU gating of two fp32 outputs of an earlier stage:
//    x = silu(g) * u, formed while x is staged (the dense FFN's down projection on its gate/up outputs).
// A wait that runs out records Q4_ERR_TIMEOUT, raises the abort word (sync[0]) that every other CTA's wait
// also watches, lets the CTA's own bulk copies land and returns.
#include "gemv_common.cuh"

namespace {

using namespace gemv;

#ifndef Q4_CHAIN_WARPS
#define Q4_CHAIN_WARPS 16
#endif
constexpr int kCW = Q4_CHAIN_WARPS;        // compute warps
constexpr int kCT = kCW * 32;
constexpr int kThreads = kCT + 64;         // + a producer warp and an L2 prefetch warp
constexpr int kChunkW = 32768;             // packed weight bytes per ring chunk
constexpr int kMaxK = 16384;
constexpr int kMaxProblems = 256;
constexpr int kMaxStages = 128;
constexpr int kMaxStageProblems = 8;
constexpr int kRedFloats = 2048;           // split-k partial sums per CTA and stage
#ifndef Q4_CHAIN_L2_AHEAD
#define Q4_CHAIN_L2_AHEAD 12
#endif
// chunks the prefetch warp keeps in L2 ahead of the compute warps (about 1.3 decode layers of a CTA's rows:
// some 60 MB of the 126 MB L2 over all SMs)
constexpr int kL2Ahead = Q4_CHAIN_L2_AHEAD;

struct ChainProblem {
    const uint16_t* x;       // bf16 [k] (null when g is set)
    const float* g;          // SwiGLU input: x = silu(g) * u, fp32 [k] each
    const float* u;
    const uint8_t* packed;   // [n][k/2]
    const __half* scales;    // [n][k/group]
    const __half* zeros;     // [n][k/group] or null
    void* y;                 // [n]
    int n;
    int row0;                // first row of the problem in its stage's row concatenation
    int cta0, ncta, rpc;     // the CTAs that share its rows (a CTA serves one problem per stage), rows each
};

struct ChainStage {
    int k;                   // reduction length of every problem of the stage
    int p0, np;              // problems p0 .. p0+np-1
    int rows;                // sum of their n
    int rps;                 // rows per ring chunk
    int ksplit;              // warps per row (k > 2048 * ksplit never)
    int bulk_scales;         // scales (and zeros) travel in the chunks
};

struct ChainParams {
    ChainProblem prob[kMaxProblems];
    ChainStage st[kMaxStages];
    int nstages, group, out_bf16;
    int slot_bytes, nslots;
    int xs_off, xinv_off, red_off, ring_off, bar_off;
    uint32_t* sync;          // [0] abort word, [32 (1 + s)] arrivals at stage s (a 128-byte line each)
    int32_t* status;
};

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)), "l"(pol) : "memory");
}

// Wait (plain shared-memory loads, a short sleep between rounds so the compute warps on the producer's
// scheduler keep their issue slots) until every compute warp has finished `target` chunks.  Bounded: after
// tc::kWaitLimitNs, or when the CTA's abort flag rises, it records Q4_ERR_TIMEOUT / returns false.
__device__ __forceinline__ bool poll_consumed(const uint32_t* consumed, uint32_t target, int32_t* status,
                                              volatile int* abort_cta)
{
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t round = 0;; round++) {
        bool ok = true;
#pragma unroll
        for (int i = 0; i < kCW; i++) ok &= tc::lds_weak(consumed + i) >= target;
        if (ok) return true;
        if (*abort_cta) return false;
        if (tc::wait_expired(t0, tc::kWaitLimitNs, round, 1u << 12)) {
            q4_set_status(status, Q4_ERR_TIMEOUT);
            *abort_cta = 1;
            return false;
        }
        __nanosleep(64);
    }
}

// The CTA's rows [a, b) of stage s, and its chunks: a chunk is at most rps rows of one problem.
struct Chunk {
    int pi;       // problem
    int lr;       // first row inside the problem
    int rows;
    int cr;       // first row relative to the CTA's range (split-k partial sums)
};

// The CTA's rows [a, b) of stage S (concatenated row numbers): a block of one problem's rows, so that the CTA
// stages one x per stage; a CTA beyond the stage's CTAs gets none.
__device__ __forceinline__ void cta_range(const ChainParams& p, const ChainStage& S, int& a, int& b)
{
    a = b = S.rows;
    for (int pi = S.p0; pi < S.p0 + S.np; pi++) {
        const ChainProblem& P = p.prob[pi];
        const int c = (int)blockIdx.x - P.cta0;
        if (c >= 0 && c < P.ncta) {
            a = min(P.row0 + P.n, P.row0 + c * P.rpc);
            b = min(P.row0 + P.n, a + P.rpc);
        }
    }
}

// Chunk starting at concatenated row r (< b) of stage S.
__device__ __forceinline__ Chunk chunk_at(const ChainParams& p, const ChainStage& S, int r, int a, int b)
{
    int pi = S.p0;
    while (pi + 1 < S.p0 + S.np && p.prob[pi + 1].row0 <= r) pi++;
    const ChainProblem& P = p.prob[pi];
    Chunk c;
    c.pi = pi;
    c.lr = r - P.row0;
    c.rows = min(min(b, P.row0 + P.n), r + S.rps) - r;
    c.cr = r - a;
    return c;
}

// x (or silu(g) * u) of problem P -> int16 per 64-value block with a power-of-two scale, staged in
// shared memory exactly as the single-launch GEMV stages it (word w of block L at 8L + ((w % 8) ^ (L % 8))).
__device__ __forceinline__ void stage_x(const ChainProblem& P, int k, uint4* xs, float* xinv, int32_t* status)
{
    const int nw = k / 8;
    uint32_t bad = 0;
    if (P.g) {
        bool nonfinite = false;
        for (int i = 0; i * kCT < nw; i++) {   // uniform; nw % 8 == 0 keeps blocks of 8 threads together
            const int w = i * kCT + threadIdx.x;
            float h[8];
            uint32_t a = 0;
            if (w < nw) {
                const float4* gr = reinterpret_cast<const float4*>(P.g);
                const float4* ur = reinterpret_cast<const float4*>(P.u);
                const float4 g0 = __ldcg(gr + 2 * w), g1 = __ldcg(gr + 2 * w + 1);
                const float4 u0 = __ldcg(ur + 2 * w), u1 = __ldcg(ur + 2 * w + 1);
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    h[j] = gv[j] * __frcp_rn(1.0f + __expf(-gv[j])) * uv[j];
                    nonfinite |= !isfinite(h[j]);
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
                xs[(L << 3) + (j ^ (L & 7))] = x_ints_f32(h, sc.x);
                if (j == 0) xinv[L] = sc.y;
            }
        }
        if (nonfinite) q4_set_status(status, Q4_ERR_NONFINITE);
        return;
    }
    const uint4* xrow = reinterpret_cast<const uint4*>(P.x);
    constexpr int kPasses = kMaxK / 8 / kCT;
    uint4 raw[kPasses];
#pragma unroll
    for (int i = 0; i < kPasses; i++) {
        const int w = i * kCT + threadIdx.x;
        raw[i] = w < nw ? __ldcg(xrow + w) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kPasses; i++) {
        if (i * kCT < nw) {
            const int w = i * kCT + threadIdx.x;
            uint32_t a = bf16_mag_max(raw[i], bad);
            a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 1));
            a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 2));
            a = __vmaxu2(a, __shfl_xor_sync(0xffffffffu, a, 4));
            const float2 sc = block_scale(max(a & 0xFFFFu, a >> 16));
            if (w < nw) {
                const int L = w >> 3, j = w & 7;
                xs[(L << 3) + (j ^ (L & 7))] = x_ints(raw[i], sc.x);
                if (j == 0) xinv[L] = sc.y;
            }
        }
    }
    if (bad) q4_set_status(status, Q4_ERR_NONFINITE);
}

template <bool SYM>
__global__ void __launch_bounds__(kThreads, 1) w4a16_gemv_chain_kernel(const __grid_constant__ ChainParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
    uint32_t* consumed = reinterpret_cast<uint32_t*>(full + p.nslots);   // [kCW] chunks finished per warp
    volatile int* abort_cta = reinterpret_cast<volatile int*>(consumed + kCW);
    uint4* xs = reinterpret_cast<uint4*>(smem + p.xs_off);
    float* xinv = reinterpret_cast<float*>(smem + p.xinv_off);
    float* red = reinterpret_cast<float*>(smem + p.red_off);
    uint8_t* ring = smem + p.ring_off;
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int ng_of = p.group;   // k / group per stage below

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.nslots; i++) tc::mbar_init(&full[i], 1);
        for (int i = 0; i < kCW; i++) consumed[i] = 0;
        *abort_cta = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();

    if (warp == kCW + 1) {
        // -------------------------------------------------------------- L2 prefetch warp
        // Walks the same chunks as the producer and pulls each into L2 (weights, scales, zeros, and the
        // stage's x) once the compute warps are within kL2Ahead chunks of it, so that HBM keeps streaming
        // while the compute warps wait at a stage boundary and the ring refills from L2.  It issues no
        // copy into shared memory and waits on no mbarrier.
        if (lane != 0 || kL2Ahead <= 0) return;
        uint32_t j = 0;
        for (int s = 0; s < p.nstages; s++) {
            const ChainStage& S = p.st[s];
            int a, b;
            cta_range(p, S, a, b);
            const int64_t rowbytes = S.k / 2;
            const int ng = S.k / ng_of;
            int cur = -1;
            for (int r = a; r < b; j++) {
                const Chunk c = chunk_at(p, S, r, a, b);
                const ChainProblem& P = p.prob[c.pi];
                if (j > (uint32_t)kL2Ahead && !poll_consumed(consumed, j - kL2Ahead, p.status, abort_cta)) return;
                prefetch_l2(P.packed + (int64_t)c.lr * rowbytes, (uint32_t)(c.rows * rowbytes));
                if (S.bulk_scales) {
                    prefetch_l2(P.scales + (int64_t)c.lr * ng, (uint32_t)(c.rows * ng * 2));
                    if constexpr (!SYM) prefetch_l2(P.zeros + (int64_t)c.lr * ng, (uint32_t)(c.rows * ng * 2));
                }
                if (c.pi != cur) {   // the problem's input (a hint only: L2 serves the latest writes)
                    cur = c.pi;
                    if (P.g) {
                        prefetch_l2(P.g, (uint32_t)(S.k * 4));
                        prefetch_l2(P.u, (uint32_t)(S.k * 4));
                    } else {
                        prefetch_l2(P.x, (uint32_t)(S.k * 2));
                    }
                }
                r += c.rows;
            }
        }
        return;
    }
    if (warp == kCW) {
        // -------------------------------------------------------------- producer (weights only)
        if (lane != 0) return;
        const uint64_t pol = evict_first_policy();
        uint32_t it = 0;          // chunks issued
        bool ok = true;
        for (int s = 0; s < p.nstages && ok; s++) {
            const ChainStage& S = p.st[s];
            int a, b;
            cta_range(p, S, a, b);
            const int64_t rowbytes = S.k / 2;
            const int ng = S.k / ng_of;
            const int wbytes = S.rps * (int)rowbytes, sbytes = S.rps * ng * 2;
            for (int r = a; r < b; it++) {
                const Chunk c = chunk_at(p, S, r, a, b);
                const ChainProblem& P = p.prob[c.pi];
                const int slot = it % p.nslots;
                if (it >= (uint32_t)p.nslots) {
                    // chunk it - nslots, the slot's previous one, is finished by every compute warp
                    if (!(ok = poll_consumed(consumed, it - p.nslots + 1, p.status, abort_cta))) break;
                    // the warps' reads of the slot (generic proxy) before the copy's writes (async proxy)
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                uint8_t* dst = ring + slot * p.slot_bytes;
                const uint32_t wb = (uint32_t)(c.rows * rowbytes);
                uint32_t bytes = wb;
                if (S.bulk_scales) bytes += (uint32_t)(c.rows * ng * 2 * (SYM ? 1 : 2));
                tc::mbar_arrive_expect_tx(&full[slot], bytes);
                bulk_g2s_hint(dst, P.packed + (int64_t)c.lr * rowbytes, wb, &full[slot], pol);
                if (S.bulk_scales) {
                    bulk_g2s_hint(dst + wbytes, P.scales + (int64_t)c.lr * ng, (uint32_t)(c.rows * ng * 2), &full[slot], pol);
                    if constexpr (!SYM)
                        bulk_g2s_hint(dst + wbytes + sbytes, P.zeros + (int64_t)c.lr * ng, (uint32_t)(c.rows * ng * 2),
                                      &full[slot], pol);
                }
                r += c.rows;
            }
        }
        if (!ok) {   // let every copy this thread issued land before the CTA can exit
            for (uint32_t j = it > (uint32_t)p.nslots ? it - p.nslots : 0; j < it; j++)
                tc::mbar_wait(&full[j % p.nslots], (j / p.nslots) & 1, p.status, nullptr, 100000000ull);
        }
        return;
    }

    // ------------------------------------------------------------------ compute warps
    // A raised abort word means an earlier call gave up and left the counters behind: report, do nothing.
    if (threadIdx.x == 0 && ld_relaxed_gpu(p.sync)) {
        q4_set_status(p.status, Q4_ERR_TIMEOUT);
        *abort_cta = 1;
    }
    compute_bar();
    if (*abort_cta) return;
    uint32_t it = 0;   // chunks consumed
    for (int s = 0; s < p.nstages; s++) {
        const ChainStage& S = p.st[s];
        // wait for every CTA to have finished stage s - 1 (its outputs may be this stage's inputs)
        if (s > 0) {
            if (threadIdx.x == 0) {
                const uint32_t* cnt = p.sync + 32 * s;   // arrivals at stage s - 1
                const uint64_t t0 = tc::globaltimer_ns();
                for (uint32_t i = 0;; i++) {
                    if (ld_relaxed_gpu(cnt) >= gridDim.x) {
                        // acquire: the arrivals' released writes (stage s-1's outputs) are visible from here
                        asm volatile("fence.acq_rel.gpu;" ::: "memory");
                        break;
                    }
                    if ((i & 63u) == 63u && ld_relaxed_gpu(p.sync)) { *abort_cta = 1; break; }
                    if ((i & 63u) == 63u) {
                        if (tc::wait_expired(t0, tc::kWaitLimitNs, i >> 6, 64)) {
                            q4_set_status(p.status, Q4_ERR_TIMEOUT);
                            atomicExch(p.sync, 1u);
                            *abort_cta = 1;
                            break;
                        }
                    }
                }
            }
            compute_bar();
            if (*abort_cta) {
                if (threadIdx.x == 0) q4_set_status(p.status, Q4_ERR_TIMEOUT);
                return;
            }
        }
        int a, b;
        cta_range(p, S, a, b);
        const int k = S.k, ks = S.ksplit, teams = kCW / ks;
        const int team = warp / ks, kq = warp % ks;
        const int64_t rowbytes = k / 2;
        const int ng = k / ng_of, C = k / 32;
        const int wbytes = S.rps * (int)rowbytes, sbytes = S.rps * ng * 2;
        const int L = kq * 32 + lane;                // the lane's 64-value block of k
        const int c0 = 2 * L;
        const bool cvalid = c0 < C;
        const int gl = L * 64 / ng_of;
        int cur = -1;                                // problem whose x is staged
        uint4 X[1][8];
        float inv_xs[1];
        int xsum[1];
        for (int r = a; r < b; it++) {
            const Chunk c = chunk_at(p, S, r, a, b);
            const ChainProblem& P = p.prob[c.pi];
            if (c.pi != cur) {
                if (cur >= 0) compute_bar();         // every warp is done with the previous x
                stage_x(P, k, xs, xinv, p.status);
                compute_bar();
                cur = c.pi;
                // (a warp with no rows in this stage's range skips its share of x: 4 KB of shared-memory
                // reads per warp and problem)
                const bool xwarp = cvalid && team < b - a;
#pragma unroll
                for (int i = 0; i < 8; i++) X[0][i] = xwarp ? xs[(L << 3) + (i ^ (L & 7))] : make_uint4(0, 0, 0, 0);
                inv_xs[0] = xwarp ? xinv[L] : 0.0f;
                int s4[4] = {0, 0, 0, 0};
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    s4[0] = dp2a_lo(X[0][i].x, 0x01010101u, s4[0]);
                    s4[1] = dp2a_lo(X[0][i].y, 0x01010101u, s4[1]);
                    s4[2] = dp2a_lo(X[0][i].z, 0x01010101u, s4[2]);
                    s4[3] = dp2a_lo(X[0][i].w, 0x01010101u, s4[3]);
                }
                xsum[0] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            const int slot = it % p.nslots;
            // (after an expired wait the warp skips its rows but keeps to the barriers below, so that every
            // compute warp leaves together at the end of the stage; the abort word stops the other CTAs)
            const bool have = !*abort_cta && tc::mbar_wait(&full[slot], (it / p.nslots) & 1, p.status, abort_cta);
            if (!have) {   // (the producer may have given up first: the other CTAs must learn of it too)
                *abort_cta = 1;
                atomicExch(p.sync, 1u);
            }
            const uint8_t* sb = ring + slot * p.slot_bytes;
            for (int ra = team; have && ra < c.rows; ra += 2 * teams) {
                const int rb = ra + teams;
                const bool hasb = rb < c.rows;
                float pa[1] = {0.0f}, pb[1] = {0.0f};
                if (cvalid) {
                    const __half* sa = S.bulk_scales ? reinterpret_cast<const __half*>(sb + wbytes) + ra * ng
                                                     : P.scales + (int64_t)(c.lr + ra) * ng;
                    const __half* za = S.bulk_scales ? reinterpret_cast<const __half*>(sb + wbytes + sbytes) + ra * ng
                                                     : P.zeros + (int64_t)(c.lr + ra) * ng;
                    row_dot<SYM, 1>(sb + ra * rowbytes + c0 * 16, sa, za, gl, X, inv_xs, xsum, pa);
                    if (hasb) {
                        const int d = (rb - ra) * ng;
                        row_dot<SYM, 1>(sb + rb * rowbytes + c0 * 16, sa + d, SYM ? za : za + d, gl, X, inv_xs, xsum, pb);
                    }
                }
                // lanes 0-15 end with row a, lanes 16-31 with row b
                const bool hi = lane & 16;
                float v = hi ? pb[0] : pa[0];
                v += __shfl_xor_sync(0xffffffffu, hi ? pa[0] : pb[0], 16);
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if ((lane & 15) == 0 && (!hi || hasb)) {
                    const int rr = hi ? rb : ra;
                    if (ks == 1) store_y(P.y, c.lr + rr, v, p.out_bf16, P.n, p.status);
                    else red[(c.cr + rr) * ks + kq] = v;
                }
            }
            __syncwarp();
            if (lane == 0) tc::sts_publish(&consumed[warp], it + 1);   // this warp is done with the slot
            r += c.rows;
        }
        compute_bar();   // every row of the stage is reduced (and, ksplit 1, stored)
        if (*abort_cta) return;   // read by every compute thread after the same barrier: a uniform exit
        if (ks > 1) {
            for (int i = threadIdx.x; i < b - a; i += kCT) {
                float v = 0.0f;
                for (int t = 0; t < ks; t++) v += red[i * ks + t];
                const Chunk c = chunk_at(p, S, a + i, a, b);
                store_y(p.prob[c.pi].y, c.lr, v, p.out_bf16, p.prob[c.pi].n, p.status);
            }
            compute_bar();
        }
        // publish: this CTA's outputs of stage s are written (the barrier above orders every compute
        // thread's stores before thread 0's release, which carries them to the other CTAs' acquire)
        if (threadIdx.x == 0) {
            if (s < p.nstages - 1) {
                asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.sync + 32 * (1 + s)) : "memory");
            } else {
                uint32_t old;
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.sync + 32 * (1 + s)) : "memory");
                if (old == gridDim.x - 1) {
                    // the last arrival of the last stage: every CTA is past every wait; leave the counters zero
                    for (int i = 1; i <= p.nstages; i++) p.sync[32 * i] = 0u;
                }
            }
        }
    }
}

}  // namespace

// Host entry (api.cu validates the arguments): count problems in n_stages stages, stage_begin[s] ..
// stage_begin[s+1]-1 the problems of stage s.
int q4_gemv_w4a16_chain_launch(int n_stages, const int32_t* stage_begin, const uint16_t* const* x,
                               const float* const* g, const float* const* u, const q4_weight* w, void* const* y,
                               int32_t out_dtype, uint32_t* sync, int32_t* dev_status, cudaStream_t stream)
{
    if (n_stages < 1 || n_stages > kMaxStages) return Q4_ERR_UNSUPPORTED;
    const int count = stage_begin[n_stages];
    if (count > kMaxProblems) return Q4_ERR_UNSUPPORTED;
    const int group = w[0].group, sym = w[0].symmetric;
    ChainParams P{};
    P.nstages = n_stages;
    P.group = group;
    P.out_bf16 = out_dtype == Q4_OUT_BF16;
    P.sync = sync;
    P.status = dev_status;
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = q4_num_sms();
    int slot_bytes = 0, kmax = 0, redmax = 0;
    for (int s = 0; s < n_stages; s++) {
        ChainStage& S = P.st[s];
        S.p0 = stage_begin[s];
        S.np = stage_begin[s + 1] - stage_begin[s];
        if (S.np < 1 || S.np > kMaxStageProblems) return Q4_ERR_UNSUPPORTED;
        S.k = w[S.p0].k;
        int rows = 0;
        for (int i = S.p0; i < S.p0 + S.np; i++) {
            if (w[i].k != S.k || w[i].group != group || w[i].symmetric != sym) return Q4_ERR_UNSUPPORTED;
            ChainProblem& Q = P.prob[i];
            Q.x = x ? x[i] : nullptr;
            Q.g = g ? g[i] : nullptr;
            Q.u = u ? u[i] : nullptr;
            Q.packed = w[i].packed;
            Q.scales = reinterpret_cast<const __half*>(w[i].scales);
            Q.zeros = reinterpret_cast<const __half*>(w[i].zeros);
            Q.y = y[i];
            Q.n = w[i].n;
            Q.row0 = rows;
            rows += w[i].n;
        }
        if (S.k % 64 || S.k > kMaxK) return Q4_ERR_UNSUPPORTED;
        S.rows = rows;
        // CTAs per problem in proportion to its rows (at least one each), rows per CTA within the problem
        {
            int nc[kMaxStageProblems], tot = 0;
            for (int i = 0; i < S.np; i++) {
                nc[i] = std::max(1, (int)((int64_t)w[S.p0 + i].n * grid / rows));
                tot += nc[i];
            }
            while (tot > grid) {   // (only with many tiny problems) take from the problem with the most CTAs
                int j = 0;
                for (int i = 1; i < S.np; i++) if (nc[i] > nc[j]) j = i;
                nc[j]--; tot--;
            }
            while (tot < grid) {   // give the rest to the problem with the most rows per CTA
                int j = 0;
                for (int i = 1; i < S.np; i++)
                    if ((int64_t)w[S.p0 + i].n * nc[j] > (int64_t)w[S.p0 + j].n * nc[i]) j = i;
                nc[j]++; tot++;
            }
            int c0 = 0;
            for (int i = 0; i < S.np; i++) {
                ChainProblem& Q = P.prob[S.p0 + i];
                Q.cta0 = c0;
                Q.ncta = nc[i];
                Q.rpc = (Q.n + nc[i] - 1) / nc[i];
                c0 += nc[i];
            }
        }
        int ks = 1;
        while (ks * 2048 < S.k) ks *= 2;
        S.ksplit = ks;
        const int rowbytes = S.k / 2, ng = S.k / group;
        S.rps = std::max(1, kChunkW / rowbytes);
        int rpc_max = 1;
        for (int i = S.p0; i < S.p0 + S.np; i++) rpc_max = std::max(rpc_max, P.prob[i].rpc);
        if (ks > 1 && rpc_max * ks > kRedFloats) return Q4_ERR_UNSUPPORTED;
        S.bulk_scales = (ng * 2) % 16 == 0;
        const int sb = S.rps * rowbytes + (S.bulk_scales ? S.rps * ng * 2 * (sym ? 1 : 2) : 0);
        slot_bytes = std::max(slot_bytes, sb);
        kmax = std::max(kmax, S.k);
        redmax = std::max(redmax, ks > 1 ? rpc_max * ks : 0);
    }
    slot_bytes = (slot_bytes + 127) & ~127;
    // shared memory: x (int16) | per-block inverse scales | split-k partials | barriers | ring
    P.xs_off = 0;
    P.xinv_off = kmax * 2;
    P.red_off = P.xinv_off + (kmax / 64) * 4;
    P.bar_off = (P.red_off + redmax * 4 + 127) & ~127;
    const int bar_bytes = 8 * 8 + 4 * kCW + 16;   // up to 8 slots' full barriers, consumed counters, abort flag
    P.ring_off = (P.bar_off + bar_bytes + 127) & ~127;
    const int avail = 227 * 1024 - P.ring_off;
    P.nslots = std::min(8, avail / slot_bytes);
    P.slot_bytes = slot_bytes;
    if (P.nslots < 2) return Q4_ERR_UNSUPPORTED;
    const size_t smem = (size_t)P.ring_off + (size_t)P.nslots * slot_bytes;

    auto kern = sym ? w4a16_gemv_chain_kernel<true> : w4a16_gemv_chain_kernel<false>;
    static uint64_t opted[2] = {0, 0};
    const uint64_t bit = 1ull << (dev & 63);
    if (!(opted[sym ? 1 : 0] & bit)) {
        if (const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024))
            return q4_cuda_status(e);
        opted[sym ? 1 : 0] |= bit;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the stage waits need that
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return q4_cuda_status(cudaLaunchKernelEx(&cfg, kern, P));
}
