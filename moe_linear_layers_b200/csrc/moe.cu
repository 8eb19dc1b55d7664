// Top-k routed MoE layer of SwiGLU experts with INT4 weights (moe_q4_forward).
//
// Sources: "大模型之Dense、MoE与量化" 混合专家架构 MoE (a Linear router scores the experts, a few are chosen,
// their outputs are recombined in proportion); "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §3.2
// (router output through softmax, kept in high precision) and §1 (dispatch and merge cost extra);
// "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" MoE架构设计 (experts are small FFNs behind a gating
// network, SwiGLU as in the base model).
//
// Launch sequence (one stream, no host synchronisation):
//   1. route     fp32 logits in a pinned reduction order, top-k by (logit desc, id asc), softmax
//                weights over the chosen logits, per-chunk expert histograms (16 tokens per chunk);
//   2. scan      expert counts and offsets, per-chunk bases (a column scan of the histograms), and the
//                tile counts of both grouped GEMMs;
//   3. scatter   stable counting sort: every (token, slot) pair gets its row in the permuted order
//                (expert, token ascending), and the token's activation row is gathered there;
//   4. gate/up   grouped tcgen05 GEMM over (expert, token tile, 64 intermediate rows) tiles with the
//                SwiGLU epilogue, h as bf16 hi/lo pairs (h to about 2^-17 of its magnitude);
//   5. down      grouped tcgen05 GEMM over (expert, token tile, 128 hidden rows) tiles whose epilogue
//                adds w[t][j] * out into the fp32 output (float atomics: the sum order is not fixed);
//   6. (bf16 output) a conversion pass.
#include <mutex>

#include "tc_host.cuh"

namespace {

constexpr int kRouteTok = 16;           // tokens per route CTA (= one histogram chunk)
constexpr int kRouteWarps = 8;
constexpr int kRouteKC = 64;            // K columns staged per step
constexpr int kMaxTopk = 16;
// (token, slot) pairs of one call: their positions t * topk + j are int32
constexpr int64_t kMaxPairs = INT32_MAX;

// ---------------------------------------------------------------------------------------------- //
// 1. route
// ---------------------------------------------------------------------------------------------- //
// A CTA scores one chunk of 16 tokens against 64 experts at a time.  Warp w owns 8 tokens x 16 experts
// (128 register partials per lane, so each staged value feeds 8 or 16 FMAs); lane l owns the
// k = l (mod 32) partial sums, each an fma chain with k ascending (two experts per packed
// fma.rn.f32x2, which rounds each half exactly like fmaf); the 32 partials of a logit are combined by
// the xor butterfly s = 16, 8, 4, 2, 1 -- computed as a transposing reduction (at each level a lane
// keeps half of its values and adds its partner's copy of them, 124 shuffles for 128 logits instead of
// 640), which adds exactly the same pairs as the butterfly.  This is the pinned order the oracle
// reproduces bit for bit.  A producer warp streams 64-column tiles of Wr (fp32) and x (bf16) through a
// 4-stage TMA ring.
constexpr int kRouteStages = 4;
constexpr int kRouteThreads = (kRouteWarps + 2) * 32;   // + producer warp + ring-slot watcher warp
constexpr int kRouteWTile = 64 * kRouteKC * 4;       // 64 experts x 64 columns, fp32
constexpr int kRouteXTile = kRouteTok * kRouteKC * 2;  // 16 tokens x 64 columns, bf16

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t pack2(float lo, float hi)
{
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}

__global__ void __launch_bounds__(kRouteThreads, 1)
moe_route_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, int T, int H,
                 const float* __restrict__ bias, int E, int topk, int32_t* __restrict__ ids, float* __restrict__ wts,
                 int32_t* __restrict__ hist, int32_t* status)
{
    extern __shared__ __align__(128) uint8_t rsm[];
    float* wst = reinterpret_cast<float*>(rsm);                                       // [stage][64][KC]
    uint16_t* xst = reinterpret_cast<uint16_t*>(rsm + kRouteStages * kRouteWTile);    // [stage][16][KC]
    __shared__ float logits[kRouteTok][tcg::kMaxExperts];
    __shared__ int hcount[tcg::kMaxExperts];
    __shared__ uint64_t full[kRouteStages], empty[kRouteStages];
    __shared__ uint32_t slot_free;   // ring stages released so far (published by the watcher)
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kRouteTok;
    const int nk = H / kRouteKC;
    const int neb = (E + 63) / 64;
    const int nsteps = neb * nk;          // (expert block, k chunk) pairs in order

    if (threadIdx.x == 0) {
        for (int i = 0; i < kRouteStages; i++) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], kRouteWarps); }
        slot_free = 0;
        tc::fence_mbar_init();
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) hcount[e] = 0;
    __syncthreads();

    if (warp == kRouteWarps + 1) {
        // ------------------------------------------------------------------ ring-slot watcher: waits for each
        // stage's slot to be released and publishes the count (the producer, which issues the copies, must
        // not wait on an mbarrier: such a wait also waits for the thread's own bulk copies in flight)
        if (lane == 0)
            for (int st = 0; st < nsteps; st++) {
                if (!tc::mbar_wait(&empty[st % kRouteStages], (st / kRouteStages) & 1, status, nullptr)) break;
                tc::sts_publish(&slot_free, st + 1);
            }
    } else if (warp == kRouteWarps) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            for (int st = 0; st < nsteps; st++) {
                const int s = st % kRouteStages;
                if (st >= kRouteStages) {
                    if (!tc::poll_counters<1>(&slot_free, st - kRouteStages + 1, status, nullptr)) break;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                const int eb = st / nk, kc = st % nk;
                tc::mbar_arrive_expect_tx(&full[s], kRouteWTile + kRouteXTile);
                tc::tma_load_2d(wst + s * (kRouteWTile / 4), &tm_w, &full[s], kc * kRouteKC, eb * 64);
                tc::tma_load_2d(xst + s * (kRouteXTile / 2), &tm_x, &full[s], kc * kRouteKC, t0);
            }
        }
    } else {
        // ------------------------------------------------------------------ 8 compute warps
        const int tg = warp / 4, eg = warp % 4;   // tokens 8*tg.., experts 16*eg.. of the 64-block
        for (int eb = 0; eb < neb; eb++) {
            uint64_t acc[8][8];   // [token][expert pair]
#pragma unroll
            for (int a = 0; a < 8; a++)
#pragma unroll
                for (int b = 0; b < 8; b++) acc[a][b] = 0;
            for (int kc = 0; kc < nk; kc++) {
                const int st = eb * nk + kc, s = st % kRouteStages;
                if (!tc::mbar_wait(&full[s], (st / kRouteStages) & 1, status, nullptr)) break;
                const float* wt = wst + s * (kRouteWTile / 4);
                const uint16_t* xt = xst + s * (kRouteXTile / 2);
#pragma unroll
                for (int i = 0; i < kRouteKC / 32; i++) {
                    const int c = lane + 32 * i;
                    uint64_t wv[8];
#pragma unroll
                    for (int b = 0; b < 8; b++)
                        wv[b] = pack2(wt[(16 * eg + 2 * b) * kRouteKC + c], wt[(16 * eg + 2 * b + 1) * kRouteKC + c]);
#pragma unroll
                    for (int a = 0; a < 8; a++) {
                        const float f = bf16_bits_to_float(xt[(8 * tg + a) * kRouteKC + c]);
                        const uint64_t xv = pack2(f, f);
#pragma unroll
                        for (int b = 0; b < 8; b++) acc[a][b] = ffma2(xv, wv[b], acc[a][b]);
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&empty[s]);
            }
            // transposing butterfly over the 128 partials j = 16 * token + expert (packed in expert pairs):
            // at the level on lane bit q the lane keeps the half of its values selected by that bit and adds
            // its partner's copy of them; lane l ends with j = 4l .. 4l+3 in acc[0][0], acc[0][1]
            auto level = [&](uint64_t& x, uint64_t& y, int bit) {   // x: lower index, y: upper index
                const bool upper = (lane >> bit) & 1;
                const uint64_t keep = upper ? y : x, send = upper ? x : y;
                const uint32_t r0 = __shfl_xor_sync(0xffffffffu, (uint32_t)send, 1 << bit);
                const uint32_t r1 = __shfl_xor_sync(0xffffffffu, (uint32_t)(send >> 32), 1 << bit);
                x = pack2(__uint_as_float((uint32_t)keep) + __uint_as_float(r0),
                          __uint_as_float((uint32_t)(keep >> 32)) + __uint_as_float(r1));
            };
#pragma unroll
            for (int a = 0; a < 4; a++)
#pragma unroll
                for (int b = 0; b < 8; b++) level(acc[a][b], acc[a + 4][b], 4);   // j, j + 64
#pragma unroll
            for (int a = 0; a < 2; a++)
#pragma unroll
                for (int b = 0; b < 8; b++) level(acc[a][b], acc[a + 2][b], 3);   // j, j + 32
#pragma unroll
            for (int b = 0; b < 8; b++) level(acc[0][b], acc[1][b], 2);            // j, j + 16
#pragma unroll
            for (int b = 0; b < 4; b++) level(acc[0][b], acc[0][b + 4], 1);        // j, j + 8
#pragma unroll
            for (int b = 0; b < 2; b++) level(acc[0][b], acc[0][b + 2], 0);        // j, j + 4
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int j = 4 * lane + q;
                const int e = eb * 64 + 16 * eg + (j & 15);
                const float lv = __uint_as_float((uint32_t)(acc[0][q >> 1] >> (32 * (q & 1))));
                if (e < E) logits[8 * tg + (j >> 4)][e] = bias ? lv + bias[e] : lv;
            }
        }
    }
    __syncthreads();

    // top-k per token (warp w handles tokens w, w + 10 of the chunk)
    for (int tt = warp; tt < kRouteTok; tt += kRouteWarps + 2) {
        const int t = t0 + tt;
        if (t >= T) break;
        constexpr int PER = tcg::kMaxExperts / 32;
        float v[PER];
        bool finite = true;
#pragma unroll
        for (int q = 0; q < PER; q++) {
            const int e = lane + 32 * q;
            v[q] = e < E ? logits[tt][e] : -INFINITY;
            if (e < E) finite &= isfinite(v[q]);
        }
        if (!__all_sync(0xffffffffu, finite)) {
            if (lane == 0) q4_set_status(status, Q4_ERR_NONFINITE);
        }
        float sel_l[kMaxTopk];
        int sel_e[kMaxTopk];
        for (int j = 0; j < topk; j++) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int q = 0; q < PER; q++) {
                const int e = lane + 32 * q;
                if (e < E && (v[q] > bv || (v[q] == bv && e < be))) { bv = v[q]; be = e; }
            }
#pragma unroll
            for (int sft = 16; sft >= 1; sft >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, sft);
                const int oe = __shfl_xor_sync(0xffffffffu, be, sft);
                if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
            }
            sel_l[j] = bv;
            sel_e[j] = be;
#pragma unroll
            for (int q = 0; q < PER; q++)
                if (lane + 32 * q == be) v[q] = -INFINITY;
        }
        if (lane == 0) {
            float den = 0.0f;
            for (int j = 0; j < topk; j++) den += expf(sel_l[j] - sel_l[0]);
            for (int j = 0; j < topk; j++) {
                ids[(int64_t)t * topk + j] = sel_e[j];
                wts[(int64_t)t * topk + j] = expf(sel_l[j] - sel_l[0]) / den;
                atomicAdd(&hcount[sel_e[j]], 1);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = hcount[e];
}

// ---------------------------------------------------------------------------------------------- //
// 2. scan (one CTA of 1024 threads: P = 1024 / E threads per expert, each over a range of chunks)
// ---------------------------------------------------------------------------------------------- //
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) moe_scan_kernel(const int32_t* __restrict__ hist, int nchunks, int E,
                                                               int I, int H, int32_t* __restrict__ chunk_base,
                                                               int32_t* __restrict__ offsets, int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ tiles_gu, int32_t* __restrict__ tiles_dn)
{
    __shared__ int part[kScanThreads];
    __shared__ int cnt[tcg::kMaxExperts], off[tcg::kMaxExperts];
    const int P = kScanThreads / E;                  // >= 4 (E <= 256)
    const int e = threadIdx.x % E, pi = threadIdx.x / E;
    const int per = (nchunks + P - 1) / P;
    const int c0 = min(nchunks, pi * per), c1 = min(nchunks, c0 + per);
    int sum = 0;
    if (pi < P)
        for (int c = c0; c < c1; c++) sum += hist[(int64_t)c * E + e];   // coalesced across e
    part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x < E) {   // expert totals
        int cq = 0;
        for (int u = 0; u < P; u++) cq += part[u * E + threadIdx.x];
        cnt[threadIdx.x] = cq;
        if (counts) counts[threadIdx.x] = cq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int o = 0, tg = 0, td = 0;
        for (int q = 0; q < E; q++) {
            const int cq = cnt[q];
            off[q] = o;
            offsets[q] = o;
            tiles_gu[q] = tg;
            tiles_dn[q] = td;
            const int mt = (cq + tcg::BN - 1) / tcg::BN;
            o += cq;
            tg += mt * (I / 64);
            td += mt * (H / tcg::BM);
        }
        offsets[E] = o;
        tiles_gu[E] = tg;
        tiles_dn[E] = td;
    }
    __syncthreads();
    if (pi < P) {
        int run = off[e];
        for (int u = 0; u < pi; u++) run += part[u * E + e];
        for (int c = c0; c < c1; c++) {
            chunk_base[(int64_t)c * E + e] = run;
            run += hist[(int64_t)c * E + e];
        }
    }
}

// ---------------------------------------------------------------------------------------------- //
// 3. scatter + gather (one CTA per chunk of 16 tokens).  Rows are row_bytes long (bf16 activations,
//    or their int8 codes, whose per-token scales tok_scale then follow them into row_scale).
// ---------------------------------------------------------------------------------------------- //
__global__ void __launch_bounds__(256) moe_scatter_kernel(const uint8_t* __restrict__ x, int T, int row_bytes, int E,
                                                          int topk, const int32_t* __restrict__ ids,
                                                          const float* __restrict__ wts,
                                                          const int32_t* __restrict__ chunk_base,
                                                          int32_t* __restrict__ perm, int32_t* __restrict__ row_tok,
                                                          float* __restrict__ row_w, uint8_t* __restrict__ xperm,
                                                          const float* __restrict__ tok_scale,
                                                          float* __restrict__ row_scale,
                                                          int32_t* __restrict__ pair_pos = nullptr,
                                                          int32_t* __restrict__ row_exp = nullptr,
                                                          int32_t* status = nullptr)
{
    const int64_t P = (int64_t)T * topk;   // permuted rows
    __shared__ int pos[kRouteTok * kMaxTopk];
    __shared__ int cid[kRouteTok * kMaxTopk];   // the chunk's expert ids, token-major
    const int c = blockIdx.x;
    const int t0 = c * kRouteTok;
    const int npairs = min(kRouteTok, T - t0) * topk;
    for (int q = threadIdx.x; q < npairs; q += blockDim.x) cid[q] = ids[(int64_t)t0 * topk + q];
    __syncthreads();
    for (int q = threadIdx.x; q < npairs; q += blockDim.x) {
        const int tl = q / topk, j = q % topk;
        const int e = cid[q];
        int rank = 0;  // earlier tokens of this chunk that chose the same expert (a token picks an expert once)
        for (int u = 0; u < tl * topk; u++) rank += cid[u] == e;
        const int p = chunk_base[(int64_t)c * E + e] + rank;
        pos[q] = q4_in_bounds(p, P, status) ? p : -1;   // (debug build: a position outside the rows is not used)
        if (pos[q] < 0) continue;
        perm[p] = (t0 + tl) * topk + j;
        row_tok[p] = t0 + tl;
        row_w[p] = wts[(int64_t)(t0 + tl) * topk + j];
        if (tok_scale) row_scale[p] = tok_scale[t0 + tl];
        if (pair_pos) pair_pos[(int64_t)t0 * topk + q] = p;   // the inverse permutation
        if (row_exp) row_exp[p] = e;
    }
    __syncthreads();
    if (!xperm) return;
    // gather: a warp takes a token, reads its row once (eight 16-byte loads in flight per lane) and writes
    // it to the permuted rows of all its topk slots
    const int vec = row_bytes / 16;  // 16-byte units per row
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31, nwarps = blockDim.x / 32;
    const int ntok = npairs / topk;
    for (int tl = warp; tl < ntok; tl += nwarps) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)(t0 + tl) * row_bytes);
        int u = lane;
        for (; u + 7 * 32 < vec; u += 8 * 32) {
            uint4 r[8];
#pragma unroll
            for (int j = 0; j < 8; j++) r[j] = __ldg(src + u + 32 * j);
            for (int k = 0; k < topk; k++) {
                if (pos[tl * topk + k] < 0) continue;
                uint4* dst = reinterpret_cast<uint4*>(xperm + (int64_t)pos[tl * topk + k] * row_bytes);
#pragma unroll
                for (int j = 0; j < 8; j++) dst[u + 32 * j] = r[j];
            }
        }
        for (; u < vec; u += 32) {
            const uint4 r = __ldg(src + u);
            for (int k = 0; k < topk; k++)
                if (pos[tl * topk + k] >= 0) reinterpret_cast<uint4*>(xperm + (int64_t)pos[tl * topk + k] * row_bytes)[u] = r;
        }
    }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ a, __nv_bfloat16* __restrict__ b, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        b[i] = __float2bfloat16_rn(a[i]);
}

struct Workspace {
    uint16_t* xperm;          // permuted activations: bf16 rows, or int8 codes (W4A8 gate/up)
    __nv_bfloat16* h;         // [P][I/64][hi 64 | lo 64]
    // shared expert (I_shared > 0): its h, and the one-expert bookkeeping the grouped GEMMs read
    __nv_bfloat16* h_s;
    int32_t *offsets_s, *tiles_gu_s, *tiles_dn_s, *row_tok_s;
    float* row_w_s;
    float* y32;
    int32_t *ids, *perm, *offsets, *counts, *hist, *chunk_base, *tiles_gu, *tiles_dn, *row_tok;
    float *wts, *row_w;
    // INT8 activations (W4A8 expert GEMMs): the tokens' codes and scales, the permuted rows' scales,
    // and the codes and scales of h
    int8_t *xq_tok, *hq;
    float *sa_tok, *sa_row, *sh_row;
    size_t bytes;
};

inline size_t al(size_t v) { return (v + 255) & ~(size_t)255; }

// The shared expert is a one-expert grouped GEMM over every token in order, with routing weight 1.
__global__ void moe_shared_setup_kernel(int T, int H, int I_s, int32_t* __restrict__ offsets,
                                        int32_t* __restrict__ tiles_gu, int32_t* __restrict__ tiles_dn,
                                        int32_t* __restrict__ row_tok, float* __restrict__ row_w)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) {
        const int mt = (T + tcg::BN - 1) / tcg::BN;
        offsets[0] = 0;
        offsets[1] = T;
        tiles_gu[0] = 0;
        tiles_gu[1] = mt * (I_s / 64);
        tiles_dn[0] = 0;
        tiles_dn[1] = mt * (H / tcg::BM);
    }
    if (i < T) {
        row_tok[i] = i;
        row_w[i] = 1.0f;
    }
}

// The routing outputs of a call without tokens: offsets [E + 1] and counts [E] all 0 (each nullable).
int zero_routing(int32_t* offsets, int32_t* counts, int E, cudaStream_t s)
{
    if (offsets)
        if (const cudaError_t e = cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s)) return q4_cuda_status(e);
    if (counts)
        if (const cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), s)) return q4_cuda_status(e);
    return Q4_OK;
}

Workspace carve(void* base, int T, int H, int I, int E, int topk, int I_s = 0, int a8_mask = 0)
{
    Workspace w = {};
    const size_t P = (size_t)T * topk;
    const size_t nch = (size_t)(T + kRouteTok - 1) / kRouteTok;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) { uint8_t* q = p ? p + o : nullptr; o += al(bytes); return q; };
    w.xperm = reinterpret_cast<uint16_t*>(take(P * H * 2));
    w.h = reinterpret_cast<__nv_bfloat16*>(take(P * I * 4));
    w.y32 = reinterpret_cast<float*>(take((size_t)T * H * 4));
    w.ids = reinterpret_cast<int32_t*>(take(P * 4));
    w.wts = reinterpret_cast<float*>(take(P * 4));
    w.perm = reinterpret_cast<int32_t*>(take(P * 4));
    w.row_tok = reinterpret_cast<int32_t*>(take(P * 4));
    w.row_w = reinterpret_cast<float*>(take(P * 4));
    w.offsets = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    w.counts = reinterpret_cast<int32_t*>(take(E * 4));
    w.hist = reinterpret_cast<int32_t*>(take(nch * E * 4));
    w.chunk_base = reinterpret_cast<int32_t*>(take(nch * E * 4));
    w.tiles_gu = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    w.tiles_dn = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    if (I_s > 0) {
        w.h_s = reinterpret_cast<__nv_bfloat16*>(take((size_t)T * I_s * 4));
        w.offsets_s = reinterpret_cast<int32_t*>(take(2 * 4));
        w.tiles_gu_s = reinterpret_cast<int32_t*>(take(2 * 4));
        w.tiles_dn_s = reinterpret_cast<int32_t*>(take(2 * 4));
        w.row_tok_s = reinterpret_cast<int32_t*>(take((size_t)T * 4));
        w.row_w_s = reinterpret_cast<float*>(take((size_t)T * 4));
    }
    if (a8_mask & 1) {
        w.xq_tok = reinterpret_cast<int8_t*>(take((size_t)T * H));
        w.sa_tok = reinterpret_cast<float*>(take((size_t)T * 4));
        w.sa_row = reinterpret_cast<float*>(take(P * 4));
    }
    if (a8_mask & 2) {
        w.hq = reinterpret_cast<int8_t*>(take(P * I));
        w.sh_row = reinterpret_cast<float*>(take(P * 4));
    }
    w.bytes = o;
    return w;
}

template <int G, bool SYM>
int launch_experts(const Workspace& ws, const q4_weight* ex, int T, int H, int I, int E, int topk, float* y32,
                   int32_t* status, cudaStream_t s, int a8_mask = 0)
{
    using namespace tcg;
    const int P = T * topk;
    const int sms = q4_num_sms();
    int rc;
    if (a8_mask & 1) {   // gate/up on the permuted rows' int8 codes
        rc = q4_moe_gateup_a8(reinterpret_cast<const int8_t*>(ws.xperm), ws.sa_row, &ex[0], &ex[1], P, H, I, E,
                              ws.offsets, ws.tiles_gu, ws.h, (a8_mask & 2) != 0, status, s);
    } else {
        CUtensorMap mx, mg, mu;
        if (!make_act_map(&mx, ws.xperm, H, P, 2) || !make_packed_map(&mg, ex[0].packed, H, (uint64_t)E * I, 64) ||
            !make_packed_map(&mu, ex[1].packed, H, (uint64_t)E * I, 64))
            return Q4_ERR_CUDA;
        Args a = {};
        a.M = P;
        a.N = I;
        a.K = H;
        a.scales_a = reinterpret_cast<const __half*>(ex[0].scales);
        a.zeros_a = reinterpret_cast<const __half*>(ex[0].zeros);
        a.scales_b = reinterpret_cast<const __half*>(ex[1].scales);
        a.zeros_b = reinterpret_cast<const __half*>(ex[1].zeros);
        a.status = status;
        a.expert_tiles = ws.tiles_gu;
        a.offsets = ws.offsets;
        a.h = ws.h;
        a.h_f16 = (a8_mask & 2) != 0;   // an INT8 down projection quantizes h as an fp16 activation
        a.E = E;
        a.topk = topk;
        rc = launch<false, G, SYM, Mode::GateUp>(mx, mg, mu, a, sms, s);
    }
    if (rc) return rc;
    if (a8_mask & 2) {   // h (fp16) -> per-row int8 codes, then down on them
        if ((rc = q4_act_quant_rows(reinterpret_cast<const uint16_t*>(ws.h), true, P, I, ws.hq, ws.sh_row, status, s)))
            return rc;
        return q4_moe_down_a8(ws.hq, ws.sh_row, &ex[2], P, H, I, E, ws.offsets, ws.tiles_dn, ws.row_tok, ws.row_w,
                              y32, T, status, s);
    }
    CUtensorMap mh, md;
    if (!make_act_map(&mh, ws.h, 2 * (uint64_t)I, P, 2, 4) || !make_packed_map(&md, ex[2].packed, I, (uint64_t)E * H, BM))
        return Q4_ERR_CUDA;
    Args d = {};
    d.M = P;
    d.N = H;
    d.K = I;
    d.scales_a = reinterpret_cast<const __half*>(ex[2].scales);
    d.zeros_a = reinterpret_cast<const __half*>(ex[2].zeros);
    d.y = y32;
    d.status = status;
    d.expert_tiles = ws.tiles_dn;
    d.offsets = ws.offsets;
    d.row_tok = ws.row_tok;
    d.row_w = ws.row_w;
    d.E = E;
    d.topk = topk;
    d.T = T;
    return launch<false, G, SYM, Mode::Down>(mh, md, md, d, sms, s);
}

// groups 32 and 256 are built for the 16-bit expert GEMMs only (the INT8 paths take 64 and 128)
int launch_experts_any(const Workspace& ws, const q4_weight* ex, int T, int H, int I, int E, int topk, float* y32,
                       int32_t* status, cudaStream_t s, int a8_mask)
{
    const bool sym = ex[0].symmetric != 0;
    switch (ex[0].group) {
    case 128:
        return sym ? launch_experts<128, true>(ws, ex, T, H, I, E, topk, y32, status, s, a8_mask)
                   : launch_experts<128, false>(ws, ex, T, H, I, E, topk, y32, status, s, a8_mask);
    case 64:
        return sym ? launch_experts<64, true>(ws, ex, T, H, I, E, topk, y32, status, s, a8_mask)
                   : launch_experts<64, false>(ws, ex, T, H, I, E, topk, y32, status, s, a8_mask);
    case 32:
        if (a8_mask) return Q4_ERR_UNSUPPORTED;
        return sym ? launch_experts<32, true>(ws, ex, T, H, I, E, topk, y32, status, s, 0)
                   : launch_experts<32, false>(ws, ex, T, H, I, E, topk, y32, status, s, 0);
    case 256:
        if (a8_mask) return Q4_ERR_UNSUPPORTED;
        return sym ? launch_experts<256, true>(ws, ex, T, H, I, E, topk, y32, status, s, 0)
                   : launch_experts<256, false>(ws, ex, T, H, I, E, topk, y32, status, s, 0);
    default:
        return Q4_ERR_UNSUPPORTED;
    }
}

}  // namespace

extern "C" size_t moe_q4_workspace_size(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk)
{
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0) return 0;
    return carve(nullptr, T, H, I, E, topk).bytes;
}

static int forward_impl(const uint16_t* x, int32_t T, int32_t H, const float* router_w, const float* router_bias,
                        int32_t E, int32_t topk, const q4_weight* experts, int32_t I, const q4_weight* shared,
                        int32_t I_shared, int a8_mask, void* y, int32_t out_dtype, int32_t* topk_ids, float* topk_w,
                        int32_t* perm, int32_t* offsets, int32_t* expert_counts, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream, int n_classes = 1,
                        const int32_t* class_begin = nullptr, bool expert_range = false);

extern "C" int moe_q4_forward(const uint16_t* x, int32_t T, int32_t H, const float* router_w, const float* router_bias,
                              int32_t E, int32_t topk, const q4_weight* experts, int32_t I, void* y, int32_t out_dtype,
                              int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                              void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    return forward_impl(x, T, H, router_w, router_bias, E, topk, experts, I, nullptr, 0, 0, y, out_dtype, topk_ids,
                        topk_w, perm, offsets, expert_counts, workspace, workspace_bytes, dev_status, stream);
}

extern "C" size_t moe_q4_workspace_size_ex(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk, int32_t I_shared)
{
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0 || I_shared < 0) return 0;
    return carve(nullptr, T, H, I, E, topk, I_shared).bytes;
}

extern "C" size_t moe_q4_workspace_size_a8(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk, int32_t a8_mask)
{
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || topk <= 0 || a8_mask < 0 || a8_mask > 3) return 0;
    return carve(nullptr, T, H, I, E, topk, 0, a8_mask).bytes;
}

extern "C" int moe_q4_forward_ex(const uint16_t* x, int32_t T, int32_t H, const float* router_w,
                                 const float* router_bias, int32_t E, int32_t topk, const q4_weight* experts, int32_t I,
                                 const q4_weight* shared, int32_t I_shared, void* y, int32_t out_dtype,
                                 int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets,
                                 int32_t* expert_counts, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                 void* stream)
{
    return forward_impl(x, T, H, router_w, router_bias, E, topk, experts, I, shared, I_shared, 0, y, out_dtype,
                        topk_ids, topk_w, perm, offsets, expert_counts, workspace, workspace_bytes, dev_status, stream);
}

extern "C" int moe_q4_forward_a8(const uint16_t* x, int32_t T, int32_t H, const float* router_w,
                                 const float* router_bias, int32_t E, int32_t topk, const q4_weight* experts, int32_t I,
                                 int32_t a8_mask, void* y, int32_t out_dtype, int32_t* topk_ids, float* topk_w,
                                 int32_t* perm, int32_t* offsets, int32_t* expert_counts, void* workspace,
                                 size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (a8_mask < 0 || a8_mask > 3) return Q4_ERR_UNSUPPORTED;
    return forward_impl(x, T, H, router_w, router_bias, E, topk, experts, I, nullptr, 0, a8_mask, y, out_dtype,
                        topk_ids, topk_w, perm, offsets, expert_counts, workspace, workspace_bytes, dev_status, stream);
}

extern "C" int moe_q4_forward_classes(const uint16_t* x, int32_t T, int32_t H, const float* router_w,
                                      const float* router_bias, int32_t E, int32_t topk, int32_t n_classes,
                                      const int32_t* class_begin, const q4_weight* experts, int32_t I, void* y,
                                      int32_t out_dtype, int32_t* topk_ids, float* topk_w, int32_t* perm,
                                      int32_t* offsets, int32_t* expert_counts, void* workspace,
                                      size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (!class_begin) return Q4_ERR_NULL;
    return forward_impl(x, T, H, router_w, router_bias, E, topk, experts, I, nullptr, 0, 0, y, out_dtype, topk_ids,
                        topk_w, perm, offsets, expert_counts, workspace, workspace_bytes, dev_status, stream,
                        n_classes, class_begin);
}

extern "C" int moe_q4_forward_range(const uint16_t* x, int32_t T, int32_t H, const float* router_w,
                                    const float* router_bias, int32_t E, int32_t topk, int32_t e_begin, int32_t e_end,
                                    const q4_weight* experts, int32_t I, float* y, int32_t* topk_ids, float* topk_w,
                                    int32_t* perm, int32_t* offsets, int32_t* expert_counts, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (e_begin < 0 || e_end > E || e_begin >= e_end) return Q4_ERR_SHAPE;
    const int32_t range[2] = {e_begin, e_end};
    return forward_impl(x, T, H, router_w, router_bias, E, topk, experts, I, nullptr, 0, 0, y, Q4_OUT_F32, topk_ids,
                        topk_w, perm, offsets, expert_counts, workspace, workspace_bytes, dev_status, stream, 1, range,
                        true);
}

static int forward_impl(const uint16_t* x, int32_t T, int32_t H, const float* router_w, const float* router_bias,
                        int32_t E, int32_t topk, const q4_weight* experts, int32_t I, const q4_weight* shared,
                        int32_t I_shared, int a8_mask, void* y, int32_t out_dtype, int32_t* topk_ids, float* topk_w,
                        int32_t* perm, int32_t* offsets, int32_t* expert_counts, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream, int n_classes,
                        const int32_t* class_begin, bool expert_range)
{
    // x and y hold T rows: with no tokens they may be NULL
    if (!router_w || !experts || !workspace || (T > 0 && (!x || !y))) return Q4_ERR_NULL;
    if (T < 0 || H <= 0 || I <= 0 || E < 1 || E > tcg::kMaxExperts || topk < 1 || topk > kMaxTopk || topk > E)
        return Q4_ERR_SHAPE;
    if ((int64_t)T * topk > kMaxPairs) return Q4_ERR_SHAPE;
    if (H % 128 || I % 128) return Q4_ERR_UNSUPPORTED;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    // expert classes: experts [begin[c], begin[c+1]) share one stacked weight triple (one class = all)
    int32_t single[2] = {0, E};
    if (!class_begin) {
        n_classes = 1;
        class_begin = single;
    }
    // the classes cover every expert, or (expert_range) one contiguous range of them
    if (n_classes < 1 || n_classes > E) return Q4_ERR_SHAPE;
    if (expert_range ? (class_begin[0] < 0 || class_begin[n_classes] > E)
                     : (class_begin[0] != 0 || class_begin[n_classes] != E))
        return Q4_ERR_SHAPE;
    for (int c = 0; c < n_classes; c++) {
        const int Ec = class_begin[c + 1] - class_begin[c];
        if (Ec < 1) return Q4_ERR_SHAPE;
        const q4_weight* cw = experts + 3 * c;
        for (int i = 0; i < 3; i++) {
            const q4_weight& w = cw[i];
            if (!w.packed || !w.scales || (!w.symmetric && !w.zeros)) return Q4_ERR_NULL;
            if (w.group != cw[0].group || w.symmetric != cw[0].symmetric) return Q4_ERR_UNSUPPORTED;
            if (w.group <= 0 || w.k % w.group) return Q4_ERR_SHAPE;
            if (!q4_aligned16(w.packed) || !q4_aligned16(w.scales) || (!w.symmetric && !q4_aligned16(w.zeros)))
                return Q4_ERR_ALIGN;
        }
        if (cw[0].group != 64 && cw[0].group != 128 && !((cw[0].group == 32 || cw[0].group == 256) && a8_mask == 0))
            return Q4_ERR_UNSUPPORTED;
        if (cw[0].n != Ec * I || cw[0].k != H || cw[1].n != Ec * I || cw[1].k != H || cw[2].n != Ec * H || cw[2].k != I)
            return Q4_ERR_SHAPE;
    }
    const q4_weight& g = experts[0];
    if (shared) {   // the same group and symmetry as the routed experts
        if (I_shared <= 0) return Q4_ERR_SHAPE;
        if (I_shared % 128) return Q4_ERR_UNSUPPORTED;
        for (int i = 0; i < 3; i++) {
            const q4_weight& w = shared[i];
            if (!w.packed || !w.scales || (!w.symmetric && !w.zeros)) return Q4_ERR_NULL;
            if (w.group != g.group || w.symmetric != g.symmetric) return Q4_ERR_UNSUPPORTED;
            if (!q4_aligned16(w.packed) || !q4_aligned16(w.scales) || (!w.symmetric && !q4_aligned16(w.zeros)))
                return Q4_ERR_ALIGN;
        }
        if (shared[0].n != I_shared || shared[0].k != H || shared[1].n != I_shared || shared[1].k != H ||
            shared[2].n != H || shared[2].k != I_shared)
            return Q4_ERR_SHAPE;
    } else {
        I_shared = 0;
    }
    if (!q4_aligned16(x) || !q4_aligned16(y) || ((uintptr_t)workspace & 255u) || ((uintptr_t)router_w & 15u))
        return Q4_ERR_ALIGN;
    Workspace ws = carve(workspace, T, H, I, E, topk, I_shared, a8_mask);
    if (workspace_bytes < ws.bytes) return Q4_ERR_WORKSPACE;
    if (T == 0)   // no tokens: the optional routing outputs are empty ranges and zero counts
        return zero_routing(offsets, expert_counts, E, (cudaStream_t)stream);
    if (topk_ids) ws.ids = topk_ids;
    if (topk_w) ws.wts = topk_w;
    if (perm) ws.perm = perm;
    if (offsets) ws.offsets = offsets;
    if (expert_counts) ws.counts = expert_counts;
    cudaStream_t s = (cudaStream_t)stream;
    const int nch = (T + kRouteTok - 1) / kRouteTok;
    float* y32 = out_dtype == Q4_OUT_F32 ? reinterpret_cast<float*>(y) : ws.y32;

    CUtensorMap mrx, mrw;
    if (!tcg::make_map(&mrx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, T, (uint64_t)H * 2, kRouteKC, kRouteTok,
                       CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !tcg::make_map(&mrw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, router_w, H, E, (uint64_t)H * 4, kRouteKC, 64,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    constexpr int route_smem = kRouteStages * (kRouteWTile + kRouteXTile);
    if (const cudaError_t e = cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, route_smem))
        return q4_cuda_status(e);
    moe_route_kernel<<<nch, kRouteThreads, route_smem, s>>>(mrx, mrw, T, H, router_bias, E, topk, ws.ids, ws.wts,
                                                            ws.hist, dev_status);
    moe_scan_kernel<<<1, kScanThreads, 0, s>>>(ws.hist, nch, E, I, H, ws.chunk_base, ws.offsets, ws.counts,
                                                   ws.tiles_gu, ws.tiles_dn);
    int rc;
    if (a8_mask & 1) {
        // one per-token quantization of x serves every expert the token visits; the codes and their
        // scales are permuted together
        if ((rc = q4_act_quant_rows(x, false, T, H, ws.xq_tok, ws.sa_tok, dev_status, s))) return rc;
        moe_scatter_kernel<<<nch, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(ws.xq_tok), T, H, E, topk, ws.ids,
                                               ws.wts, ws.chunk_base, ws.perm, ws.row_tok, ws.row_w,
                                               reinterpret_cast<uint8_t*>(ws.xperm), ws.sa_tok, ws.sa_row, nullptr, nullptr,
                                               dev_status);
    } else {
        moe_scatter_kernel<<<nch, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(x), T, 2 * H, E, topk, ws.ids,
                                               ws.wts, ws.chunk_base, ws.perm, ws.row_tok, ws.row_w,
                                               reinterpret_cast<uint8_t*>(ws.xperm), nullptr, nullptr, nullptr, nullptr,
                                               dev_status);
    }
    if (const cudaError_t e = cudaMemsetAsync(y32, 0, (size_t)T * H * sizeof(float), s)) return q4_cuda_status(e);
    rc = q4_launch_status();
    if (rc) return rc;
    for (int c = 0; c < n_classes && !rc; c++) {
        // the class's slice of the routing bookkeeping: its experts' row offsets and tile prefix sums
        const int e0 = class_begin[c], Ec = class_begin[c + 1] - e0;
        const q4_weight* cw = experts + 3 * c;
        Workspace wc = ws;
        wc.offsets = ws.offsets + e0;
        wc.tiles_gu = ws.tiles_gu + e0;
        wc.tiles_dn = ws.tiles_dn + e0;
        rc = launch_experts_any(wc, cw, T, H, I, Ec, topk, y32, dev_status, s, a8_mask);
    }
    if (rc) return rc;
    if (I_shared > 0) {
        // the shared expert: every token, weight 1, its output added into the same fp32 sums
        moe_shared_setup_kernel<<<(T + 255) / 256, 256, 0, s>>>(T, H, I_shared, ws.offsets_s, ws.tiles_gu_s,
                                                                  ws.tiles_dn_s, ws.row_tok_s, ws.row_w_s);
        if ((rc = q4_launch_status())) return rc;
        Workspace w1 = ws;
        w1.xperm = const_cast<uint16_t*>(x);
        w1.h = ws.h_s;
        w1.offsets = ws.offsets_s;
        w1.tiles_gu = ws.tiles_gu_s;
        w1.tiles_dn = ws.tiles_dn_s;
        w1.row_tok = ws.row_tok_s;
        w1.row_w = ws.row_w_s;
        rc = launch_experts_any(w1, shared, T, H, I_shared, 1, 1, y32, dev_status, s, 0);
        if (rc) return rc;
    }
    if (out_dtype == Q4_OUT_BF16) {
        const int64_t n = (int64_t)T * H;
        f32_to_bf16_kernel<<<(int)std::min<int64_t>((n + 255) / 256, 4096), 256, 0, s>>>(y32, reinterpret_cast<__nv_bfloat16*>(y), n);
        rc = q4_launch_status();
    }
    return rc;
}

// ---------------------------------------------------------------------------------------------- //
// The layer's steps as separate calls, the units of expert parallelism in its all-to-all form: routing
// with the permutation and the dispatch buffer (moe_q4_route), the expert FFN on rows routed elsewhere
// (moe_q4_forward_rows) and the weighted combine back into token order (moe_q4_combine).
// ---------------------------------------------------------------------------------------------- //

// Pre-routed rows: one CTA per chunk of kRouteTok rows writes the rows' local expert ids and weights
// (topk = 1) and the chunk's expert histogram, as the route kernel does for routed tokens.  A row whose
// expert id lies outside [e_base, e_base + E) is reported (Q4_ERR_SHAPE) and counted as expert 0 with
// weight 0, so it contributes nothing.
__global__ void __launch_bounds__(64) moe_rows_setup_kernel(const int32_t* __restrict__ row_expert,
                                                            const float* __restrict__ row_weight, int R, int E,
                                                            int e_base, int32_t* __restrict__ ids,
                                                            float* __restrict__ wts, int32_t* __restrict__ hist,
                                                            int32_t* status)
{
    __shared__ int hc[tcg::kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hc[e] = 0;
    __syncthreads();
    const int r = blockIdx.x * kRouteTok + threadIdx.x;
    if (threadIdx.x < kRouteTok && r < R) {
        int e = row_expert[r] - e_base;
        float w = row_weight ? row_weight[r] : 1.0f;
        if (e < 0 || e >= E) {
            q4_set_status(status, Q4_ERR_SHAPE);
            e = 0;
            w = 0.0f;
        }
        ids[r] = e;
        wts[r] = w;
        atomicAdd(&hc[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = hc[e];
}

// y[t] = sum_j w[t][j] * o[pair_pos[t*topk + j]] in slot order (deterministic): one CTA per token.
__global__ void __launch_bounds__(256) moe_combine_kernel(const float* __restrict__ o, const int32_t* __restrict__ pair_pos,
                                                          const float* __restrict__ w, int H, int topk, int P,
                                                          void* __restrict__ y, int out_bf16, int32_t* status)
{
    const int64_t t = blockIdx.x;
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) {
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int j = 0; j < topk; j++) {
            const int p = pair_pos[t * topk + j];
            if (p < 0 || p >= P) {   // not a position of the permuted rows: report, contribute nothing
                if (c == threadIdx.x) q4_set_status(status, Q4_ERR_SHAPE);
                continue;
            }
            const float wj = w[t * topk + j];
            const float4 v = __ldg(reinterpret_cast<const float4*>(o + (int64_t)p * H) + c);
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
        if (out_bf16) {
            __nv_bfloat162* yb = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(y) + t * H) + 2 * c;
            yb[0] = __floats2bfloat162_rn(acc.x, acc.y);
            yb[1] = __floats2bfloat162_rn(acc.z, acc.w);
        } else {
            reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + t * H)[c] = acc;
        }
    }
}

struct RouteWorkspace {
    int32_t *hist, *chunk_base, *tiles_gu, *tiles_dn, *counts, *perm, *row_tok;
    float* row_w;
    size_t bytes;
};

static RouteWorkspace carve_route(void* base, int T, int E, int topk)
{
    RouteWorkspace w = {};
    const size_t P = (size_t)T * topk, nch = (size_t)(T + kRouteTok - 1) / kRouteTok;
    uint8_t* p = reinterpret_cast<uint8_t*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) { uint8_t* q = p ? p + o : nullptr; o += al(bytes); return q; };
    w.hist = reinterpret_cast<int32_t*>(take(nch * E * 4));
    w.chunk_base = reinterpret_cast<int32_t*>(take(nch * E * 4));
    w.tiles_gu = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    w.tiles_dn = reinterpret_cast<int32_t*>(take((E + 1) * 4));
    w.counts = reinterpret_cast<int32_t*>(take(E * 4));
    w.perm = reinterpret_cast<int32_t*>(take(P * 4));
    w.row_tok = reinterpret_cast<int32_t*>(take(P * 4));
    w.row_w = reinterpret_cast<float*>(take(P * 4));
    w.bytes = o;
    return w;
}

extern "C" size_t moe_q4_route_workspace_size(int32_t T, int32_t E, int32_t topk)
{
    if (T < 0 || E <= 0 || topk <= 0) return 0;
    return carve_route(nullptr, T, E, topk).bytes;
}

extern "C" int moe_q4_route(const uint16_t* x, int32_t T, int32_t H, const float* router_w, const float* router_bias,
                            int32_t E, int32_t topk, int32_t* topk_ids, float* topk_w, int32_t* offsets,
                            int32_t* pair_pos, uint16_t* x_perm, int32_t* row_expert, int32_t* perm,
                            int32_t* expert_counts, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream)
{
    // the per-token and per-pair arrays hold T and T*topk entries: with no tokens they may be NULL
    if (!router_w || !offsets || !workspace || (T > 0 && (!x || !topk_ids || !topk_w || !pair_pos))) return Q4_ERR_NULL;
    if (T < 0 || H <= 0 || E < 1 || E > tcg::kMaxExperts || topk < 1 || topk > kMaxTopk || topk > E) return Q4_ERR_SHAPE;
    if ((int64_t)T * topk > kMaxPairs) return Q4_ERR_SHAPE;
    if (H % 128) return Q4_ERR_UNSUPPORTED;
    if (!q4_aligned16(x) || (x_perm && !q4_aligned16(x_perm)) || ((uintptr_t)workspace & 255u) ||
        ((uintptr_t)router_w & 15u))
        return Q4_ERR_ALIGN;
    RouteWorkspace ws = carve_route(workspace, T, E, topk);
    if (workspace_bytes < ws.bytes) return Q4_ERR_WORKSPACE;
    if (T == 0)   // no pairs: every expert's range is empty and its count 0
        return zero_routing(offsets, expert_counts, E, (cudaStream_t)stream);
    if (perm) ws.perm = perm;
    if (expert_counts) ws.counts = expert_counts;
    cudaStream_t s = (cudaStream_t)stream;
    const int nch = (T + kRouteTok - 1) / kRouteTok;
    CUtensorMap mrx, mrw;
    if (!tcg::make_map(&mrx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, T, (uint64_t)H * 2, kRouteKC, kRouteTok,
                       CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !tcg::make_map(&mrw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, router_w, H, E, (uint64_t)H * 4, kRouteKC, 64,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    constexpr int route_smem = kRouteStages * (kRouteWTile + kRouteXTile);
    if (const cudaError_t e = cudaFuncSetAttribute(moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, route_smem))
        return q4_cuda_status(e);
    moe_route_kernel<<<nch, kRouteThreads, route_smem, s>>>(mrx, mrw, T, H, router_bias, E, topk, topk_ids, topk_w,
                                                            ws.hist, dev_status);
    moe_scan_kernel<<<1, kScanThreads, 0, s>>>(ws.hist, nch, E, 128, H, ws.chunk_base, offsets, ws.counts,
                                                   ws.tiles_gu, ws.tiles_dn);
    moe_scatter_kernel<<<nch, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(x), T, 2 * H, E, topk, topk_ids, topk_w,
                                           ws.chunk_base, ws.perm, ws.row_tok, ws.row_w,
                                           reinterpret_cast<uint8_t*>(x_perm), nullptr, nullptr, pair_pos, row_expert,
                                           dev_status);
    return q4_launch_status();
}

extern "C" size_t moe_q4_rows_workspace_size(int32_t R, int32_t H, int32_t I, int32_t E)
{
    if (R < 0 || H <= 0 || I <= 0 || E <= 0) return 0;
    return carve(nullptr, R, H, I, E, 1).bytes;
}

extern "C" int moe_q4_forward_rows(const uint16_t* x_rows, int32_t R, int32_t H, const int32_t* row_expert,
                                   int32_t e_base, const float* row_weight, int32_t E, const q4_weight* experts,
                                   int32_t I, float* y_rows, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream)
{
    // the row arrays hold R entries: with no rows they may be NULL
    if (!experts || !workspace || (R > 0 && (!x_rows || !row_expert || !y_rows))) return Q4_ERR_NULL;
    if (R < 0 || H <= 0 || I <= 0 || E < 1 || E > tcg::kMaxExperts) return Q4_ERR_SHAPE;
    if (H % 128 || I % 128) return Q4_ERR_UNSUPPORTED;
    for (int i = 0; i < 3; i++) {
        const q4_weight& w = experts[i];
        if (!w.packed || !w.scales || (!w.symmetric && !w.zeros)) return Q4_ERR_NULL;
        if (w.group != experts[0].group || w.symmetric != experts[0].symmetric) return Q4_ERR_UNSUPPORTED;
        if (w.group <= 0 || w.k % w.group) return Q4_ERR_SHAPE;
        if (!q4_aligned16(w.packed) || !q4_aligned16(w.scales) || (!w.symmetric && !q4_aligned16(w.zeros)))
            return Q4_ERR_ALIGN;
    }
    if (experts[0].group != 32 && experts[0].group != 64 && experts[0].group != 128 && experts[0].group != 256)
        return Q4_ERR_UNSUPPORTED;
    if (experts[0].n != E * I || experts[0].k != H || experts[1].n != E * I || experts[1].k != H ||
        experts[2].n != E * H || experts[2].k != I)
        return Q4_ERR_SHAPE;
    if (!q4_aligned16(x_rows) || !q4_aligned16(y_rows) || ((uintptr_t)workspace & 255u)) return Q4_ERR_ALIGN;
    Workspace ws = carve(workspace, R, H, I, E, 1);
    if (workspace_bytes < ws.bytes) return Q4_ERR_WORKSPACE;
    if (R == 0) return Q4_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int nch = (R + kRouteTok - 1) / kRouteTok;
    moe_rows_setup_kernel<<<nch, 64, 0, s>>>(row_expert, row_weight, R, E, e_base, ws.ids, ws.wts, ws.hist, dev_status);
    moe_scan_kernel<<<1, kScanThreads, 0, s>>>(ws.hist, nch, E, I, H, ws.chunk_base, ws.offsets, ws.counts,
                                                   ws.tiles_gu, ws.tiles_dn);
    moe_scatter_kernel<<<nch, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(x_rows), R, 2 * H, E, 1, ws.ids, ws.wts,
                                           ws.chunk_base, ws.perm, ws.row_tok, ws.row_w,
                                           reinterpret_cast<uint8_t*>(ws.xperm), nullptr, nullptr, nullptr, nullptr,
                                           dev_status);
    if (const cudaError_t e = cudaMemsetAsync(y_rows, 0, (size_t)R * H * sizeof(float), s)) return q4_cuda_status(e);
    int rc = q4_launch_status();
    if (rc) return rc;
    return launch_experts_any(ws, experts, R, H, I, E, 1, y_rows, dev_status, s, 0);
}

extern "C" int moe_q4_combine(const float* o_rows, int32_t P, int32_t H, const int32_t* pair_pos, const float* topk_w,
                              int32_t T, int32_t topk, void* y, int32_t out_dtype, int32_t* dev_status, void* stream)
{
    // with no tokens nothing is read or written and the arrays may be NULL
    if (T > 0 && (!o_rows || !pair_pos || !topk_w || !y)) return Q4_ERR_NULL;
    if (T < 0 || P < 0 || H <= 0 || topk < 1 || topk > kMaxTopk || H % 4 || (int64_t)T * topk > kMaxPairs)
        return Q4_ERR_SHAPE;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    if (!q4_aligned16(o_rows) || !q4_aligned16(y)) return Q4_ERR_ALIGN;
    if (T == 0) return Q4_OK;
    moe_combine_kernel<<<T, 256, 0, (cudaStream_t)stream>>>(o_rows, pair_pos, topk_w, H, topk, P, y,
                                                            out_dtype == Q4_OUT_BF16, dev_status);
    return q4_launch_status();
}

// ---------------------------------------------------------------------------------------------- //
// moe_q4_forward without a caller workspace (for callers that cannot allocate device memory; see
// include/q4.h).  The scratch is one file-scope device array shared by every call; its device address
// is looked up once per device with cudaGetSymbolAddress (host code must not use the array's name
// as a device pointer) and then passed to moe_q4_forward as the workspace.
// ---------------------------------------------------------------------------------------------- //
static __device__ __align__(256) uint8_t q4_moe_noalloc_scratch[Q4_MOE_NOALLOC_SCRATCH_BYTES];

// The current driver context (nullptr when the entry point is unavailable): a device reset makes a new
// primary context, in which the module and its array may sit elsewhere, so the cache is keyed on it too.
static void* current_context()
{
    using GetCurrent = CUresult (*)(CUcontext*);
    static GetCurrent fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess) ? reinterpret_cast<GetCurrent>(f) : nullptr;
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

static int noalloc_scratch_address(void** out)
{
    static void* cache[64] = {nullptr};
    static const void* cache_ctx[64] = {nullptr};
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return Q4_ERR_CUDA;
    const void* ctx = current_context();   // nullptr until the runtime has made a context current here
    std::lock_guard<std::mutex> guard(lock);
    if (!cache[dev] || !ctx || cache_ctx[dev] != ctx) {
        void* p = nullptr;   // the lookup makes the device's primary context current on this thread
        if (cudaGetSymbolAddress(&p, q4_moe_noalloc_scratch) != cudaSuccess || !p) return Q4_ERR_CUDA;
        cache[dev] = p;
        cache_ctx[dev] = current_context();
    }
    *out = cache[dev];
    return Q4_OK;
}

extern "C" int moe_q4_forward_noalloc(const uint16_t* x, int32_t T, int32_t H, const float* router_w,
                                      const float* router_bias, int32_t E, int32_t topk, const q4_weight* experts,
                                      int32_t I, void* y, int32_t out_dtype, int32_t* topk_ids, float* topk_w,
                                      int32_t* perm, int32_t* offsets, int32_t* expert_counts, int32_t* dev_status,
                                      void* stream)
{
    const size_t need = moe_q4_workspace_size(T, H, I, E, topk);
    if (need > Q4_MOE_NOALLOC_SCRATCH_BYTES) return Q4_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = noalloc_scratch_address(&scratch);
    if (rc) return rc;
    return moe_q4_forward(x, T, H, router_w, router_bias, E, topk, experts, I, y, out_dtype, topk_ids, topk_w, perm,
                          offsets, expert_counts, scratch, Q4_MOE_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
