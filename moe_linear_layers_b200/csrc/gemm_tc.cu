// Tensor-core (tcgen05) GEMM for INT4 weights: W4A16 (bf16 MMA) and W4A8 (int8 MMA).
//
// Sources: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a 16-bit
// type for W4A16), §2.3 (INT4 widened to INT8, INT8 x INT8 into INT32, rescale by scale_w*scale_a),
// §2.2 (INT8 tensor cores at twice the FP16 rate); "从FP32到INT4" §1.3 (one scale per group).
//
// Computes y[m][n] = sum_g s[n][g] * D_g[n][m] (W4A16) or y = s_a[m] * sum_g s[n][g] * D_g (W4A8), where
// D_g = sum_{k in g} (code - zero)[n][k] * x[m][k] is exact: the MMA sees integer codes (exact in bf16 /
// int8) and accumulates one group at a time; the group scale is applied in fp32 in the epilogue.
//
// Tile: 128 weight rows (the MMA's M, one TMEM lane each) x 128 tokens (the MMA's N), K staged 128
// at a time.  The weights are the A operand and live in TMEM: converter warps read the packed
// nibbles (TMA -> shared memory, 64-byte swizzle), widen them in registers and write them with
// tcgen05.st, so the widened weights never touch shared memory.  The activations are the B operand:
// TMA tiles with 128-byte swizzle in shared memory.  Per-group accumulators are double-buffered in
// TMEM so the MMA of group g+1 overlaps the epilogue's drain of group g.
//
// Warp roles (448 threads): warp 0 TMA producer, warp 1 MMA issuer (+ TMEM owner), warps 2-5
// converters (TMEM lanes 32*(warp%4) ...), warps 6-13 epilogue (two warps per TMEM lane quarter,
// each draining 64 of the 128 token columns).  Persistent: one CTA per SM walks tiles with a
// stride of gridDim.x; the rings carry their phases across tiles.
#include <cudaTypedefs.h>

#include "tc_ptx.cuh"

namespace {

constexpr int BM = 128;          // weight rows per tile
constexpr int BN = 128;          // tokens per tile
constexpr int KBLK = 128;        // K per stage
constexpr int NS = 4;            // shared-memory stages (x + packed)
constexpr int NA = 4;            // TMEM stages of widened weights
constexpr int WSTAGE = BM * KBLK / 2;  // packed bytes per stage
constexpr int kThreads = 448;
constexpr uint32_t kTmemCols = 512;

template <bool INT8> struct Cfg {
    static constexpr int XSTAGE = BN * KBLK * (INT8 ? 1 : 2);   // activation bytes per stage
    static constexpr int ACOLS = KBLK / (INT8 ? 4 : 2);         // TMEM columns of one widened stage
    static constexpr int KI = INT8 ? 32 : 16;                   // K per MMA instruction
    static constexpr uint32_t A_COL0 = 2 * BN;                  // widened weights after the 2 D buffers
    static constexpr int SMEM = NS * (XSTAGE + WSTAGE) + 1024 + 256;
};

struct TcParams {
    int M, N, K, sym, out_bf16;
    const __half* scales;
    const __half* zeros;
    const float* scale_a;
    void* y;
    int32_t* acc_dbg;
    int32_t* status;
};

struct Bars {
    uint64_t xw_full[NS], xw_empty[NS], a_full[NA], a_empty[NA], d_full[2], d_empty[2], done;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// bf16x2 (a - b), exact here: both operands are small integers offset by 128.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 8 nibbles (k = 0..7, even k in the low nibble of each byte) -> 4 bf16x2 words of the exact integers
// (code - zero) in natural k order.  A PRMT puts nibble 2b at bits 0-3 and nibble 2b+1 at bits 16-19;
// one LOP3 ORs in the bf16 exponent of 128.0 (and flips bit 3 of symmetric two's-complement codes,
// which turns them into code + 8); one bf16x2 subtract removes 128 + zero.
template <bool SYM>
__device__ __forceinline__ void widen_bf16(uint32_t w, uint32_t bias2, uint32_t (&o)[4])
{
    constexpr uint32_t key = SYM ? (0x43004300u ^ 0x00080008u) : 0x43004300u;
    const uint32_t u = w >> 4;
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const uint32_t sel = (uint32_t)b | ((uint32_t)b << 4) | ((uint32_t)(4 + b) << 8) | ((uint32_t)(4 + b) << 12);
        const uint32_t t = prmt(w, u, sel);
        o[b] = bf16x2_sub(lop3_and_xor(t, 0x000F000Fu, key), bias2);
    }
}

// 8 symmetric nibbles -> 8 int8 of value 16*code in natural k order (two 32-bit words).  The nibble
// is placed in the high half of its byte, which makes the byte the two's-complement value 16*code;
// the epilogue folds the factor 1/16 into the (exact, power-of-two) scale.
__device__ __forceinline__ void widen_s8x16(uint32_t w, uint32_t& o0, uint32_t& o1)
{
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // codes of even k
    const uint32_t hi = w & 0xF0F0F0F0u;         // codes of odd k
    o0 = prmt(lo, hi, 0x5140u);
    o1 = prmt(lo, hi, 0x7362u);
}

__device__ __forceinline__ uint32_t bf16x2_bits(float v)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(v, v);
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <bool INT8, int G, bool SYM>
__global__ void __launch_bounds__(kThreads, 1)
q4_gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w, TcParams p)
{
    using C = Cfg<INT8>;
    constexpr int GPK = KBLK / G;      // groups per K stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* xs = smem;                            // NS x XSTAGE, 1024-aligned stages
    uint8_t* wsm = smem + NS * C::XSTAGE;          // NS x WSTAGE
    Bars* bars = reinterpret_cast<Bars*>(wsm + NS * WSTAGE);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int tiles_m = (p.M + BN - 1) / BN, tiles_n = (p.N + BM - 1) / BM;
    const int total = tiles_m * tiles_n;
    const int kblocks = p.K / KBLK, ngroups = p.K / G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) { tc::mbar_init(&bars->xw_full[i], 1); tc::mbar_init(&bars->xw_empty[i], 1 + 4); }
        for (int i = 0; i < NA; i++) { tc::mbar_init(&bars->a_full[i], 4); tc::mbar_init(&bars->a_empty[i], 1); }
        for (int i = 0; i < 2; i++) { tc::mbar_init(&bars->d_full[i], 1); tc::mbar_init(&bars->d_empty[i], 8); }
        tc::mbar_init(&bars->done, 1);
        bars->abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tm_x);
        tc::tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) tc::tmem_alloc(&bars->tmem_base, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const int m0 = (t % tiles_m) * BN, n0 = (t / tiles_m) * BM;
                for (int kb = 0; kb < kblocks; kb++, it++) {
                    const int s = it % NS;
                    if (!tc::mbar_wait(&bars->xw_empty[s], ((it / NS) & 1) ^ 1, p.status, abort_flag)) break;
                    tc::mbar_arrive_expect_tx(&bars->xw_full[s], C::XSTAGE + WSTAGE);
                    uint8_t* xdst = xs + s * C::XSTAGE;
                    if constexpr (INT8) {
                        tc::tma_load_2d(xdst, &tm_x, &bars->xw_full[s], kb * KBLK, m0);
                    } else {
                        tc::tma_load_2d(xdst, &tm_x, &bars->xw_full[s], kb * KBLK, m0);
                        tc::tma_load_2d(xdst + BN * 128, &tm_x, &bars->xw_full[s], kb * KBLK + 64, m0);
                    }
                    tc::tma_load_2d(wsm + s * WSTAGE, &tm_w, &bars->xw_full[s], kb * (KBLK / 2), n0);
                }
            }
            // let every copy this thread issued land before the CTA can exit
            if (*abort_flag) {
                const uint32_t first = it > (uint32_t)NS ? it - NS : 0;
                for (uint32_t j = first; j < it; j++)
                    tc::mbar_wait(&bars->xw_full[j % NS], (j / NS) & 1, p.status, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = INT8 ? tc::idesc_s8_s32(BN) : tc::idesc_bf16_f32(BN);
            uint32_t it = 0, g = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                for (int kb = 0; kb < kblocks && ok; kb++, it++) {
                    const int s = it % NS, sa = it % NA;
                    ok = tc::mbar_wait(&bars->xw_full[s], (it / NS) & 1, p.status, abort_flag) &&
                         tc::mbar_wait(&bars->a_full[sa], (it / NA) & 1, p.status, abort_flag);
                    if (!ok) break;
                    tc::fence_after_sync();
                    const uint32_t xaddr = tc::smem_u32(xs + s * C::XSTAGE);
#pragma unroll
                    for (int gi = 0; gi < GPK; gi++, g++) {
                        const uint32_t db = g & 1;
                        if (!(ok = tc::mbar_wait(&bars->d_empty[db], ((g >> 1) & 1) ^ 1, p.status, abort_flag))) break;
                        tc::fence_after_sync();
#pragma unroll
                        for (int i = 0; i < G / C::KI; i++) {
                            const int kk = gi * G + i * C::KI;   // k offset inside the stage
                            const uint32_t a_tmem = tbase + C::A_COL0 + sa * C::ACOLS + (INT8 ? kk / 4 : kk / 2);
                            uint32_t boff;
                            if constexpr (INT8) boff = kk;                                   // one 128-byte row box
                            else boff = (kk / 64) * (BN * 128) + (kk % 64) * 2;               // two 64-column boxes
                            const uint64_t bdesc = tc::smem_desc_sw128(xaddr + (boff & ~127u)) + ((boff & 127u) >> 4);
                            if constexpr (INT8) tc::mma_i8_ts(tbase + db * BN, a_tmem, bdesc, idesc, i > 0);
                            else tc::mma_bf16_ts(tbase + db * BN, a_tmem, bdesc, idesc, i > 0);
                        }
                        tc::mma_commit(&bars->d_full[db]);
                    }
                    tc::mma_commit(&bars->xw_empty[s]);
                    tc::mma_commit(&bars->a_empty[sa]);
                }
            }
            // every MMA issued so far has completed once `done` flips
            tc::mma_commit(&bars->done);
            tc::mbar_wait(&bars->done, 0, p.status, abort_flag, 100000000ull);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------------ converters
        const int sub = warp & 3;
        const int r = 32 * sub + lane;                 // row in tile == TMEM lane
        const uint32_t lane_field = (uint32_t)(32 * sub) << 16;
        uint32_t it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const int n0 = (t / tiles_m) * BM;
            const int n = n0 + r;
            for (int kb = 0; kb < kblocks; kb++, it++) {
                const int s = it % NS, sa = it % NA;
                if (!tc::mbar_wait(&bars->xw_full[s], (it / NS) & 1, p.status, abort_flag)) goto conv_done;
                uint4 v[4];
                const uint32_t wrow = tc::smem_u32(wsm + s * WSTAGE) + r * 64;
#pragma unroll
                for (int c = 0; c < 4; c++) v[c] = lds128(wrow + ((c ^ ((r >> 1) & 3)) << 4));
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->xw_empty[s]);
                uint32_t bias[GPK];
                if constexpr (!INT8) {
#pragma unroll
                    for (int gi = 0; gi < GPK; gi++) {
                        float z = 8.0f;
                        if constexpr (!SYM) z = (n < p.N) ? __half2float(p.zeros[(int64_t)n * ngroups + kb * GPK + gi]) : 0.0f;
                        bias[gi] = bf16x2_bits(128.0f + z);
                    }
                }
                if (!tc::mbar_wait(&bars->a_empty[sa], ((it / NA) & 1) ^ 1, p.status, abort_flag)) goto conv_done;
                __syncwarp();
                tc::fence_after_sync();
                const uint32_t words[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                            v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
                const uint32_t acol = tbase + lane_field + C::A_COL0 + sa * C::ACOLS;
                if constexpr (INT8) {
                    uint32_t o[32];
#pragma unroll
                    for (int w = 0; w < 16; w++) widen_s8x16(words[w], o[2 * w], o[2 * w + 1]);
                    tc::tmem_st32(acol, o);
                } else {
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        uint32_t o[32];
#pragma unroll
                        for (int w = 0; w < 8; w++) {
                            const int ww = 8 * h + w;                  // word index: k = 8*ww .. 8*ww+7
                            uint32_t q[4];
                            widen_bf16<SYM>(words[ww], bias[(8 * ww) / G], q);
#pragma unroll
                            for (int b = 0; b < 4; b++) o[4 * w + b] = q[b];
                        }
                        tc::tmem_st32(acol + 32 * h, o);
                    }
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->a_full[sa]);
            }
        }
    conv_done:;
    } else {
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 6;
        const int sub = warp & 3, half = ew >> 2;
        const int r = 32 * sub + lane;
        const uint32_t lane_field = (uint32_t)(32 * sub) << 16;
        uint32_t g = 0;
        float acc[64];
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const int m0 = (t % tiles_m) * BN, n0 = (t / tiles_m) * BM;
            const int n = n0 + r;
            const bool nvalid = n < p.N;
#pragma unroll
            for (int j = 0; j < 64; j++) acc[j] = 0.0f;
            float s_next = nvalid ? __half2float(p.scales[(int64_t)n * ngroups]) : 0.0f;
            for (int gl = 0; gl < ngroups; gl++, g++) {
                const uint32_t db = g & 1;
                float s = s_next;
                if (gl + 1 < ngroups) s_next = nvalid ? __half2float(p.scales[(int64_t)n * ngroups + gl + 1]) : 0.0f;
                if constexpr (INT8) s *= 0.0625f;   // the MMA saw 16 * code
                if (!tc::mbar_wait(&bars->d_full[db], (g >> 1) & 1, p.status, abort_flag)) goto epi_done;
                __syncwarp();
                tc::fence_after_sync();
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    uint32_t v[32];
                    tc::tmem_ld32(tbase + lane_field + db * BN + half * 64 + 32 * h, v);
                    tc::tmem_wait_ld();
                    if constexpr (INT8) {
                        if (p.acc_dbg && nvalid) {
#pragma unroll
                            for (int j = 0; j < 32; j++) {
                                const int m = m0 + half * 64 + 32 * h + j;
                                if (m < p.M) p.acc_dbg[((int64_t)m * p.N + n) * ngroups + gl] = ((int32_t)v[j]) >> 4;
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 32; j++) acc[32 * h + j] = fmaf(s, (float)(int32_t)v[j], acc[32 * h + j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++) acc[32 * h + j] = fmaf(s, __uint_as_float(v[j]), acc[32 * h + j]);
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->d_empty[db]);
            }
            if (nvalid) {
#pragma unroll
                for (int j = 0; j < 64; j++) {
                    const int m = m0 + half * 64 + j;
                    if (m < p.M) {
                        float v = acc[j];
                        if constexpr (INT8) v *= p.scale_a[m];
                        const int64_t o = (int64_t)m * p.N + n;
                        if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
                        else reinterpret_cast<float*>(p.y)[o] = v;
                    }
                }
            }
        }
    epi_done:;
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) {
        __syncwarp();
        tc::tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------- //
// host side
// ---------------------------------------------------------------------------------------------- //

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 2-D tensor map: inner dimension `inner` elements (contiguous), `outer` rows, row pitch in bytes.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool INT8, int G, bool SYM>
int launch(const CUtensorMap& mx, const CUtensorMap& mw, const TcParams& p, cudaStream_t s)
{
    auto kern = q4_gemm_tc_kernel<INT8, G, SYM>;
    constexpr int smem = Cfg<INT8>::SMEM;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return Q4_ERR_CUDA;
    const int tiles = ((p.M + BN - 1) / BN) * ((p.N + BM - 1) / BM);
    const int grid = std::min(tiles, q4_num_sms());
    kern<<<grid, kThreads, smem, s>>>(mx, mw, p);
    return q4_launch_status();
}

}  // namespace

// m >= 1, k % 128 == 0, group in {64, 128}; W4A8 requires symmetric weights.
int q4_gemm_tc_launch(const void* x, const float* scale_a, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                      int32_t* acc_dbg, bool int8_path, int32_t* dev_status, cudaStream_t stream)
{
    if (w->k % KBLK) return Q4_ERR_UNSUPPORTED;
    CUtensorMap mx, mw;
    const uint64_t K = (uint64_t)w->k;
    bool ok = int8_path
        ? make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, x, K, (uint64_t)m, K, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B)
        : make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, (uint64_t)m, 2 * K, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->packed, K / 2, (uint64_t)w->n, K / 2, KBLK / 2, BM,
                        CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) return Q4_ERR_CUDA;
    TcParams p;
    p.M = m;
    p.N = w->n;
    p.K = w->k;
    p.sym = w->symmetric;
    p.out_bf16 = out_dtype == Q4_OUT_BF16;
    p.scales = reinterpret_cast<const __half*>(w->scales);
    p.zeros = reinterpret_cast<const __half*>(w->zeros);
    p.scale_a = scale_a;
    p.y = y;
    p.acc_dbg = acc_dbg;
    p.status = dev_status;
    if (int8_path) {
        if (!w->symmetric) return Q4_ERR_UNSUPPORTED;
        return w->group == 128 ? launch<true, 128, true>(mx, mw, p, stream) : launch<true, 64, true>(mx, mw, p, stream);
    }
    if (w->group == 128)
        return w->symmetric ? launch<false, 128, true>(mx, mw, p, stream) : launch<false, 128, false>(mx, mw, p, stream);
    return w->symmetric ? launch<false, 64, true>(mx, mw, p, stream) : launch<false, 64, false>(mx, mw, p, stream);
}
