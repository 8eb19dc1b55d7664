// Tensor-core (tcgen05) GEMM with INT4 weights widened into TMEM, shared by the dense linear layers
// (W4A16 and W4A8) and by the two grouped expert GEMMs of the MoE layer.
//
// Sources: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.1 (4-bit storage restored to a 16-bit
// type for W4A16), §2.3 (INT4 widened to INT8, INT8 x INT8 into INT32, rescale by scale_w*scale_a),
// §2.2 (INT8 tensor cores at twice the FP16 rate); "从FP32到INT4" §1.3 (one scale per group);
// "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" MoE架构设计 (experts are small SwiGLU FFNs);
// "大模型之Dense、MoE与量化" 混合专家架构 MoE (expert outputs recombined in proportion to the router).
//
// Every mode computes, for a tile of 128 weight rows (the MMA's M, one TMEM lane each) and 128
// activation rows (the MMA's N), D_g = sum_{k in g} (code - zero)[row][k] * act[m][k] exactly (integer
// codes are exact in bf16 / fp16 / int8) one quantization group at a time, and the epilogue
// accumulates s[row][g] * D_g in fp32.  Group accumulators rotate through two TMEM buffers (three for
// W4A8 and for the hi/lo down projection) so the MMAs of the next groups overlap the epilogue's drain
// of group g.
//
// Data flow: TMA brings the packed nibbles (64-byte swizzle) and the activation tile (128-byte
// swizzle, K-major, the MMA's B operand) into a shared-memory ring of 3 to 8 stages (Cfg::NS, by mode).  Converter warps widen the
// nibbles in registers and write them into TMEM with tcgen05.st (the MMA's A operand), so widened
// weights never use shared-memory bandwidth.  Four threads in four warps issue tcgen05.mma for
// alternate K stages and commit to mbarriers.
//
// Modes:
//   Dense   y[m][n] = sum_g s[n][g] * D_g (W4A16, bf16 MMA) or y = s_a[m] * sum_g s[n][g] * D_g / 16
//           (W4A8, int8 MMA on 16*code).
//   GateUp  A rows 0-63 = gate rows i0..i0+63 of expert e, rows 64-127 = the same rows of up; B = the
//           expert's rows of the permuted activations (bf16, or int8 codes with per-row scales s_a);
//           epilogue h = SiLU(gate) * up in fp32 (gate and up rows each evaluate it for half of the
//           tokens, after exchanging the other half through shared memory), stored as bf16 hi = bf16(h) and
//           lo = bf16(h - hi), which together hold h to about 2^-17 of its magnitude (gate and up each
//           times s_a first with int8 codes).  Row layout of h: [I/64][hi 64 | lo 64].  For a down
//           projection on INT8 activations, h is stored instead as the fp16 activation it quantizes.
//   Down    A = 128 rows of the expert's down projection (bf16 codes, or int8), B = h: per K step one
//           MMA on the hi values and one on the lo values into the same accumulator (or, int8, the
//           codes of h and per-row scales s_a); epilogue y[token][n] += w[token][slot] * (s_a) * out
//           (fp32 reduction into the output).
//
// Warp roles (640 threads = 5 warpgroups, launched at 96 registers and re-partitioned with setmaxnreg):
//   warps 0-3    MMA issuers, one thread each, stage it issued by warp it % 4 (warp 1 also owns TMEM);
//   warps 4-7    converters (TMEM lanes 32*(warp%4) ...); a build with Q4_CONV_SETS=2 adds warps 20-23 for
//                the odd stages (measured slower on B200: 683 against 880 TFLOP/s, so one set is the default);
//   warp 8       TMA producer (issues every copy, never waits on an mbarrier); warp 9 ring-slot watcher;
//                warp 10 parameter loader; warp 11 the MoE gate/up's h stores (else idle);
//   warps 12-19  epilogue (two warps per TMEM lane quarter, each draining 64 of the 128 columns).
// Measured on B200: one thread issues an M128 N128 K16 MMA only every ~120 cycles, half the tensor
// pipe's rate, and any strong memory operation in that thread (an mbarrier wait included) stalls it
// until its MMAs have retired; four issuer threads in different warps that only poll progress counters
// with weak loads keep the pipe at one MMA per 64 cycles, commits included.  A thread that waits on an
// mbarrier also stalls until its own bulk copies have landed, so the thread that issues the TMA copies
// polls a counter that another thread publishes after the mbarrier wait.  Persistent CTAs walk tiles
// with a stride of gridDim.x; the rings carry their phases across tiles.  Every wait is bounded
// (Q4_ERR_TIMEOUT, then a clean exit).
//
// Epilogue arithmetic runs on packed fp32 pairs (FFMA2).  For W4A8 every int32 accumulator is preloaded
// with the bit pattern of 1.5 * 2^23, so the accumulated bits are the float 1.5 * 2^23 + acc and one
// packed subtraction replaces an integer-to-float conversion per value.
#pragma once

#include "tc_ptx.cuh"

namespace tcg {

enum class Mode { Dense, GateUp, Down };

constexpr int BM = 128;                  // weight rows per tile
constexpr int BN = 128;                  // activation rows per tile
constexpr int KBLK = 128;                // K per stage
constexpr int kMaxNA = 4;                // TMEM stages of widened weights (at most)
// 16-bit modes: group accumulators and TMEM stages of widened weights (ND16 * 128 + NA16 * 64 <= 512)
#ifndef Q4_ND16
#define Q4_ND16 2
#endif
#ifndef Q4_NA16
#define Q4_NA16 4
#endif
// the hi/lo down projection: two MMAs per K step, so two widened stages ahead suffice and a third
// accumulator covers its tile output (the atomic combine): 0.6-1 % on the MoE layer
#ifndef Q4_ND_HILO
#define Q4_ND_HILO 3
#endif
#ifndef Q4_NA_HILO
#define Q4_NA_HILO 2
#endif
// the MoE gate/up projection (its tile output, the SwiGLU epilogue, is the longest)
#ifndef Q4_ND_GU
#define Q4_ND_GU 2
#endif
#ifndef Q4_NA_GU
#define Q4_NA_GU 4
#endif
constexpr int kMaxStages = 8;            // barrier slots of the shared-memory ring
constexpr int WSTAGE = BM * KBLK / 2;    // packed bytes per stage
#ifndef Q4_CONV_SETS
#define Q4_CONV_SETS 1
#endif
constexpr int kConvSets = Q4_CONV_SETS;  // converter warpgroups, alternate stages
constexpr int kThreads = 640 + 128 * (kConvSets - 1);   // 20 or 24 warps
constexpr int kIssuers = 4;              // MMA issuer threads (warps 0-3)
// registers per thread: the launch allocation (65536 / threads, rounded down to a multiple of 8) and the
// per-warpgroup split after setmaxnreg; the split may not exceed the launch allocation
constexpr int kLaunchRegs = kConvSets == 1 ? 96 : 80;
constexpr int kRegsIssue = 48;                           // MMA issuers
constexpr int kRegsProd = kConvSets == 1 ? 56 : 40;      // TMA producers, parameter loader
constexpr int kRegsConv = kConvSets == 1 ? 88 : 64;      // converters (each set)
constexpr int kRegsEpi = kConvSets == 1 ? 144 : 128;     // epilogue (two warpgroups)
static_assert(128 * (kRegsIssue + kRegsProd + kConvSets * kRegsConv) + 256 * kRegsEpi <= kThreads * kLaunchRegs,
              "register split");
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxExperts = 256;
constexpr uint32_t kAccBias = 0x4B400000u;   // bits of 1.5 * 2^23: preloaded int32 accumulators (W4A8)
constexpr float kAccBiasF = 12582912.0f;

// PRING: the group parameters go through the shared-memory ring (every mode except symmetric W4A8)
template <bool INT8, Mode MODE, bool PRING> struct Cfg {
    // the 16-bit down projection reads h as hi and lo halves: twice the activation bytes per stage
    static constexpr bool HILO = MODE == Mode::Down && !INT8;
    static constexpr int XBLK = HILO ? 4 : 2;                   // 64-column blocks per stage (16-bit)
    static constexpr int XSTAGE = BN * KBLK * (INT8 ? 1 : 2) * (HILO ? 2 : 1);   // activation bytes per stage
    static constexpr int ACOLS = KBLK / (INT8 ? 4 : 2);         // TMEM columns of one widened stage
    static constexpr int KI = INT8 ? 32 : 16;                   // K per MMA instruction
    // group accumulators in TMEM: three for W4A8 (its MMAs are twice as fast, so the epilogue needs more
    // slack), two otherwise; the widened weights follow them (NA * ACOLS columns)
    static constexpr int ND = INT8 ? 3 : (HILO ? Q4_ND_HILO : (MODE == Mode::GateUp ? Q4_ND_GU : Q4_ND16));
    static constexpr int NA = INT8 ? 4 : (HILO ? Q4_NA_HILO : (MODE == Mode::GateUp ? Q4_NA_GU : Q4_NA16));
    static_assert(ND >= 2 && ND <= 3 && NA >= 2 && NA <= kMaxNA, "accumulator / TMEM stage counts");
    static constexpr uint32_t A_COL0 = ND * BN;
    static_assert(ND * BN + NA * ACOLS <= (int)kTmemCols, "TMEM columns");
    static constexpr int XCHG = MODE == Mode::GateUp ? 2 * 64 * 64 * 4 : 0;  // up -> gate exchange
    // group parameters staged in shared memory: 2 slots, each PW groups x 128 rows of fp16 scales and
    // zero points, group-major so a warp reads 32 consecutive rows (W4A8's epilogue reads its scales
    // through a register read-ahead instead, so symmetric W4A8 needs no ring at all)
    static constexpr int PTENS = 2;                             // scales, zero points
    static constexpr int PW = HILO ? 4 : 16;                    // quantization groups per window
    static constexpr int PSLOT = PW * BM * 2;                   // bytes of one tensor in one slot
    static constexpr int PARAMS = PRING ? 2 * PSLOT * PTENS : 0;
    // shared-memory stages (activations + packed weights): as many as fit, so that enough MMA work is
    // in flight to cover the latency of the activation copies
    static constexpr int NS = INT8 ? (MODE == Mode::GateUp ? 7 : 8) : (MODE == Mode::GateUp ? 4 : (HILO ? 3 : 5));
    static_assert(NS <= kMaxStages, "ring depth");
    static_assert(NS * (XSTAGE + WSTAGE) + XCHG + PARAMS + 1024 + 6144 <= 227 * 1024, "shared memory");
    static constexpr int SMEM = NS * (XSTAGE + WSTAGE) + XCHG + PARAMS + 1024 + 6144;
};

struct Args {
    int M, N, K;              // Dense: M activation rows, N weight rows.  MoE: N = rows per expert matrix
    int out_bf16;
    const __half* scales_a;   // Dense: W; GateUp: gate; Down: down
    const __half* zeros_a;
    const __half* scales_b;   // GateUp: up
    const __half* zeros_b;
    const float* scale_a;     // W4A8 per-activation-row scales (Dense: token; GateUp / Down: permuted row)
    void* y;                  // Dense: [M][N]; Down: fp32 [T][N] (reduction target)
    int32_t* acc_dbg;         // W4A8 debug partials (nullable)
    int32_t* status;
    // MoE
    const int32_t* expert_tiles;   // [E+1] prefix sums of tiles per expert (taken relative to [0])
    const int32_t* offsets;        // [E+1] first permuted row of each expert
    const int32_t* row_tok;        // Down: [P] token of each permuted row
    const float* row_w;            // Down: [P] routing weight of each permuted row
    __nv_bfloat16* h;              // GateUp output [P][N/64][hi 64 | lo 64], or fp16 [P][N] when h_f16
    int h_f16;                     // GateUp: h for an INT8 down projection, stored as the fp16 activation
    int E, topk;
    int T;                         // Down: rows of the output y (tokens)
    // Dense split-K (splits > 1): work item t is split t % splits of output tile t / splits and covers the
    // K blocks [split * sps, min(K / 128, (split + 1) * sps)); it stores its fp32 partial sums (times s_a
    // for W4A8) in part[split][M][N], which a second kernel adds up in split order
    int splits, sps;
    float* part;
};

struct Tile {
    int m0, m_end;    // activation rows [m0, m0+128) of which rows < m_end are valid
    int n0;           // Dense/Down: first weight row of the tile inside the (expert) matrix; GateUp: i0
    int wrow_a, wrow_b;  // packed rows of the TMA boxes
    int e;
    int kb0, kb1;     // the work item's 128-K blocks (all of them unless the K dimension is split)
    int split;
};

// The K blocks of work item t (Dense split-K) or of every tile.
template <Mode MODE>
__device__ __forceinline__ void item_blocks(int t, const Args& p, int kblocks, int& kb0, int& kb1, int& split)
{
    kb0 = 0;
    kb1 = kblocks;
    split = 0;
    if constexpr (MODE == Mode::Dense) {
        if (p.splits > 1) {
            split = t % p.splits;
            kb0 = split * p.sps;
            kb1 = min(kblocks, kb0 + p.sps);
        }
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 8 nibbles (k = 0..7, even k in the low nibble of each byte) -> 4 words of bf16 pairs holding the
// exact integers (code - zero) in natural k order.  A PRMT puts nibble 2b at bits 0-3 and nibble 2b+1
// at bits 16-19; one LOP3 ORs in the exponent of 128.0, which makes the nibble the low mantissa bits,
// and flips bit 3 of symmetric two's-complement codes (code + 8); one packed subtract removes the
// magic plus the zero point (bias2 = magic + zero in both halves).
template <bool SYM>
__device__ __forceinline__ void widen16(uint32_t w, uint32_t bias2, uint32_t (&o)[4])
{
    constexpr uint32_t magic = 0x43004300u;
    constexpr uint32_t key = SYM ? (magic ^ 0x00080008u) : magic;
    const uint32_t u = w >> 4;
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const uint32_t sel = (uint32_t)b | ((uint32_t)b << 4) | ((uint32_t)(4 + b) << 8) | ((uint32_t)(4 + b) << 12);
        const uint32_t t = lop3_and_xor(prmt(w, u, sel), 0x000F000Fu, key);
        o[b] = bf16x2_sub(t, bias2);
    }
}

// 8 symmetric nibbles -> 8 int8 of value 16*code in natural k order (two words): the nibble goes to the
// high half of its byte, which makes the byte the two's-complement value 16*code; the factor 1/16 is
// folded into the (power-of-two exact) scale.
__device__ __forceinline__ void widen_s8x16(uint32_t w, uint32_t& o0, uint32_t& o1)
{
    const uint32_t lo = (w << 4) & 0xF0F0F0F0u;
    const uint32_t hi = w & 0xF0F0F0F0u;
    o0 = prmt(lo, hi, 0x5140u);
    o1 = prmt(lo, hi, 0x7362u);
}

// 8 asymmetric nibbles (codes 0..15) -> 8 int8 of value code - z in natural k order (two words).
// zb holds 128 - z in every byte: code + (128 - z) lies in 113..143, so a plain 32-bit add has no
// carries between bytes, and flipping bit 7 of each byte turns the biased value into the two's
// complement byte of code - z.
__device__ __forceinline__ void widen_s8_asym(uint32_t w, uint32_t zb, uint32_t& o0, uint32_t& o1)
{
    const uint32_t lo = (w & 0x0F0F0F0Fu) + zb;          // codes of even k
    const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) + zb;   // codes of odd k
    o0 = prmt(lo, hi, 0x5140u) ^ 0x80808080u;
    o1 = prmt(lo, hi, 0x7362u) ^ 0x80808080u;
}

__device__ __forceinline__ uint32_t pair16_bits(float v)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(v, v);
    return *reinterpret_cast<const uint32_t*>(&h);
}

struct Shared {
    // per stage: packed weights landed, activations landed (converters wait on both), and the slot
    // free again (MMA commit + the four converter warps of the stage's set)
    uint64_t w_full[kMaxStages], x_full[kMaxStages], xw_empty[kMaxStages];
    // per TMEM slot of widened weights: the MMAs of the slot's last stage have completed.  (The ring's
    // xw_empty cannot stand in for it: with fewer ring stages than TMEM slots, or two converter sets, the
    // ring barrier of stage it - NA can complete a second phase before the converter of stage it looks.)
    uint64_t tmem_free[kMaxNA];
    uint64_t d_full[3], done;
    // progress counters read by the MMA issuer (weak loads): stages converted (and activations landed)
    // per converter warp of each set, groups drained per epilogue warp, W4A8 accumulator preload done
    uint32_t conv_done[4 * kConvSets], epi_done[8], epi_init[8];
    uint32_t slot_free;             // ring stages released so far (published by the slot watcher)
    uint64_t up_ready, gate_done;   // GateUp: gate/up hand-over written (8 epilogue warps); buffer free again (warp 11)
    uint64_t h_ready[2];            // GateUp: a half's h values are in the exchange buffer (its 4 warps)
    uint64_t p_full[2], p_empty[2]; // parameter ring: window staged (loader lanes), window consumed
    uint32_t tmem_base;
    int abort_flag;
    int total_tiles;
    int expert_tiles[kMaxExperts + 1];
    int comb_tok[8 * 64];      // Down: token of each activation row of the tile, per epilogue warp
    float comb_w[8 * 64];      // Down: its routing weight
};
static_assert(sizeof(Shared) <= 6144, "Shared must fit the space reserved in Cfg::SMEM");


template <Mode MODE>
__device__ __forceinline__ Tile map_tile(int t, const Args& p, const Shared* sh, int tiles_m)
{
    Tile T;
    item_blocks<MODE>(t, p, p.K / KBLK, T.kb0, T.kb1, T.split);
    if constexpr (MODE == Mode::Dense) {
        if (p.splits > 1) t /= p.splits;   // the output tile
        T.e = 0;
        T.m0 = (t % tiles_m) * BN;
        T.m_end = p.M;
        T.n0 = (t / tiles_m) * BM;
        T.wrow_a = T.n0;
        T.wrow_b = 0;
    } else {
        int e = 0;
        while (e + 1 < p.E && sh->expert_tiles[e + 1] <= t) e++;
        const int local = t - sh->expert_tiles[e];
        const int nt_per = MODE == Mode::GateUp ? p.N / 64 : p.N / BM;
        const int mt = local / nt_per, nt = local % nt_per;
        T.e = e;
        T.m0 = p.offsets[e] + mt * BN;
        T.m_end = p.offsets[e + 1];
        T.n0 = MODE == Mode::GateUp ? nt * 64 : nt * BM;
        T.wrow_a = e * p.N + T.n0;
        T.wrow_b = T.wrow_a;
    }
    return T;
}

// Scale and zero rows of tile row r (one TMEM lane); nullptr when the row is outside the matrix.
template <Mode MODE>
__device__ __forceinline__ void row_params(const Args& p, const Tile& T, int r, int ng, const __half*& srow,
                                           const __half*& zrow)
{
    if constexpr (MODE == Mode::Dense) {
        const int n = T.n0 + r;
        srow = n < p.N ? p.scales_a + (int64_t)n * ng : nullptr;
        zrow = (n < p.N && p.zeros_a) ? p.zeros_a + (int64_t)n * ng : nullptr;
    } else if constexpr (MODE == Mode::GateUp) {
        const int64_t row = (int64_t)T.e * p.N + T.n0 + (r & 63);
        srow = (r < 64 ? p.scales_a : p.scales_b) + row * ng;
        const __half* z = r < 64 ? p.zeros_a : p.zeros_b;
        zrow = z ? z + row * ng : nullptr;
    } else {
        const int64_t row = (int64_t)T.e * p.N + T.n0 + r;
        srow = p.scales_a + row * ng;
        zrow = p.zeros_a ? p.zeros_a + row * ng : nullptr;
    }
}

// W4A8 epilogue: fp16 scales of one row, n of them, read 4 at a time, one 8-byte block ahead: the
// block for positions [4j, 4j+4) is loaded when position 4j-4 is taken, so a register that is still
// loading is touched (moved) only 4 positions later.  n % 4 != 0 or a row that is not 8-byte aligned (a
// split-K item's slice of the row) falls back to direct loads.
// preload() issues the first block of the next row one tile early, so start() does not wait for it.
struct QuadRing {
    const __half* row = nullptr;
    const __half* pre_row = nullptr;
    int n = 0;
    uint2 cur, nxt, pre;
    bool vec = false;   // 8-byte blocks (count % 4 == 0 and an 8-byte aligned row; else direct loads)
    __device__ __forceinline__ void preload(const __half* r, int count)
    {
        pre_row = (r && (count & 3) == 0 && ((uintptr_t)r & 7) == 0) ? r : nullptr;
        if (pre_row) pre = __ldg(reinterpret_cast<const uint2*>(r));
    }
    __device__ __forceinline__ void start(const __half* r, int count)
    {
        row = r;
        n = count;
        cur = nxt = make_uint2(0u, 0u);
        vec = row && (n & 3) == 0 && ((uintptr_t)row & 7) == 0;
        if (vec) nxt = row == pre_row ? pre : __ldg(reinterpret_cast<const uint2*>(row));
    }
    __device__ __forceinline__ float get(int i)   // positions in increasing order, from 0
    {
        if (!row) return 0.0f;
        if (!vec) return __half2float(row[i]);
        if ((i & 3) == 0) {
            cur = nxt;
            nxt = i + 4 < n ? __ldg(reinterpret_cast<const uint2*>(row + i + 4)) : make_uint2(0u, 0u);
        }
        const uint32_t w = (i & 2) ? cur.y : cur.x;
        return __half2float(__ushort_as_half((unsigned short)((i & 1) ? (w >> 16) : (w & 0xFFFFu))));
    }
};

// PW consecutive fp16 group parameters of one row, from group g0 (zeros past the row's end or for a
// missing row), stored group-major at dst[j * BM].
template <int PW>
__device__ __forceinline__ void stage_params(const __half* row, int g0, int ng, __half* dst)
{
    uint16_t* d = reinterpret_cast<uint16_t*>(dst);
    if (PW % 8 == 0 && row && (ng & 7) == 0 && ((uintptr_t)row & 15) == 0) {
#pragma unroll
        for (int q = 0; q < PW / 8; q++) {
            const uint4 u = g0 + 8 * q < ng ? __ldg(reinterpret_cast<const uint4*>(row + g0 + 8 * q)) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                d[(8 * q + 2 * j) * BM] = (uint16_t)(e[j] & 0xFFFFu);
                d[(8 * q + 2 * j + 1) * BM] = (uint16_t)(e[j] >> 16);
            }
        }
    } else {
#pragma unroll 4
        for (int j = 0; j < PW; j++) d[j * BM] = (row && g0 + j < ng) ? __half_as_ushort(row[g0 + j]) : (uint16_t)0;
    }
}

template <bool INT8, int G, bool SYM, Mode MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wa,
               const __grid_constant__ CUtensorMap tm_wb, Args p)
{
    constexpr bool PRING = !INT8 || !SYM;
    using C = Cfg<INT8, MODE, PRING>;
    // a group narrower than a stage: GPK groups per stage; a wider one (group 256): SPG stages per group
    constexpr int GPK = G <= KBLK ? KBLK / G : 1;
    constexpr int SPG = G > KBLK ? G / KBLK : 1;
    constexpr int GK = G <= KBLK ? G : KBLK;    // K of one group inside one stage
    constexpr int PW = C::PW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr int NS = C::NS;
    uint8_t* xs = smem;                          // NS x XSTAGE (1024-aligned stages)
    uint8_t* wsm = smem + NS * C::XSTAGE;        // NS x WSTAGE
    float* xchg = reinterpret_cast<float*>(wsm + NS * WSTAGE);   // GateUp only
    __half* params = reinterpret_cast<__half*>(wsm + NS * WSTAGE + C::XCHG);   // [slot][scale|zero][PW][BM]
    Shared* sh = reinterpret_cast<Shared*>(wsm + NS * WSTAGE + C::XCHG + C::PARAMS);
    volatile int* abort_flag = &sh->abort_flag;
    int* comb_tok = sh->comb_tok;
    float* comb_w = sh->comb_w;

    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int kblocks = p.K / KBLK, ngroups = p.K / G;
    const int tiles_m = (p.M + BN - 1) / BN;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) {
            tc::mbar_init(&sh->w_full[i], 1);
            tc::mbar_init(&sh->x_full[i], 1);
            tc::mbar_init(&sh->xw_empty[i], 1 + 4);
        }
        for (int i = 0; i < C::ND; i++) tc::mbar_init(&sh->d_full[i], 1);
        for (int i = 0; i < C::NA; i++) tc::mbar_init(&sh->tmem_free[i], 1);
        for (int i = 0; i < 4 * kConvSets; i++) sh->conv_done[i] = 0;
        sh->slot_free = 0;
        for (int i = 0; i < 8; i++) sh->epi_done[i] = sh->epi_init[i] = 0;
        tc::mbar_init(&sh->done, kIssuers);
        // consumers: the converters, and the epilogue unless it is W4A8's
        // parameter windows are released by every converter warp of both sets (and the 16-bit epilogue)
        for (int i = 0; i < 2; i++) {
            tc::mbar_init(&sh->p_full[i], 32);
            tc::mbar_init(&sh->p_empty[i], 4 * kConvSets + (INT8 ? 0 : 8));
        }
        // GateUp exchange: every epilogue warp writes its half of the hand-over (up_ready); warp 11 stores
        // the h values and frees the buffer (gate_done)
        tc::mbar_init(&sh->up_ready, 8);
        tc::mbar_init(&sh->gate_done, 1);
        tc::mbar_init(&sh->h_ready[0], 4);
        tc::mbar_init(&sh->h_ready[1], 4);
        sh->abort_flag = 0;
        if constexpr (MODE == Mode::Dense) sh->total_tiles = tiles_m * ((p.N + BM - 1) / BM) * max(p.splits, 1);
        else sh->total_tiles = p.expert_tiles[p.E] - p.expert_tiles[0];
        tc::fence_mbar_init();
    }
    // (a class of experts passes its slice of the layer's tile prefix sums: counted from its first expert)
    if constexpr (MODE != Mode::Dense)
        for (int i = threadIdx.x; i <= p.E; i += blockDim.x) sh->expert_tiles[i] = p.expert_tiles[i] - p.expert_tiles[0];
    // Dense: the first work item's first parameter window is staged here by every thread, one group row
    // piece each, so its global reads are one round trip instead of the loader warp's one per row it
    // stages (which delayed every launch's first stage by ~2.5 us); the loader then only publishes it
    if constexpr (MODE == Mode::Dense && PRING) {
        const int total0 = tiles_m * ((p.N + BM - 1) / BM) * max(p.splits, 1);
        if ((int)blockIdx.x < total0) {
            const Tile T0 = map_tile<MODE>(blockIdx.x, p, sh, tiles_m);
            const int grp0 = T0.kb0 * GPK, ngr = (T0.kb1 - T0.kb0) * GPK;   // (Dense: SPG == 1)
            constexpr int kPieces = C::PTENS * BM * (PW / 8);                 // tensor x row x 8 groups
            for (int i = threadIdx.x; i < kPieces; i += kThreads) {
                const int ten = i / (BM * (PW / 8)), r = (i / (PW / 8)) % BM, q = i % (PW / 8);
                if (SYM && ten == 1) continue;
                const __half *srow, *zrow;
                row_params<MODE>(p, T0, r, ngroups, srow, zrow);
                const __half* row = ten == 0 ? srow : zrow;
                uint16_t* d = reinterpret_cast<uint16_t*>(params + ten * PW * BM + r);   // window slot 0
                uint16_t v[8];
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int gg = 8 * q + j;
                    v[j] = (row && gg < ngr) ? __half_as_ushort(row[grp0 + gg]) : (uint16_t)0;
                }
#pragma unroll
                for (int j = 0; j < 8; j++) d[(8 * q + j) * BM] = v[j];
            }
        }
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tm_x);
        tc::tma_prefetch_desc(&tm_wa);
        if constexpr (MODE == Mode::GateUp) tc::tma_prefetch_desc(&tm_wb);
    }
    if (warp == 1) tc::tmem_alloc(&sh->tmem_base, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sh->tmem_base;
    const int total = sh->total_tiles;
    // Dense launches use programmatic dependent launch: the next kernel on the stream may start (its
    // prologue and weight copies) while this one runs; it reads this one's outputs only after its own
    // griddepcontrol.wait, which waits for this grid's completion and memory flush
    if constexpr (MODE == Mode::Dense)
        if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int wg = warp / 4;
    if (wg == 2) {
        tc::setmaxnreg_dec<kRegsProd>();
        // ------------------------------------------------------------------ TMA producer (warp 8) and
        // ring-slot watcher (warp 9).  A thread that waits on an mbarrier also waits for its own bulk copies
        // in flight, so the thread that issues the copies never waits on one: the watcher (which issues no
        // copies) waits for each stage's slot to be released (MMA commit + converters) and publishes the
        // count in shared memory, and the producer polls that count with plain loads.
        if (lane == 0 && warp == 9) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                int kb0, kb1, sp;
                item_blocks<MODE>(t, p, kblocks, kb0, kb1, sp);
                for (int kb = kb0; kb < kb1; kb++, it++) {
                    if (!tc::mbar_wait(&sh->xw_empty[it % NS], (it / NS) & 1, p.status, abort_flag)) goto watch_done;
                    tc::sts_publish(&sh->slot_free, it + 1);
                }
            }
        watch_done:;
        } else if (lane == 0 && warp == 8) {
            uint32_t it = 0;
            bool ok = true;
            bool dep_ready = MODE != Mode::Dense;   // (Dense: x may come from the previous kernel)
            for (int t = blockIdx.x; t < total && ok && !*abort_flag; t += gridDim.x) {
                const Tile T = map_tile<MODE>(t, p, sh, tiles_m);
                for (int kb = T.kb0; kb < T.kb1; kb++, it++) {
                    const int s = it % NS;
                    if (it >= (uint32_t)NS) {
                        // stage it - NS, the slot's previous one, has been released
                        if (!(ok = tc::poll_counters<1>(&sh->slot_free, it - NS + 1, p.status, abort_flag))) break;
                        // its readers' accesses (generic and tensor) before this copy's writes (async proxy)
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    }
                    // weights first (small; the converters start on them while the activations land)
                    tc::mbar_arrive_expect_tx(&sh->w_full[s], WSTAGE);
                    uint8_t* wdst = wsm + s * WSTAGE;
                    if constexpr (MODE == Mode::GateUp) {
                        tc::tma_load_2d(wdst, &tm_wa, &sh->w_full[s], kb * (KBLK / 2), T.wrow_a);
                        tc::tma_load_2d(wdst + 64 * 64, &tm_wb, &sh->w_full[s], kb * (KBLK / 2), T.wrow_b);
                    } else {
                        tc::tma_load_2d(wdst, &tm_wa, &sh->w_full[s], kb * (KBLK / 2), T.wrow_a);
                    }
                    tc::mbar_arrive_expect_tx(&sh->x_full[s], C::XSTAGE);
                    uint8_t* xdst = xs + s * C::XSTAGE;
                    if (!dep_ready) {   // the weights above may be read early; the activations only now
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                        dep_ready = true;
                    }
                    if constexpr (INT8) tc::tma_load_2d(xdst, &tm_x, &sh->x_full[s], kb * KBLK, T.m0);
                    else tc::tma_load_3d(xdst, &tm_x, &sh->x_full[s], 0, T.m0, kb * C::XBLK);   // the stage's 64-column blocks
                }
            }
            if (!ok || *abort_flag) {  // let every copy this thread issued land before the CTA can exit
                for (uint32_t j = it > (uint32_t)NS ? it - NS : 0; j < it; j++) {
                    tc::mbar_wait(&sh->w_full[j % NS], (j / NS) & 1, p.status, nullptr, 100000000ull);
                    tc::mbar_wait(&sh->x_full[j % NS], (j / NS) & 1, p.status, nullptr, 100000000ull);
                }
            }
        } else if (MODE == Mode::GateUp && warp == 11) {
            // -------------------------------------------------------------- h stores (warp 11, GateUp)
            // Once both halves of a tile's h are in the exchange buffer, store them by token rows (lanes 0-15
            // token j, lanes 16-31 token j + 1, each lane 4 consecutive intermediate indices: a row's 64 hi
            // values, one 128-byte line, in one store and its 64 lo values in a second, or its 64 fp16
            // values; intermediate index i = n0 + c: hi in block n0 / 64 of the row, lo 64 later, fp16 at
            // column i of an [P][N] row), then free the buffer.  The epilogue warps meanwhile drain the next
            // tile's groups.
            const bool f16 = p.h_f16;
            const int64_t hstride = f16 ? p.N : 2 * p.N;
            const int c4 = 4 * (lane & 15);
            uint32_t tl = 0;
            for (int t = blockIdx.x; t < total; t += gridDim.x, tl++) {
                const Tile T = map_tile<MODE>(t, p, sh, tiles_m);
                for (int hf = 0; hf < 2; hf++) {
                    if (!tc::mbar_wait(&sh->h_ready[hf], tl & 1, p.status, abort_flag)) goto hstore_done;
                    const float* xb = xchg + hf * 64 * 64;
                    const int mb = T.m0 + hf * 64;
                    const int rows = min(64, T.m_end - mb);
#pragma unroll 4
                    for (int pr = 0; pr < 32; pr++) {
                        const int j = 2 * pr + (lane >> 4);
                        if (j >= rows) continue;
                        const float4 hv = *reinterpret_cast<const float4*>(xb + j * 64 + c4);
                        const int64_t o = (int64_t)(mb + j) * hstride + (f16 ? T.n0 : 2 * T.n0) + c4;
                        if (!q4_in_bounds(o + (f16 ? 3 : 67), (int64_t)p.M * hstride, p.status)) continue;
                        if (f16) {
                            const __half2 a = __floats2half2_rn(hv.x, hv.y), b = __floats2half2_rn(hv.z, hv.w);
                            *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(p.h) + o) =
                                make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
                        } else {
                            const __nv_bfloat162 h0 = __floats2bfloat162_rn(hv.x, hv.y), h1 = __floats2bfloat162_rn(hv.z, hv.w);
                            const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
                            const __nv_bfloat162 l0 = __floats2bfloat162_rn(hv.x - f0.x, hv.y - f0.y);
                            const __nv_bfloat162 l1 = __floats2bfloat162_rn(hv.z - f1.x, hv.w - f1.y);
                            *reinterpret_cast<uint2*>(p.h + o) =
                                make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
                            *reinterpret_cast<uint2*>(p.h + o + 64) =
                                make_uint2(*reinterpret_cast<const uint32_t*>(&l0), *reinterpret_cast<const uint32_t*>(&l1));
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sh->gate_done);
            }
        hstore_done:;
        } else if (PRING && warp == 10) {
            // -------------------------------------------------------------- parameter loader (warp 10)
            // Stages each window of PW groups of the tile's scales (and zero points) in shared memory,
            // ahead of the converters and the epilogue, so that their loops make no global loads.
            uint32_t wi = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const Tile T = map_tile<MODE>(t, p, sh, tiles_m);
                // the item's groups (all of the tile's unless K is split)
                const int grp0 = SPG > 1 ? T.kb0 / SPG : T.kb0 * GPK;
                const int ngr = SPG > 1 ? (T.kb1 - T.kb0) / SPG : (T.kb1 - T.kb0) * GPK;
                const int nwin = (ngr + PW - 1) / PW;
                for (int w = 0; w < nwin; w++, wi++) {
                    if (!tc::mbar_wait(&sh->p_empty[wi & 1], ((wi >> 1) & 1) ^ 1, p.status, abort_flag)) goto load_done;
                    __half* ps = params + (wi & 1) * C::PTENS * PW * BM;
#pragma unroll 1
                    for (int i = 0; i < BM / 32 && !(MODE == Mode::Dense && wi == 0); i++) {   // (window 0: staged above)
                        const int r = 32 * i + lane;
                        const __half *srow, *zrow;
                        row_params<MODE>(p, T, r, ngroups, srow, zrow);
                        stage_params<PW>(srow ? srow + grp0 : nullptr, w * PW, ngr, ps + r);
                        if constexpr (!SYM) stage_params<PW>(zrow ? zrow + grp0 : nullptr, w * PW, ngr, ps + PW * BM + r);
                    }
                    tc::mbar_arrive(&sh->p_full[wi & 1]);   // every lane: its stores are visible
                }
            }
        load_done:;
        }
    } else if (wg == 0) {
        tc::setmaxnreg_dec<kRegsIssue>();
        // ------------------------------------------------------------------ MMA issuers (warps 0-3)
        // They wait only by polling progress counters with weak loads (tc::poll_counters), so the tensor
        // pipe never drains between stages; their completions go out through tcgen05.commit, which tracks
        // the issuing thread's own MMAs: every stage is issued and committed by one thread.
        if (lane == 0) {
            constexpr uint32_t idesc = INT8 ? tc::idesc_s8_s32(BN) : tc::idesc_bf16_f32(BN);
            uint32_t it = 0, g = 0;
            bool ok = true;
            if constexpr (INT8) ok = tc::poll_counters<8>(sh->epi_init, 1, p.status, abort_flag);
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                int kb0, kb1, sp;
                item_blocks<MODE>(t, p, kblocks, kb0, kb1, sp);
                for (int kb = kb0; kb < kb1 && ok; kb++, it++) {
                    // (the SPG stages of one group go to one issuer, whose MMAs into the group's accumulator
                    // are then ordered)
                    if ((it / SPG) % kIssuers != (uint32_t)warp) {   // another issuer's stage
                        if (it % SPG == SPG - 1) g += GPK;
                        continue;
                    }
                    const bool g_first = it % SPG == 0, g_last = it % SPG == SPG - 1;
                    const int s = it % NS, sa = it % C::NA;
                    // the stage's weights are widened into TMEM and its activations have landed
                    if (!(ok = tc::poll_counters<4>(sh->conv_done + 4 * (it % kConvSets), it + 1, p.status, abort_flag))) break;
                    tc::fence_after_sync();
                    const uint32_t xaddr = tc::smem_u32(xs + s * C::XSTAGE);
#pragma unroll
                    for (int gi = 0; gi < GPK; gi++) {
                        const uint32_t gg = g + gi;
                        const uint32_t db = gg % C::ND;
                        // accumulator db is free once group gg-ND has been drained
                        if (g_first) {
                            if (!(ok = tc::poll_counters<8>(sh->epi_done, gg >= (uint32_t)C::ND ? gg - C::ND + 1 : 0, p.status,
                                                            abort_flag)))
                                break;
                            tc::fence_after_sync();
                        }
#pragma unroll
                        for (int i = 0; i < GK / C::KI; i++) {
                            const int kk = gi * GK + i * C::KI;   // k offset inside the stage
                            const uint32_t a_tmem = tbase + C::A_COL0 + sa * C::ACOLS + (INT8 ? kk / 4 : kk / 2);
                            uint32_t boff;
                            if constexpr (INT8) boff = kk;                              // one 128-byte row box
                            else boff = (kk / 64) * (C::HILO ? 2 : 1) * (BN * 128) + (kk % 64) * 2;   // 64-column boxes
                            const uint64_t bdesc = tc::smem_desc_sw128(xaddr + (boff & ~127u)) + ((boff & 127u) >> 4);
                            if constexpr (INT8) {
                                tc::mma_i8_ts(tbase + db * BN, a_tmem, bdesc, idesc, true);
                            } else {
                                tc::mma_16_ts(tbase + db * BN, a_tmem, bdesc, idesc, i > 0 || !g_first);
                                if constexpr (C::HILO)   // the lo half of h: the next 64-column box
                                    tc::mma_16_ts(tbase + db * BN, a_tmem, bdesc + ((BN * 128) >> 4), idesc, 1);
                            }
                        }
                        if (g_last) tc::mma_commit(&sh->d_full[db]);
                    }
                    if (g_last) g += GPK;
                    tc::mma_commit(&sh->xw_empty[s]);
                    tc::mma_commit(&sh->tmem_free[sa]);
                }
            }
            tc::mma_commit(&sh->done);   // every MMA of this thread has completed once `done` flips
            // This wait must not honour the abort flag: after another role gave up, the MMAs already
            // issued still read shared memory and write TMEM, and the CTA may leave (and free TMEM) only
            // once they have completed.  Their operands are in place, so they finish; the wall-time limit
            // still bounds the wait.
            tc::mbar_wait(&sh->done, 0, p.status, nullptr);
        }
    } else if (wg == 1 || wg == 5) {
        tc::setmaxnreg_dec<kRegsConv>();
        // ------------------------------------------------------------------ converters (warps 4-7, 20-23)
        // Set cs converts the stages it with it % 2 == cs; both sets walk every stage for the parameter
        // windows, so each releases every window once.
        const int cs = wg == 5 ? 1 : 0;
        const int sub = warp & 3;
        const int r = 32 * sub + lane;                 // row in tile == TMEM lane
        const uint32_t lane_field = (uint32_t)(32 * sub) << 16;
        constexpr float kMagic = 128.0f;
        uint32_t it = 0, wi = 0;   // stage and parameter-window counters (running across tiles)
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            int kb0, kb1, sp;
            item_blocks<MODE>(t, p, kblocks, kb0, kb1, sp);
            const int ngr = SPG > 1 ? (kb1 - kb0) / SPG : (kb1 - kb0) * GPK;   // the item's groups
            for (int kb = kb0; kb < kb1; kb++) {
                const int s = it % NS, sa = it % C::NA;
                // zero points of the stage's groups from the parameter ring
                float zcur[GPK];
#pragma unroll
                for (int gi = 0; gi < GPK; gi++) zcur[gi] = 8.0f;
                if constexpr (PRING) {
                    // the first group of the stage, counted from the item's first group
                    const int g0 = SPG > 1 ? (kb - kb0) / SPG : (kb - kb0) * GPK;
                    const bool gf = kb % SPG == 0, gl_ = kb % SPG == SPG - 1;   // first / last stage of its group
                    if (g0 % PW == 0 && gf && !tc::mbar_wait(&sh->p_full[wi & 1], (wi >> 1) & 1, p.status, abort_flag))
                        goto conv_done;
                    const __half* pz = params + (wi & 1) * C::PTENS * PW * BM + PW * BM + r;
#pragma unroll
                    for (int gi = 0; gi < GPK; gi++) zcur[gi] = SYM ? 8.0f : __half2float(pz[((g0 + gi) % PW) * BM]);
                    if (gl_ && ((g0 + GPK) % PW == 0 || g0 + GPK >= ngr)) {   // the window's last stage: release it
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&sh->p_empty[wi & 1]);
                        wi++;
                    }
                }
                if (it % kConvSets != (uint32_t)cs) {   // the other set's stage
                    it++;
                    continue;
                }
                // one combined wait: the stage's packed weights and activations have landed, and TMEM slot
                // sa is free -- the MMAs of stage it - NA, the slot's previous stage, have completed (that
                // phase cannot be older: this set converted stage it - NA; nor can a newer one have completed:
                // the slot's next stage is this one)
                {
                    uint64_t* slot_bar = it >= (uint32_t)C::NA ? &sh->tmem_free[sa] : &sh->w_full[s];
                    const uint32_t slot_par = it >= (uint32_t)C::NA ? ((it / C::NA) - 1) & 1 : (it / NS) & 1;
                    if (!tc::mbar_wait3(&sh->w_full[s], (it / NS) & 1, &sh->x_full[s], (it / NS) & 1, slot_bar, slot_par,
                                        p.status, abort_flag))
                        goto conv_done;
                }
                uint4 v[4];
                const uint32_t wrow = tc::smem_u32(wsm + s * WSTAGE) + r * 64;
#pragma unroll
                for (int c = 0; c < 4; c++) v[c] = lds128(wrow + ((c ^ ((r >> 1) & 3)) << 4));
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_relaxed(&sh->xw_empty[s]);
                __syncwarp();
                tc::fence_after_sync();
                const uint32_t words[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                            v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
                const uint32_t acol = tbase + lane_field + C::A_COL0 + sa * C::ACOLS;
                if constexpr (INT8) {
                    uint32_t o[32];
                    if constexpr (SYM) {
#pragma unroll
                        for (int w = 0; w < 16; w++) widen_s8x16(words[w], o[2 * w], o[2 * w + 1]);
                    } else {
                        uint32_t zb[GPK];   // 128 - z in every byte
#pragma unroll
                        for (int gi = 0; gi < GPK; gi++) zb[gi] = (uint32_t)(128 - (int)zcur[gi]) * 0x01010101u;
#pragma unroll
                        for (int w = 0; w < 16; w++) widen_s8_asym(words[w], zb[(8 * w) / G], o[2 * w], o[2 * w + 1]);
                    }
                    tc::tmem_st32(acol, o);
                } else {
                    uint32_t bias[GPK];
#pragma unroll
                    for (int gi = 0; gi < GPK; gi++) bias[gi] = pair16_bits(kMagic + zcur[gi]);
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        uint32_t o[32];
#pragma unroll
                        for (int w = 0; w < 8; w++) {
                            const int ww = 8 * h + w;                  // word: k = 8*ww .. 8*ww+7
                            uint32_t q[4];
                            widen16<SYM>(words[ww], bias[(8 * ww) / G], q);
#pragma unroll
                            for (int b = 0; b < 4; b++) o[4 * w + b] = q[b];
                        }
                        tc::tmem_st32(acol + 32 * h, o);
                    }
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                // publish: this warp's rows of the stage are in TMEM, and the stage's activations landed
                __syncwarp();
                if (lane == 0) tc::sts_publish(&sh->conv_done[4 * cs + sub], it + 1);
                it++;
            }
        }
    conv_done:;
    } else {
        tc::setmaxnreg_inc<kRegsEpi>();
        // ------------------------------------------------------------------ epilogue (warps 12-19)
        const int ew = warp - 12;
        const int sub = warp & 3, half = ew >> 2;
        const int r = 32 * sub + lane;
        const uint32_t lane_field = (uint32_t)(32 * sub) << 16;
        uint32_t g = 0, tl = 0;
        // fp32 accumulators in packed pairs: acc2[j] holds the values of columns 2j and 2j+1
        uint64_t acc2[32];
        auto accv = [&](int j) { return (j & 1) ? tc::f2_hi(acc2[j >> 1]) : tc::f2_lo(acc2[j >> 1]); };
        if constexpr (INT8) {
            // Every int32 accumulator starts at the bit pattern of 1.5 * 2^23 (as a float), so after the
            // group's MMAs its bits ARE the float 1.5 * 2^23 + acc (|acc| < 2^22): the epilogue converts
            // with one packed subtraction instead of an integer-to-float conversion per value.
#pragma unroll
            for (int d = 0; d < C::ND; d++)
#pragma unroll
                for (int h = 0; h < 2; h++) tc::tmem_fill32(tbase + lane_field + d * BN + half * 64 + 32 * h, kAccBias);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::sts_publish(&sh->epi_init[ew], 1);
        }
        uint32_t wi = 0;   // parameter-window counter (running across tiles; 16-bit modes)
        QuadRing sr;       // W4A8: group scales read a few groups ahead
        for (int t = blockIdx.x; t < total; t += gridDim.x, tl++) {
            const Tile T = map_tile<MODE>(t, p, sh, tiles_m);
            // the item's groups (all of the tile's unless K is split)
            const int grp0 = SPG > 1 ? T.kb0 / SPG : T.kb0 * GPK;
            const int ngr = SPG > 1 ? (T.kb1 - T.kb0) / SPG : (T.kb1 - T.kb0) * GPK;
            const __half *srow, *zrow;
            row_params<MODE>(p, T, r, ngroups, srow, zrow);
            if constexpr (INT8) {
                sr.start(srow ? srow + grp0 : nullptr, ngr);
                if (t + (int)gridDim.x < total) {   // load the next tile's first block of scales now
                    const Tile Tn = map_tile<MODE>(t + gridDim.x, p, sh, tiles_m);
                    const __half *sn, *zn;
                    row_params<MODE>(p, Tn, r, ngroups, sn, zn);
                    const int g0n = SPG > 1 ? Tn.kb0 / SPG : Tn.kb0 * GPK;
                    sr.preload(sn ? sn + g0n : nullptr, SPG > 1 ? (Tn.kb1 - Tn.kb0) / SPG : (Tn.kb1 - Tn.kb0) * GPK);
                }
            }
#pragma unroll
            for (int j = 0; j < 32; j++) acc2[j] = 0;
            if constexpr (MODE == Mode::Down) {
                // token and routing weight of this warp's 64 activation rows, staged for the tile's output
                for (int j = lane; j < 64; j += 32) {
                    const int m = T.m0 + half * 64 + j;
                    const bool ok = m < T.m_end;
                    comb_tok[ew * 64 + j] = ok ? p.row_tok[m] : 0;
                    float cw = ok ? p.row_w[m] : 0.0f;
                    if constexpr (INT8) cw = ok ? cw * p.scale_a[m] : 0.0f;   // the row's activation scale
                    comb_w[ew * 64 + j] = cw;
                }
            }
            for (int gl = 0; gl < ngr; gl++) {
                const uint32_t db = g % C::ND;
                // group scale: W4A8 from its read-ahead ring, 16-bit modes from the parameter ring
                float s;
                if constexpr (INT8) {
                    s = sr.get(gl);
                } else {
                    if (gl % PW == 0 && !tc::mbar_wait(&sh->p_full[wi & 1], (wi >> 1) & 1, p.status, abort_flag)) goto epi_done;
                    s = __half2float(params[(wi & 1) * C::PTENS * PW * BM + (gl % PW) * BM + r]);
                    if ((gl + 1) % PW == 0 || gl + 1 == ngr) {   // the window's last group: release it
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&sh->p_empty[wi & 1]);
                        wi++;
                    }
                }
                if constexpr (INT8 && SYM) s *= 0.0625f;   // the MMA saw 16 * code
                const uint64_t s2 = tc::f2_pack(__float_as_uint(s), __float_as_uint(s));
                if (!tc::mbar_wait(&sh->d_full[db], (g / C::ND) & 1, p.status, abort_flag)) goto epi_done;
                __syncwarp();
                tc::fence_after_sync();
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    uint32_t v[32];
                    tc::tmem_ld32(tbase + lane_field + db * BN + half * 64 + 32 * h, v);
                    tc::tmem_wait_ld();
                    if constexpr (INT8) {
                        if (MODE == Mode::Dense && p.acc_dbg && srow) {
#pragma unroll
                            for (int j = 0; j < 32; j++) {
                                const int m = T.m0 + half * 64 + 32 * h + j;
                                const int64_t o = ((int64_t)m * p.N + T.n0 + r) * ngroups + grp0 + gl;
                                if (m < T.m_end && q4_in_bounds(o, (int64_t)p.M * p.N * ngroups, p.status))
                                    p.acc_dbg[o] = ((int32_t)(v[j] - kAccBias)) >> (SYM ? 4 : 0);
                            }
                        }
                        const uint64_t nb2 = tc::f2_pack(__float_as_uint(-kAccBiasF), __float_as_uint(-kAccBiasF));
#pragma unroll
                        for (int j = 0; j < 16; j++)
                            acc2[16 * h + j] = tc::f2_fma(s2, tc::f2_add(tc::f2_pack(v[2 * j], v[2 * j + 1]), nb2), acc2[16 * h + j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; j++)
                            acc2[16 * h + j] = tc::f2_fma(s2, tc::f2_pack(v[2 * j], v[2 * j + 1]), acc2[16 * h + j]);
                    }
                }
                if constexpr (INT8) {
                    // hand the columns back pre-loaded for the next group in this buffer
                    tc::tmem_fill32(tbase + lane_field + db * BN + half * 64, kAccBias);
                    tc::tmem_fill32(tbase + lane_field + db * BN + half * 64 + 32, kAccBias);
                    tc::tmem_wait_st();
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::sts_publish(&sh->epi_done[ew], g + 1);   // group g drained
                g++;
            }
            // ---------------------------------------------------------- tile output
            // (every loop below has a branch-free path for a full 64-row block: a conditional branch per
            // row costs more than the store it guards)
            if constexpr (MODE == Mode::Dense) {
                const int n = T.n0 + r;
                const int mb = T.m0 + half * 64;
                const int rows = min(64, p.M - mb);
                if (n < p.N && rows > 0) {
                    const int64_t base = (int64_t)mb * p.N + n;
                    if (p.splits > 1) {   // this split's partial sums, for the split reduction
                        float* pf = p.part + (int64_t)T.split * p.M * p.N + base;
                        const int64_t lim = (int64_t)p.splits * p.M * p.N - ((int64_t)T.split * p.M * p.N + base);
#pragma unroll
                        for (int j = 0; j < 64; j++)
                            if (j < rows) {
                                float v = accv(j);
                                if constexpr (INT8) v *= __ldg(p.scale_a + mb + j);
                                if (q4_in_bounds((int64_t)j * p.N, lim, p.status)) pf[(int64_t)j * p.N] = v;
                            }
                    } else if (p.out_bf16) {
                        __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(p.y) + base;
                        if (rows == 64) {
#pragma unroll
                            for (int j = 0; j < 64; j++) {
                                float v = accv(j);
                                if constexpr (INT8) v *= __ldg(p.scale_a + mb + j);
                                if (q4_in_bounds(base + (int64_t)j * p.N, (int64_t)p.M * p.N, p.status))
                                    yb[(int64_t)j * p.N] = __float2bfloat16_rn(v);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 64; j++)
                                if (j < rows) {
                                    float v = accv(j);
                                    if constexpr (INT8) v *= __ldg(p.scale_a + mb + j);
                                    if (q4_in_bounds(base + (int64_t)j * p.N, (int64_t)p.M * p.N, p.status))
                                        yb[(int64_t)j * p.N] = __float2bfloat16_rn(v);
                                }
                        }
                    } else {
                        float* yf = reinterpret_cast<float*>(p.y) + base;
                        if (rows == 64) {
#pragma unroll
                            for (int j = 0; j < 64; j++) {
                                float v = accv(j);
                                if constexpr (INT8) v *= __ldg(p.scale_a + mb + j);
                                if (q4_in_bounds(base + (int64_t)j * p.N, (int64_t)p.M * p.N, p.status))
                                    yf[(int64_t)j * p.N] = v;
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 64; j++)
                                if (j < rows) {
                                    float v = accv(j);
                                    if constexpr (INT8) v *= __ldg(p.scale_a + mb + j);
                                    if (q4_in_bounds(base + (int64_t)j * p.N, (int64_t)p.M * p.N, p.status))
                                        yf[(int64_t)j * p.N] = v;
                                }
                        }
                    }
                }
            } else if constexpr (MODE == Mode::GateUp) {
                // Rows 0-63 hold gate, rows 64-127 up, of the same 64 intermediate indices.  Both sides
                // share the SwiGLU work: the up rows hand u of tokens 0-31 to the gate rows, the gate rows
                // hand g of tokens 32-63 to the up rows (through shared memory, [token][index]), and each
                // side then evaluates h for its 32 tokens of this warp's 64.
                float* xb = xchg + half * 64 * 64;
                const int ii = r & 63;              // intermediate index within the tile
                const bool up = r >= 64;
                // the buffer is free once both sides consumed the previous tile's values
                if (!tc::mbar_wait(&sh->gate_done, (tl & 1) ^ 1, p.status, abort_flag)) goto epi_done;
                if (up) {
#pragma unroll
                    for (int j = 0; j < 32; j++) xb[j * 64 + ii] = accv(j);
                } else {
#pragma unroll
                    for (int j = 32; j < 64; j++) xb[j * 64 + ii] = accv(j);
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sh->up_ready);
                if (!tc::mbar_wait(&sh->up_ready, tl & 1, p.status, abort_flag)) goto epi_done;
                const int mb = T.m0 + half * 64;
                const int rows = min(64, T.m_end - mb);
                // h of this thread's 32 tokens, written back over the exchanged values it read
                auto silu_mul = [&](int j, float gv, float uv) {
                    if constexpr (INT8) {   // the row's activation scale (rows past the expert's end: none)
                        const float sa = j < rows ? __ldg(p.scale_a + mb + j) : 0.0f;
                        gv *= sa;
                        uv *= sa;
                    }
                    // SiLU(g) = g / (1 + e^-g); the fast quotient's error (~1e-7 relative) is far below the
                    // bf16 hi/lo resolution of h; for g << 0 the divisor is +inf and the quotient -0
                    xb[j * 64 + ii] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                };
                if (up) {
#pragma unroll
                    for (int j = 32; j < 64; j++) silu_mul(j, xb[j * 64 + ii], accv(j));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; j++) silu_mul(j, accv(j), xb[j * 64 + ii]);
                }
                // the h values of this warp's tokens are in the buffer: warp 11 stores them by token rows
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&sh->h_ready[half]);
            } else {
                const int n = T.n0 + r;
                float* yv = reinterpret_cast<float*>(p.y) + n;
                const int rows = min(64, T.m_end - (T.m0 + half * 64));
                __syncwarp();
                if (rows == 64) {
#pragma unroll
                    for (int j = 0; j < 64; j++)
                        if (q4_in_bounds((int64_t)comb_tok[ew * 64 + j] * p.N + n, (int64_t)p.T * p.N, p.status))
                            atomicAdd(yv + (int64_t)comb_tok[ew * 64 + j] * p.N, comb_w[ew * 64 + j] * accv(j));
                } else {
#pragma unroll
                    for (int j = 0; j < 64; j++)
                        if (j < rows &&
                            q4_in_bounds((int64_t)comb_tok[ew * 64 + j] * p.N + n, (int64_t)p.T * p.N, p.status))
                            atomicAdd(yv + (int64_t)comb_tok[ew * 64 + j] * p.N, comb_w[ew * 64 + j] * accv(j));
                }
                __syncwarp();
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

}  // namespace tcg
