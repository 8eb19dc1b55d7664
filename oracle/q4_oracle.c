/*
 * q4_oracle.c -- the ORACLE for the group-wise INT4 linear layers and the INT4 MoE expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and the CPU-baseline leg
 * of the benchmark may load this code.  The product path (the CUDA library) never calls it and
 * shares no code, header, table or constant generator with it.
 *
 * Plain, slow, obviously correct host loops.  Floating results accumulate in fp64 in natural index
 * order.  Compiled without fast-math and with -ffp-contract=off, so every fp32 operation written
 * below is one IEEE operation (the only fused multiply-adds are the explicit fmaf calls of the
 * router, whose order is pinned on purpose).  OpenMP, where present, only splits independent
 * outputs across threads; each output keeps its own fixed loop order, so results do not depend on
 * the thread count.
 *
 * Sources (web pages on the subject; cited by title and section):
 *   [INT4MoE]   "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" and its English summary
 *               "Practical Exploration of Efficient LLM Inference: Integration of INT4 Quantization
 *               and MoE Architecture" -- group quantization with per-group scales; SwiGLU FFN
 *               experts behind a gating network.
 *   [FP32toINT4] "从FP32到INT4：大语言模型量化压缩实战指南", §1.3 分组量化技术解析 -- groups get
 *               their own min/max; a zero point only for the asymmetric form.
 *   [W4A8]      "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析", §2.1 (4-bit storage),
 *               §2.3 (offline INT4 quantize with scale and zero; INT4 widened to INT8; INT8 matmul
 *               into INT32; rescale by scale_w*scale_a), §3.1 (per-token amax/127 activation
 *               quantization with round and clamp to [-128,127]), §3.2 (router kept in high
 *               precision, softmax outputs).
 *   [DenseMoE]  "大模型之Dense、MoE与量化", section 混合专家架构 MoE -- a Linear router scores the
 *               experts, a few are chosen, their outputs are recombined in proportion.
 *
 * Readings where the pages are silent (each is stated beside the code that takes it):
 *   - groups run along K (the reduction dimension) inside one output row;
 *   - symmetric: scale = amax/7 in fp32, stored as fp16 (round-to-nearest-even), the STORED value is
 *     used for coding; codes = clamp(rne(w/S), -8, 7), stored as 4-bit two's complement;
 *   - asymmetric: the range always includes 0 (mn = min(min w, 0), mx = max(max w, 0)),
 *     scale = (mx-mn)/15, z = clamp(rne(-mn/S), 0, 15), code = clamp(rne(w/S) + z, 0, 15); the zero
 *     point is an integer stored exactly in fp16;
 *   - packing: element k of a row sits in byte k/2, even k in the low nibble;
 *   - a group whose stored scale is 0 codes every element to the zero point;
 *   - activation quantization divides by the fp32 scale (not a multiply by 127/amax); amax == 0
 *     gives scale 0 and all codes 0;
 *   - W4A8 with group-wise weight scales keeps one INT32 partial per (token, row, group) and
 *     rescales each before summing;
 *   - router logits are fp32 with a pinned reduction order (below), top-k selection by logit,
 *     ties to the lower expert id, weights = softmax over the chosen logits (equal to softmax over
 *     all experts followed by renormalisation over the chosen ones);
 *   - the permutation lists (token, slot) pairs grouped by expert, tokens ascending inside each
 *     expert (a stable counting sort).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_SHAPE (-2)
#define ORC_ERR_UNSUPPORTED (-4)
#define ORC_ERR_NONFINITE (-7)

/* ---------------------------------------------------------------------------------------------
 * Number formats.
 * fp16: IEEE 754 binary16, 1 sign, 5 exponent (bias 15), 10 fraction bits.
 * bf16: the upper 16 bits of an IEEE binary32.
 * ------------------------------------------------------------------------------------------- */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* fp32 -> fp16 bits, round to nearest, ties to even (IEEE 754 default rounding), with subnormals,
 * overflow to infinity and NaN kept quiet. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t u = f32_bits(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t exp = (u >> 23) & 0xFFu;
    uint32_t man = u & 0x7FFFFFu;
    if (exp == 0xFFu) return (uint16_t)(sign | 0x7C00u | (man ? 0x200u : 0u));
    int e = (int)exp - 127;            /* unbiased exponent of a normal fp32 */
    if (exp == 0) return sign;         /* fp32 subnormals are far below fp16's smallest subnormal */
    uint32_t full = man | 0x800000u;   /* 24-bit significand, value = full * 2^(e-23) */
    if (e > 15) return (uint16_t)(sign | 0x7C00u);
    if (e >= -14) {
        /* normal fp16: keep 11 significant bits, drop 13 */
        uint32_t keep = full >> 13, rest = full & 0x1FFFu;
        if (rest > 0x1000u || (rest == 0x1000u && (keep & 1u))) keep++;
        /* keep is in [2^10, 2^11]; 2^11 carries into the exponent */
        uint32_t he = (uint32_t)(e + 15);
        if (keep == 0x800u) { keep = 0x400u; he++; }
        if (he >= 31) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | (he << 10) | (keep & 0x3FFu));
    }
    /* subnormal fp16: value = m * 2^-24 with m < 2^10; m = full * 2^(e-23+24) = full >> (-e-1) */
    int shift = -e - 1;                /* >= 14 */
    if (shift > 25) return sign;       /* below half the smallest subnormal: rounds to zero */
    uint32_t keep = full >> shift;
    uint32_t rest = full & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rest > half || (rest == half && (keep & 1u))) keep++;
    return (uint16_t)(sign | keep);    /* keep == 2^10 lands exactly on the smallest normal */
}

float orc_f16_to_f32(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t exp = (h >> 10) & 0x1Fu, man = h & 0x3FFu;
    if (exp == 0x1Fu) return bits_f32(sign | 0x7F800000u | (man << 13));
    if (exp == 0) {                    /* zero or subnormal: man * 2^-24, exact in fp32 */
        float v = (float)man * 0x1p-24f;
        return sign ? -v : v;
    }
    return bits_f32(sign | ((exp + 112u) << 23) | (man << 13));
}

float orc_bf16_to_f32(uint16_t b) { return bits_f32((uint32_t)b << 16); }

/* Round to nearest integer, ties to even, in fp32 (the rounding of torch.round in [W4A8] §3.1). */
static float rne(float v) { return nearbyintf(v); }

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ---------------------------------------------------------------------------------------------
 * RTN group quantization + packing.  [INT4MoE] INT4量化实现 (4-bit integers, one scale per group);
 * [FP32toINT4] §1.3 (each group its own min/max; zero point only when asymmetric);
 * [W4A8] §2.3 step 1 (offline: INT4 codes, scale and zero); §2.1 (two 4-bit codes per byte).
 * w: fp32 [n][k] row-major; packed: [n][k/2]; scales, zeros: fp16 bits [n][k/group].
 * zeros may be NULL for symmetric.  Returns ORC_ERR_NONFINITE if a group has a non-finite value
 * or its scale overflows fp16 (outputs then undefined).
 * ------------------------------------------------------------------------------------------- */
int orc_quantize(const float* w, int n, int k, int group, int symmetric,
                 uint8_t* packed, uint16_t* scales, uint16_t* zeros)
{
    if (n < 0 || k <= 0 || group <= 0 || k % group || group % 2) return ORC_ERR_SHAPE;
    int ng = k / group, bad = 0;
    for (int r = 0; r < n; r++) {
        for (int g = 0; g < ng; g++) {
            const float* src = w + (size_t)r * k + (size_t)g * group;
            int codes_local[1024];
            int* codes = group <= 1024 ? codes_local : (int*)malloc(sizeof(int) * group);
            float S;
            int z = 0;
            if (symmetric) {
                float amax = 0.0f;
                for (int i = 0; i < group; i++) {
                    float a = fabsf(src[i]);
                    if (!isfinite(src[i])) bad = 1;
                    if (a > amax) amax = a;
                }
                float s32 = amax / 7.0f;
                uint16_t s16 = orc_f32_to_f16(s32);
                S = orc_f16_to_f32(s16);
                if (!isfinite(S)) bad = 1;
                scales[(size_t)r * ng + g] = s16;
                if (zeros) zeros[(size_t)r * ng + g] = 0;
                for (int i = 0; i < group; i++)
                    codes[i] = S == 0.0f ? 0 : (int)clampf(rne(src[i] / S), -8.0f, 7.0f);
            } else {
                float mn = 0.0f, mx = 0.0f;   /* the range always contains 0 */
                for (int i = 0; i < group; i++) {
                    if (!isfinite(src[i])) bad = 1;
                    if (src[i] < mn) mn = src[i];
                    if (src[i] > mx) mx = src[i];
                }
                float s32 = (mx - mn) / 15.0f;
                uint16_t s16 = orc_f32_to_f16(s32);
                S = orc_f16_to_f32(s16);
                if (!isfinite(S)) bad = 1;
                if (S == 0.0f) {
                    z = 0;
                    for (int i = 0; i < group; i++) codes[i] = 0;
                } else {
                    z = (int)clampf(rne(-mn / S), 0.0f, 15.0f);
                    /* round first, then add the integer zero point */
                    for (int i = 0; i < group; i++)
                        codes[i] = (int)clampf(rne(src[i] / S) + (float)z, 0.0f, 15.0f);
                }
                scales[(size_t)r * ng + g] = s16;
                if (zeros) zeros[(size_t)r * ng + g] = orc_f32_to_f16((float)z);
            }
            for (int i = 0; i < group; i += 2) {
                size_t kk = (size_t)g * group + i;
                packed[(size_t)r * (k / 2) + kk / 2] =
                    (uint8_t)((codes[i] & 0xF) | ((codes[i + 1] & 0xF) << 4));
            }
            if (codes != codes_local) free(codes);
        }
    }
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

/* The integer code of element (r, kk): two's complement nibble when symmetric, 0..15 otherwise. */
static int code_at(const uint8_t* packed, int k, int r, int kk, int symmetric)
{
    uint8_t b = packed[(size_t)r * (k / 2) + kk / 2];
    int v = (kk & 1) ? (b >> 4) : (b & 0xF);
    if (symmetric && v >= 8) v -= 16;
    return v;
}

void orc_unpack_codes(const uint8_t* packed, int n, int k, int symmetric, int8_t* codes)
{
    for (int r = 0; r < n; r++)
        for (int kk = 0; kk < k; kk++)
            codes[(size_t)r * k + kk] = (int8_t)code_at(packed, k, r, kk, symmetric);
}

/* Dequantized weight: (q - z) * S, exact in fp32 (a 5-bit integer times an 11-bit significand). */
static float deq_at(const uint8_t* packed, const uint16_t* scales, const uint16_t* zeros,
                    int k, int group, int symmetric, int r, int kk)
{
    int g = kk / group, ng = k / group;
    float S = orc_f16_to_f32(scales[(size_t)r * ng + g]);
    float z = (symmetric || !zeros) ? 0.0f : orc_f16_to_f32(zeros[(size_t)r * ng + g]);
    return ((float)code_at(packed, k, r, kk, symmetric) - z) * S;
}

void orc_dequant(const uint8_t* packed, const uint16_t* scales, const uint16_t* zeros,
                 int n, int k, int group, int symmetric, float* out)
{
    for (int r = 0; r < n; r++)
        for (int kk = 0; kk < k; kk++)
            out[(size_t)r * k + kk] = deq_at(packed, scales, zeros, k, group, symmetric, r, kk);
}

/* ---------------------------------------------------------------------------------------------
 * W4A16 linear: y[m][n] = sum_k x[m][k] * dequant(W)[n][k], fp64, k ascending.
 * [W4A8] §2.1 (4-bit storage restored to a 16-bit type before the multiply); [INT4MoE] 量化实现.
 * x: bf16 bits [M][k].  rows_m / rows_n (nullable) select a sample of outputs: y is then
 * [n_m][n_n] for the listed (m, n) pairs; NULL means all.
 * ------------------------------------------------------------------------------------------- */
void orc_linear_w4a16(const uint16_t* x, int M, int k,
                      const uint8_t* packed, const uint16_t* scales, const uint16_t* zeros,
                      int n, int group, int symmetric,
                      const int32_t* rows_m, int n_m, const int32_t* rows_n, int n_n, double* y)
{
    int cm = rows_m ? n_m : M, cn = rows_n ? n_n : n;
#pragma omp parallel for schedule(dynamic, 1)
    for (int jn = 0; jn < cn; jn++) {
        int r = rows_n ? rows_n[jn] : jn;
        double* wrow = (double*)malloc(sizeof(double) * (size_t)k);
        for (int kk = 0; kk < k; kk++)
            wrow[kk] = (double)deq_at(packed, scales, zeros, k, group, symmetric, r, kk);
        for (int im = 0; im < cm; im++) {
            int mi = rows_m ? rows_m[im] : im;
            const uint16_t* xr = x + (size_t)mi * k;
            double acc = 0.0;
            for (int kk = 0; kk < k; kk++) acc += (double)orc_bf16_to_f32(xr[kk]) * wrow[kk];
            y[(size_t)im * cn + jn] = acc;
        }
        free(wrow);
    }
}

/* ---------------------------------------------------------------------------------------------
 * Per-token INT8 activation quantization.  [W4A8] §3.1: amax over the token's row, scale =
 * amax/127, round half to even, clamp to [-128, 127].  The division is fp32.
 * x: bf16 bits [M][k] -> q int8 [M][k], s fp32 [M].
 * ------------------------------------------------------------------------------------------- */
/* One token's row, already widened to fp32 (exactly): returns the scale, writes the codes. */
static float act_quant_row(const float* v, int k, int8_t* q, int* bad)
{
    float amax = 0.0f;
    for (int kk = 0; kk < k; kk++) {
        if (!isfinite(v[kk])) *bad = 1;
        if (fabsf(v[kk]) > amax) amax = fabsf(v[kk]);
    }
    float sc = amax / 127.0f;
    for (int kk = 0; kk < k; kk++)
        q[kk] = sc == 0.0f ? 0 : (int8_t)clampf(rne(v[kk] / sc), -128.0f, 127.0f);
    return sc;
}

int orc_act_quant(const uint16_t* x, int M, int k, int8_t* q, float* s)
{
    int bad = 0;
    float* v = (float*)malloc(sizeof(float) * (size_t)k);
    for (int mi = 0; mi < M; mi++) {
        for (int kk = 0; kk < k; kk++) v[kk] = orc_bf16_to_f32(x[(size_t)mi * k + kk]);
        s[mi] = act_quant_row(v, k, q + (size_t)mi * k, &bad);
    }
    free(v);
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

/* The same quantization of fp16 rows (the library's act_quant_per_token_f16 entry point):
 * x: fp16 bits [M][k], widened to fp32 exactly. */
int orc_act_quant_f16(const uint16_t* x, int M, int k, int8_t* q, float* s)
{
    int bad = 0;
    float* v = (float*)malloc(sizeof(float) * (size_t)k);
    for (int mi = 0; mi < M; mi++) {
        for (int kk = 0; kk < k; kk++) v[kk] = orc_f16_to_f32(x[(size_t)mi * k + kk]);
        s[mi] = act_quant_row(v, k, q + (size_t)mi * k, &bad);
    }
    free(v);
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

/* ---------------------------------------------------------------------------------------------
 * W4A8 linear.  [W4A8] §2.3: INT4 codes widened to INT8, INT8 x INT8 products accumulated in
 * INT32, result rescaled by scale_w * scale_a.  With one weight scale per group the INT32 partial
 * is kept per (token, row, group):
 *   acc[m][n][g] = sum_{k in g} xq[m][k] * (q[n][k] - z[n][g])     (exact int32)
 *   y[m][n]      = sum_g acc[m][n][g] * scale_w[n][g] * scale_a[m]   (fp64)
 * Symmetric weights: codes -8..7, z = 0.  Asymmetric weights ([W4A8] §2.3's pseudo-code carries a
 * weight zero point next to the scale): codes 0..15 and the group's integer zero point z, so the
 * widened INT8 weight is q - z in [-15, 15].
 * ------------------------------------------------------------------------------------------- */
void orc_linear_w4a8(const int8_t* xq, const float* s_a, int M, int k,
                     const uint8_t* packed, const uint16_t* scales, const uint16_t* zeros, int symmetric,
                     int n, int group, const int32_t* rows_m, int n_m, const int32_t* rows_n, int n_n,
                     int32_t* acc_out, double* y)
{
    int cm = rows_m ? n_m : M, cn = rows_n ? n_n : n, ng = k / group;
#pragma omp parallel for schedule(dynamic, 1)
    for (int jn = 0; jn < cn; jn++) {
        int r = rows_n ? rows_n[jn] : jn;
        for (int im = 0; im < cm; im++) {
            int mi = rows_m ? rows_m[im] : im;
            double sum = 0.0;
            for (int g = 0; g < ng; g++) {
                int32_t acc = 0;
                const int32_t z = symmetric ? 0 : (int32_t)orc_f16_to_f32(zeros[(size_t)r * ng + g]);
                for (int kk = g * group; kk < (g + 1) * group; kk++)
                    acc += (int32_t)xq[(size_t)mi * k + kk] * ((int32_t)code_at(packed, k, r, kk, symmetric) - z);
                if (acc_out) acc_out[((size_t)im * cn + jn) * ng + g] = acc;
                sum += (double)acc * (double)orc_f16_to_f32(scales[(size_t)r * ng + g]) * (double)s_a[mi];
            }
            y[(size_t)im * cn + jn] = sum;
        }
    }
}

/* ---------------------------------------------------------------------------------------------
 * Router.  [DenseMoE] 混合专家架构: a Linear scores every expert, a few are picked, outputs are
 * recombined in proportion; [W4A8] §3.2: the router output goes through softmax and is kept in
 * high precision.
 * Logits, fp32 with a PINNED order so that a GPU can reproduce them bit for bit:
 *   32 partial sums p_l (l = 0..31), p_l = fma chain over k = l, l+32, l+64, ... (ascending),
 *   starting from +0; then p_l <- p_l + p_(l xor s) for s = 16, 8, 4, 2, 1; logit = p_0 (+ bias_e).
 * Top-k by (logit descending, expert id ascending); slot j holds the j-th best.
 * Weights (fp64): w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the chosen i.
 * x: bf16 bits [T][H]; Wr fp32 [E][H]; bias fp32 [E] or NULL.
 * Outputs: logits fp32 [T][E] (nullable), ids [T][topk], w [T][topk], counts [E] (nullable).
 * ------------------------------------------------------------------------------------------- */
float orc_router_logit(const uint16_t* xrow, const float* wrow, int H)
{
    float p[32];
    for (int l = 0; l < 32; l++) {
        p[l] = 0.0f;
        for (int kk = l; kk < H; kk += 32) p[l] = fmaf(orc_bf16_to_f32(xrow[kk]), wrow[kk], p[l]);
    }
    for (int s = 16; s >= 1; s >>= 1) {
        float q[32];
        for (int l = 0; l < 32; l++) q[l] = p[l] + p[l ^ s];
        memcpy(p, q, sizeof(p));
    }
    return p[0];
}

int orc_route(const uint16_t* x, int T, int H, const float* Wr, const float* bias, int E, int topk,
              float* logits_out, int32_t* ids, double* w, int32_t* counts)
{
    if (topk < 1 || topk > E) return ORC_ERR_SHAPE;
    int bad = 0;
    if (counts) for (int e = 0; e < E; e++) counts[e] = 0;
    float* lg = (float*)malloc(sizeof(float) * (size_t)E * (size_t)(T > 0 ? T : 1));
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            float v = orc_router_logit(x + (size_t)t * H, Wr + (size_t)e * H, H);
            if (bias) v = v + bias[e];
            lg[(size_t)t * E + e] = v;
        }
    for (int t = 0; t < T; t++) {
        const float* l = lg + (size_t)t * E;
        for (int e = 0; e < E; e++) if (!isfinite(l[e])) bad = 1;
        if (logits_out) memcpy(logits_out + (size_t)t * E, l, sizeof(float) * E);
        /* selection: repeatedly take the best expert not taken yet */
        char* taken = (char*)calloc((size_t)E, 1);
        for (int j = 0; j < topk; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict '>' keeps the lower id on ties */
            }
            taken[best] = 1;
            ids[(size_t)t * topk + j] = best;
            if (counts) counts[best]++;
        }
        free(taken);
        double l0 = (double)l[ids[(size_t)t * topk]], den = 0.0;
        for (int j = 0; j < topk; j++) den += exp((double)l[ids[(size_t)t * topk + j]] - l0);
        for (int j = 0; j < topk; j++)
            w[(size_t)t * topk + j] = exp((double)l[ids[(size_t)t * topk + j]] - l0) / den;
    }
    free(lg);
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

/* ---------------------------------------------------------------------------------------------
 * Dispatch order (token permutation by expert).  [W4A8] §1 (routing dispatch and merge cost
 * extra); [DenseMoE] 缺点 (tokens are dispatched to different experts).
 * Stable counting sort of the T*topk pairs (t, j) by expert id:
 *   offsets[e] = number of pairs with expert < e (offsets[E] = T*topk);
 *   pairs of one expert are listed with t ascending; perm[pos] = t*topk + j.
 * ------------------------------------------------------------------------------------------- */
void orc_permute(const int32_t* ids, int T, int topk, int E, int32_t* offsets, int32_t* perm)
{
    int32_t* cnt = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
    for (int p = 0; p < T * topk; p++) cnt[ids[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + cnt[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int t = 0; t < T; t++)
        for (int j = 0; j < topk; j++) {
            int e = ids[(size_t)t * topk + j];
            perm[offsets[e] + fill[e]++] = t * topk + j;
        }
    free(cnt);
    free(fill);
}

/* ---------------------------------------------------------------------------------------------
 * MoE SwiGLU expert FFN layer.  [INT4MoE] MoE架构设计 (each expert is a small feed-forward
 * network behind a gating network; the base model's FFN is SwiGLU); [DenseMoE] 混合专家架构
 * (proportional recombination).  For token t and each chosen expert e = ids[t][j]:
 *   g = x_t . dequant(Wg_e)^T,  u = x_t . dequant(Wu_e)^T           (length I, fp64)
 *   h = g / (1 + exp(-g)) * u                                       (SiLU(g) * u, fp64)
 *   o = h . dequant(Wd_e)^T                                         (length H, fp64)
 * h stays fp64 between the two projections: the pages define the expert as a SwiGLU FFN and fix no
 * storage precision for its intermediate, so the plain reading is the mathematical value; how a
 * kernel carries h is its own choice, held to the output tolerance.
 *   y_t = sum_j w[t][j] * o                                         (fp64)
 * Expert weights are stacked: gate/up packed [E*I][H/2], scales/zeros [E*I][H/group];
 * down packed [E*H][I/2], scales/zeros [E*H][I/group].
 * tokens (nullable) lists the tokens to evaluate; y is [n_tok][H] (all T when NULL).  The routing
 * ids and weights come in from orc_route.
 * ------------------------------------------------------------------------------------------- */
void orc_moe_experts(const uint16_t* x, int T, int H, const int32_t* ids, const double* w, int topk,
                     const uint8_t* g_packed, const uint16_t* g_scales, const uint16_t* g_zeros,
                     const uint8_t* u_packed, const uint16_t* u_scales, const uint16_t* u_zeros,
                     const uint8_t* d_packed, const uint16_t* d_scales, const uint16_t* d_zeros,
                     int I, int group, int symmetric,
                     const int32_t* tokens, int n_tok, double* y)
{
    int cnt = tokens ? n_tok : T;
    size_t gH = (size_t)(H / group), gI = (size_t)(I / group);
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < cnt; it++) {
        int t = tokens ? tokens[it] : it;
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        double* yr = y + (size_t)it * H;
        for (int c = 0; c < H; c++) { xr[c] = (double)orc_bf16_to_f32(x[(size_t)t * H + c]); yr[c] = 0.0; }
        for (int j = 0; j < topk; j++) {
            int e = ids[(size_t)t * topk + j];
            /* the expert's row blocks inside the stacked matrices */
            const uint8_t* gp = g_packed + (size_t)e * I * (H / 2);
            const uint8_t* up = u_packed + (size_t)e * I * (H / 2);
            const uint16_t* gs = g_scales + (size_t)e * I * gH;
            const uint16_t* us = u_scales + (size_t)e * I * gH;
            const uint16_t* gz = g_zeros ? g_zeros + (size_t)e * I * gH : NULL;
            const uint16_t* uz = u_zeros ? u_zeros + (size_t)e * I * gH : NULL;
            for (int i = 0; i < I; i++) {
                double gv = 0.0, uv = 0.0;
                for (int c = 0; c < H; c++) {
                    gv += xr[c] * (double)deq_at(gp, gs, gz, H, group, symmetric, i, c);
                    uv += xr[c] * (double)deq_at(up, us, uz, H, group, symmetric, i, c);
                }
                h[i] = gv / (1.0 + exp(-gv)) * uv;
            }
            const uint8_t* dp = d_packed + (size_t)e * H * (I / 2);
            const uint16_t* ds = d_scales + (size_t)e * H * gI;
            const uint16_t* dz = d_zeros ? d_zeros + (size_t)e * H * gI : NULL;
            double wj = w[(size_t)t * topk + j];
            for (int c = 0; c < H; c++) {
                double o = 0.0;
                for (int i = 0; i < I; i++) o += h[i] * (double)deq_at(dp, ds, dz, I, group, symmetric, c, i);
                yr[c] += wj * o;
            }
        }
        free(xr);
        free(h);
    }
}

/* ---------------------------------------------------------------------------------------------
 * MoE expert FFN with INT8 activations.  [W4A8] §3.1 (per-token INT8 activations), §2.3 (INT8 x
 * INT4-widened-to-INT8 products in INT32, rescaled by scale_w * scale_a), §3.2 (the router stays in
 * high precision: routing ids and weights come in from orc_route unchanged), §5.1 (the projections
 * of an FFN can take different precisions: the down projection is the first to go W4A8).
 * a8_mask bit 0: gate and up run W4A8 on the token's INT8 codes (one quantization of x_t serves every
 * expert the token visits); bit 1: down runs W4A8 on the INT8 codes of h.  For token t, slot j,
 * e = ids[t][j]:
 *   bit 0 set:   xq, sa = act_quant(x_t);
 *                g_i = sum_g sa * sg[i][g] * sum_{k in g} xq[k] * (qg[i][k] - zg[i][g])   (fp64
 *                of the exact INT32 partials), u_i likewise with the up matrix;
 *   bit 0 clear: g, u as in orc_moe_experts (fp64 over the dequantized weights);
 *   h = g / (1 + exp(-g)) * u (fp64), as in orc_moe_experts;
 *   bit 1 set:   hq, sh = act_quant(h16) over the row's I values, h16 = fp16(fp32(h)): §3.1's per-token
 *                quantizer takes the layer's 16-bit activation tensor (fp16, the pages' activation
 *                format) as its input, so the down projection's INT8 activations are the codes of h as an
 *                fp16 activation; then
 *                o_c = sum_g sh * sd[c][g] * sum_{i in g} hq[i] * (qd[c][i] - zd[c][g]);
 *   bit 1 clear: o = h . dequant(Wd_e)^T (fp64, as orc_moe_experts);
 *   y_t = sum_j w[t][j] * o (fp64).
 * Returns ORC_ERR_NONFINITE when a quantized row holds a non-finite value.
 * ------------------------------------------------------------------------------------------- */
static double w4a8_dot(const int8_t* aq, double sa, const uint8_t* packed, const uint16_t* scales,
                       const uint16_t* zeros, int symmetric, int k, int group, int r)
{
    int ng = k / group;
    double sum = 0.0;
    for (int g = 0; g < ng; g++) {
        int32_t acc = 0;
        const int32_t z = (symmetric || !zeros) ? 0 : (int32_t)orc_f16_to_f32(zeros[(size_t)r * ng + g]);
        for (int kk = g * group; kk < (g + 1) * group; kk++)
            acc += (int32_t)aq[kk] * ((int32_t)code_at(packed, k, r, kk, symmetric) - z);
        sum += (double)acc * (double)orc_f16_to_f32(scales[(size_t)r * ng + g]) * sa;
    }
    return sum;
}

int orc_moe_experts_a8(const uint16_t* x, int T, int H, const int32_t* ids, const double* w, int topk,
                       const uint8_t* g_packed, const uint16_t* g_scales, const uint16_t* g_zeros,
                       const uint8_t* u_packed, const uint16_t* u_scales, const uint16_t* u_zeros,
                       const uint8_t* d_packed, const uint16_t* d_scales, const uint16_t* d_zeros,
                       int I, int group, int symmetric, int a8_mask,
                       const int32_t* tokens, int n_tok, double* y)
{
    int cnt = tokens ? n_tok : T;
    size_t gH = (size_t)(H / group), gI = (size_t)(I / group);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int it = 0; it < cnt; it++) {
        int t = tokens ? tokens[it] : it;
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        int8_t* xq = (int8_t*)malloc((size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        float* hf = (float*)malloc(sizeof(float) * (size_t)I);
        int8_t* hq = (int8_t*)malloc((size_t)I);
        double* yr = y + (size_t)it * H;
        int rb = 0;
        for (int c = 0; c < H; c++) { xf[c] = orc_bf16_to_f32(x[(size_t)t * H + c]); yr[c] = 0.0; }
        double sa = (a8_mask & 1) ? (double)act_quant_row(xf, H, xq, &rb) : 0.0;
        for (int j = 0; j < topk; j++) {
            int e = ids[(size_t)t * topk + j];
            const uint8_t* gp = g_packed + (size_t)e * I * (H / 2);
            const uint8_t* up = u_packed + (size_t)e * I * (H / 2);
            const uint16_t* gs = g_scales + (size_t)e * I * gH;
            const uint16_t* us = u_scales + (size_t)e * I * gH;
            const uint16_t* gz = g_zeros ? g_zeros + (size_t)e * I * gH : NULL;
            const uint16_t* uz = u_zeros ? u_zeros + (size_t)e * I * gH : NULL;
            for (int i = 0; i < I; i++) {
                double gv = 0.0, uv = 0.0;
                if (a8_mask & 1) {
                    gv = w4a8_dot(xq, sa, gp, gs, gz, symmetric, H, group, i);
                    uv = w4a8_dot(xq, sa, up, us, uz, symmetric, H, group, i);
                } else {
                    for (int c = 0; c < H; c++) {
                        gv += (double)xf[c] * (double)deq_at(gp, gs, gz, H, group, symmetric, i, c);
                        uv += (double)xf[c] * (double)deq_at(up, us, uz, H, group, symmetric, i, c);
                    }
                }
                h[i] = gv / (1.0 + exp(-gv)) * uv;
            }
            const uint8_t* dp = d_packed + (size_t)e * H * (I / 2);
            const uint16_t* ds = d_scales + (size_t)e * H * gI;
            const uint16_t* dz = d_zeros ? d_zeros + (size_t)e * H * gI : NULL;
            double wj = w[(size_t)t * topk + j];
            double sh = 0.0;
            for (int i = 0; i < I; i++) hf[i] = orc_f16_to_f32(orc_f32_to_f16((float)h[i]));
            if (a8_mask & 2) sh = (double)act_quant_row(hf, I, hq, &rb);
            for (int c = 0; c < H; c++) {
                double o = 0.0;
                if (a8_mask & 2) o = w4a8_dot(hq, sh, dp, ds, dz, symmetric, I, group, c);
                else for (int i = 0; i < I; i++) o += h[i] * (double)deq_at(dp, ds, dz, I, group, symmetric, c, i);
                yr[c] += wj * o;
            }
        }
        bad |= rb;
        free(xf);
        free(xq);
        free(h);
        free(hf);
        free(hq);
    }
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

int orc_version(void) { return 1; }
