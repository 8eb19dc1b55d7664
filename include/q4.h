/*
 * q4.h -- C ABI of the group-wise INT4 linear layers and the INT4 MoE expert FFN for NVIDIA B200
 * (sm_100a).  Library: moe_linear_layers_b200/libq4.so.
 *
 * The calls follow the problem as the source pages state it:
 *   - "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" (below: the W4A8 page) §2.3: weights are
 *     quantized offline to INT4 with a scale and a zero point; at run time INT4 is widened to INT8,
 *     multiplied with INT8 activations into INT32, and rescaled by scale_w*scale_a; §3.1: per-token
 *     activation quantization from amax/127; §2.1: 4-bit storage restored to a 16-bit type for
 *     W4A16;
 *   - "从FP32到INT4：大语言模型量化压缩实战指南" §1.3: group-wise quantization, each group its own
 *     range, a zero point only for the asymmetric form;
 *   - "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" (INT4 group quantization; MoE experts
 *     are small SwiGLU FFNs behind a gating network) and "大模型之Dense、MoE与量化" section
 *     混合专家架构 MoE (a Linear router scores experts, a few are chosen, their outputs are
 *     recombined in proportion).
 *
 * Conventions for every call:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise.  The caller owns every
 *     buffer and no call allocates device memory: scratch space of the MoE layer is the caller's
 *     workspace (the one exception, moe_q4_forward_noalloc, uses a fixed array that exists from the
 *     moment the library is loaded).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Every call is
 *     asynchronous on it.
 *   - The return value reports errors the host can see before launching (null pointers, shapes,
 *     alignment, unsupported options, workspace too small, a failed launch).  When it is not Q4_OK
 *     nothing was launched (except Q4_ERR_CUDA, which reports a failed launch).
 *   - `dev_status` (nullable) is a device int32 the kernels set, with the first error seen, when
 *     they detect a problem in the data: Q4_ERR_NONFINITE for a non-finite input group/row,
 *     Q4_ERR_TIMEOUT when a bounded wait inside a kernel ran out.  The library never clears it;
 *     the caller zeroes it and reads it when convenient.  Outputs are undefined when it is set.
 *   - A problem without rows (m = 0 in the linear and activation calls, n = 0 in the quantizer,
 *     T = 0 tokens, R = 0 rows) is valid: the call checks its sizes, options and weights, zeroes the
 *     expert offsets and counts it is given, and launches nothing else.  Pointers to arrays that then
 *     hold no elements (x, y, the per-token and per-row arrays, the quantizer's four) may be NULL.
 *     The decode GEMV calls (q4_linear_w4a16_grouped, q4_linear_w4a16_swiglu, q4_linear_w4a16_chain)
 *     take 1 <= m <= 4.
 *   - fp16 and bf16 values are passed as their 16-bit patterns (uint16_t).
 *   - Matrices are row-major.
 *
 * Data layout of an INT4 weight W [n][k] (groups of `group` consecutive elements along k):
 *   packed [n][k/2] u8   element k of a row is in byte k/2, even k in the low nibble;
 *                        symmetric codes are 4-bit two's complement (-8..7, -8 never produced),
 *                        asymmetric codes are 0..15;
 *   scales [n][k/group]  fp16;
 *   zeros  [n][k/group]  fp16 holding an integer 0..15 (asymmetric only; NULL when symmetric).
 * Dequantized weight = (code - zero) * scale.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    Q4_OK = 0,
    Q4_ERR_NULL = -1,        /* a required pointer is NULL */
    Q4_ERR_SHAPE = -2,       /* a size is out of range or inconsistent */
    Q4_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
    Q4_ERR_UNSUPPORTED = -4, /* an option this build does not implement */
    Q4_ERR_WORKSPACE = -5,   /* workspace too small */
    Q4_ERR_CUDA = -6,        /* a CUDA call failed (launch error) */
    Q4_ERR_NONFINITE = -7,   /* (device) non-finite input, or a scale that overflows fp16 */
    Q4_ERR_TIMEOUT = -8,     /* (device) a bounded wait inside a kernel gave up */
    Q4_ERR_BOUNDS = -9       /* (device, debug build only) a computed index fell outside its buffer */
} q4_status;

enum { Q4_OUT_F32 = 0, Q4_OUT_BF16 = 1 };

/* Descriptor of one INT4 weight matrix (all pointers device pointers, 16-byte aligned). */
typedef struct q4_weight {
    int32_t n, k;        /* rows (output features) and columns (input features) */
    int32_t group;       /* 64 or 128 (32 and 256 for the MoE entry points' 16-bit expert GEMMs); k % group == 0 */
    int32_t symmetric;   /* 1: codes -8..7, zeros == NULL; 0: codes 0..15 with zeros */
    const uint8_t* packed;
    const uint16_t* scales;
    const uint16_t* zeros;
} q4_weight;

/* Human-readable name of a status code (static string). */
const char* q4_status_string(int status);

/* Library version (increments with the ABI). */
int q4_version(void);

/* Description of the last CUDA error behind a Q4_ERR_CUDA return on the calling host thread. */
const char* q4_last_cuda_error_string(void);

/*
 * Build flags of the loaded library: bit 0 set in the debug build (libq4_debug.so, compiled with
 * Q4_DEBUG), whose kernels check every global-memory index they compute against the extent of its buffer
 * and, instead of making the access, record Q4_ERR_BOUNDS in dev_status.  The debug build stands in for
 * a memory checker; it computes the same results as the release build, more slowly.
 */
int q4_build_flags(void);

/*
 * q4_quantize_pack -- round-to-nearest group quantization and packing of an fp32 matrix.
 * Source: the W4A8 page §2.3 (offline INT4 quantization keeping scale and zero point) and §2.1
 * (4-bit storage); "从FP32到INT4" §1.3 (per-group range; zero point only when asymmetric).
 *   symmetric:  S = fp16(amax/7);            code = clamp(rne(w/S), -8, 7)
 *   asymmetric: mn = min(min w, 0), mx = max(max w, 0), S = fp16((mx-mn)/15),
 *               z = clamp(rne(-mn/S), 0, 15), code = clamp(rne(w/S) + z, 0, 15)
 * All divisions are IEEE fp32; rne = round half to even; the STORED fp16 scale codes the group;
 * a group whose scale is 0 codes to its zero point.
 * w [n][k] fp32 (16-byte aligned); packed [n][k/2]; scales [n][k/group]; zeros [n][k/group]
 * (required when symmetric == 0, ignored otherwise).  group in {32, 64, 128, 256}; k % group == 0 (groups
 * 32 and 256 serve the MoE layer's expert matrices; the dense linear entry points take 64 and 128).
 * dev_status: Q4_ERR_NONFINITE when a group holds a non-finite value or its scale overflows fp16.
 */
int q4_quantize_pack(const float* w, int32_t n, int32_t k, int32_t group, int32_t symmetric,
                     uint8_t* packed, uint16_t* scales, uint16_t* zeros,
                     int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a16 -- y = x . dequant(W)^T with the dequantization fused in the kernel.
 * Source: the W4A8 page §2.1 (4-bit storage restored to a 16-bit compute type) and §1 (small batch:
 * memory bound; larger batch: compute bound).
 * x [m][k] bf16; y [m][n] fp32 (out_dtype Q4_OUT_F32) or bf16 (Q4_OUT_BF16, round to nearest even of
 * the fp32 result).  m >= 0 (m = 0 launches nothing).  Small m runs the memory-bound GEMV kernel
 * (CUDA cores, in-register dequant); larger m runs the tcgen05 tensor-core GEMM (exact integer codes
 * in bf16, fp32 accumulation per group, scale applied per group in the epilogue).  The choice is by shape only.
 * The GEMV serves k % 64 == 0, k <= 16384; the GEMM serves k % 128 == 0 (see q4_linear_w4a16_max_gemv_m).
 * Both kernels may start, and read W (packed, scales, zeros) into shared memory, TMEM and L2, before the
 * previous kernel on the stream has finished (programmatic dependent launch); they read x and write y
 * only after that kernel's writes are visible.  So W must not be written by the immediately preceding
 * kernel when that kernel releases its dependents early (none of this library's kernels that write
 * weights does).  Inside the GEMV, x is taken per 64-value block as int16 with a power-of-two scale
 * (each value kept to 2^-15 of its block's largest magnitude) and the dot products are exact in int32.
 * dev_status: Q4_ERR_NONFINITE when x holds a non-finite value (GEMV path).
 */
int q4_linear_w4a16(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                    int32_t* dev_status, void* stream);

/*
 * q4_linear_workspace_size -- bytes of device workspace with which q4_linear_w4a16_ws and
 * q4_linear_w4a8_ws split a tensor-core GEMM of these sizes along K (0: the shape is not split; a
 * library convenience, not a step of the pages' method).  A problem whose 128 x 128 output tiles fill
 * fewer than half of the GPU's SMs is cut into K ranges of at least two 128-K blocks, so that every SM
 * gets work; each range stores its fp32 partial sums in the workspace and a second kernel adds them
 * in range order (the result does not depend on the timing).  0 for m < 1, n < 1 or k % 128 != 0.
 */
size_t q4_linear_workspace_size(int32_t m, const q4_weight* w);

/*
 * q4_linear_w4a16_ws -- q4_linear_w4a16 with a caller workspace (nullable; device memory, 256-byte
 * aligned, at least q4_linear_workspace_size(m, w) bytes, else Q4_ERR_ALIGN / Q4_ERR_WORKSPACE).  The
 * library owns it during the call (kernels on `stream`); it needs no initial contents.  Without a
 * workspace, or for a shape that is not split, this is q4_linear_w4a16.  The split form computes the
 * same per-group products; only the order of the fp32 additions across K ranges differs.
 */
int q4_linear_w4a16_ws(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a16_grouped -- up to 8 independent small-m W4A16 products in one launch:
 * y[i] = x[i] . dequant(W[i])^T for i < count, each exactly as q4_linear_w4a16 with m <= 4 computes it.
 * Source: as q4_linear_w4a16; the grouping is a launch-level choice (independent linears of one layer
 * -- q, k, v, or gate and up -- need not wait for each other), not part of the method.
 * x, w, y are HOST arrays of `count` entries (device pointers / descriptors).  Every w[i] has the
 * same k (k % 64 == 0, k <= 16384), group and symmetry; n may differ.  1 <= m <= 4, the same for all.
 */
int q4_linear_w4a16_grouped(int32_t count, const uint16_t* const* x, int32_t m, const q4_weight* w,
                            void* const* y, int32_t out_dtype, int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a16_swiglu -- the down projection of a dense SwiGLU FFN at small m, with the gating
 * fused into its input: y[m][n] = sum_k h[m][k] * dequant(W)[n][k], h = silu(gate) * up =
 * gate / (1 + e^-gate) * up, computed in fp32 from the gate and up projections' fp32 outputs.
 * Source: "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" MoE架构设计 (experts and the base
 * model's FFN are SwiGLU); the fusion is a launch-level choice (h is never written to memory).
 * gate, up: fp32 [m][k], 16-byte aligned; 1 <= m <= 4; k % 64 == 0, k <= 16384.  h is carried like
 * x in q4_linear_w4a16's GEMV (int16 per 64-value block with a power-of-two scale, one binade lower
 * so that no fp32 value rounds out of range).  dev_status: Q4_ERR_NONFINITE when an h is not finite.
 */
int q4_linear_w4a16_swiglu(const float* gate, const float* up, int32_t m, const q4_weight* w, void* y,
                           int32_t out_dtype, int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a16_chain -- a chain of DEPENDENT stages of m = 1 W4A16 GEMVs in one launch (a decode step:
 * per layer [q, k, v], o, [gate, up], down).
 * Source: the W4A8 page §2.1 (4-bit storage restored before the multiply) and §1 (small model, small
 * batch: memory bound); "高效大语言模型推理实践：INT4量化与MoE架构的融合探索" MoE架构设计 (the FFN is
 * SwiGLU: a stage may take silu(gate) * up as its input).  Each problem computes exactly what
 * q4_linear_w4a16 computes at m = 1; the chain only orders the work: stage s reads its inputs only after
 * every output of stages 0 .. s-1 is written, so an input may be (or be gated from) an earlier output.
 * Inside the launch the weights of later stages are already streaming while a stage waits.
 *   stage_begin: HOST array of n_stages + 1 ints, 0 = stage_begin[0] < ... ; stage s holds problems
 *                stage_begin[s] .. stage_begin[s+1]-1 (1 to 8 problems with the same k).
 *   x, gate, up, w, y: HOST arrays of count = stage_begin[n_stages] entries (device pointers / descriptors).
 *                x[i]: bf16 [k]; or, when gate and up are given and gate[i] != NULL, problem i's input is
 *                silu(gate[i]) * up[i] from fp32 [k] vectors (then x may be NULL or x[i] ignored).
 *                gate and up may be NULL (no gated problem).  y[i]: [n] in out_dtype.
 *   Every w[i] has the same group and symmetry, k % 64 == 0, k <= 16384, n >= 1.  n_stages <= 128,
 *   count <= 256.
 *   sync: device memory of q4_linear_w4a16_chain_sync_bytes(n_stages) bytes (a 128-byte line per stage
 *   counter, so that the stages' counters do not share cache lines), 4-byte aligned, ZERO before
 *   the first call; the kernel leaves it zero on completion, so calls (and graph replays) on one stream can
 *   reuse it.  Calls sharing a sync buffer must not overlap on the GPU.
 * The launch is cooperative (every CTA resident at once: one per SM); the library's other launches need
 * not be.  dev_status: Q4_ERR_NONFINITE for a non-finite input; Q4_ERR_TIMEOUT when a stage wait ran out
 * (the other CTAs then stop too) -- outputs are undefined and the sync buffer must be zeroed again.
 */
size_t q4_linear_w4a16_chain_sync_bytes(int32_t n_stages);
int q4_linear_w4a16_chain(int32_t n_stages, const int32_t* stage_begin, const uint16_t* const* x,
                          const float* const* gate, const float* const* up, const q4_weight* w, void* const* y,
                          int32_t out_dtype, uint32_t* sync, int32_t* dev_status, void* stream);

/*
 * q4_selftest_bounded_wait -- exercises the bounded waits the kernels rely on (no counterpart in the
 * source pages; a test hook for the failure-detection path).  Launches one small kernel whose wait is
 * never satisfied: which = 0 an mbarrier phase no thread completes, 1 a progress counter no thread
 * raises (the issuers' weak-load polling).  After limit_us microseconds (1 .. 1000000) the wait gives
 * up and records Q4_ERR_TIMEOUT in *dev_status (required); the context stays usable.
 */
int q4_selftest_bounded_wait(int32_t which, int32_t limit_us, int32_t* dev_status, void* stream);

/* Largest m that q4_linear_w4a16 serves with the GEMV kernel. */
int q4_linear_w4a16_max_gemv_m(void);

/*
 * act_quant_per_token -- per-token INT8 quantization of bf16 activations.
 * Source: the W4A8 page §3.1: amax over the token, scale = amax/127, round half to even, clamp to
 * [-128, 127].  scale_a[m] = amax/127 (fp32 division); xq = clamp(rne(x / scale_a), -128, 127);
 * a token with amax == 0 gets scale 0 and all-zero codes.
 * x [m][k] bf16; xq [m][k] int8; scale_a [m] fp32.  k % 8 == 0.
 * dev_status: Q4_ERR_NONFINITE when a token holds a non-finite value.
 */
int act_quant_per_token(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                        int32_t* dev_status, void* stream);

/*
 * act_quant_per_token_f16 -- act_quant_per_token for fp16 rows (the same arithmetic on values widened
 * exactly from fp16), for activations a caller keeps in fp16.  x [m][k] fp16 bits; everything else as
 * act_quant_per_token.
 */
int act_quant_per_token_f16(const uint16_t* x, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                            int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a8 -- INT8 activations x INT4 weights widened to INT8, INT32 accumulation, rescale.
 * Source: the W4A8 page §2.3 (three steps and the pseudo-code: dequant_int4_to_int8, int8 matmul
 * into int32, rescale by scale_w * scale_a).  With one weight scale per group of 128 (or 64) the
 * INT32 partial is kept per (token, row, group):
 *   acc[m][n][g] = sum_{k in g} xq[m][k] * (code[n][k] - zero[n][g])   (exact int32)
 *   y[m][n]      = scale_a[m] * sum_g scale_w[n][g] * acc[m][n][g]     (fp32)
 * Symmetric W: codes -8..7, zero 0.  Asymmetric W (the page's pseudo-code keeps a weight zero point
 * beside the scale): codes 0..15 and integer zero points 0..15, so the widened INT8 weight is
 * code - zero in [-15, 15].  y [m][n] fp32 or bf16.  acc_dbg (nullable): [m][n][k/group] int32 copy
 * of the partials, for verification only (slow).  k % 128 == 0.
 */
int q4_linear_w4a8(const int8_t* xq, const float* scale_a, int32_t m, const q4_weight* w, void* y,
                   int32_t out_dtype, int32_t* acc_dbg, int32_t* dev_status, void* stream);

/*
 * q4_linear_w4a8_ws -- q4_linear_w4a8 with a caller workspace, exactly as q4_linear_w4a16_ws (the INT32
 * partials are unchanged: each group lies in one K range; the ranges' sums are times scale_a already).
 */
int q4_linear_w4a8_ws(const int8_t* xq, const float* scale_a, int32_t m, const q4_weight* w, void* y,
                      int32_t out_dtype, int32_t* acc_dbg, void* workspace, size_t workspace_bytes,
                      int32_t* dev_status, void* stream);

/*
 * moe_q4_workspace_size -- bytes of device workspace moe_q4_forward needs for these sizes.
 */
size_t moe_q4_workspace_size(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk);

/*
 * moe_q4_forward -- top-k routed MoE layer of SwiGLU experts with INT4 weights (W4A16).
 * Source: "大模型之Dense、MoE与量化" 混合专家架构 MoE (Linear router, a few experts per token,
 * proportional recombination); the W4A8 page §3.2 (router kept in high precision, softmax output)
 * and §1 (dispatch and merge cost); "高效大语言模型推理实践" MoE架构设计 (each expert a small FFN,
 * SwiGLU as in the base model).
 *   logits[t][e] = fp32 dot(x_t, router_w[e]) in a pinned order (+ router_bias[e]):
 *                  32 partial sums over k = l (mod 32), each an fma chain with k ascending,
 *                  combined by the butterfly p_l + p_(l xor s), s = 16, 8, 4, 2, 1;
 *   ids[t][j]    = the topk experts by (logit descending, id ascending), slot j = j-th best;
 *   w[t][j]      = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the chosen (= softmax, renormalised);
 *   perm/offsets = stable counting sort of the pairs (t, j) by expert (tokens ascending);
 *   h            = SiLU(x . Wg_e^T) * (x . Wu_e^T) in fp32, carried to the down projection as two bf16
 *                  values hi = bf16(h), lo = bf16(h - hi) (h to about 2^-17 of its magnitude; the down
 *                  projection multiplies both);  o = h . Wd_e^T;
 *   y[t]         = sum_j w[t][j] * o_(t,j).
 * x [T][H] bf16; router_w [E][H] fp32; router_bias [E] fp32 or NULL.
 * experts[3] = {gate, up, down}: gate and up are [E*I][H] stacked by expert (rows e*I .. e*I+I-1),
 * down is [E*H][I]; all three with the same group (256, 128, 64, or 32) and symmetry.
 * y [T][H] fp32 or bf16.  Optional outputs (nullable): topk_ids [T][topk] int32, topk_w [T][topk]
 * fp32, perm [T*topk] int32 (value t*topk+j), offsets [E+1] int32, expert_counts [E] int32.
 * workspace: device memory of at least moe_q4_workspace_size(T, H, I, E, topk) bytes, 256-byte
 * aligned, owned by the caller; contents on entry are ignored.
 * Limits: E <= 256, topk <= 16, T * topk <= 2^31 - 1 (pair positions are int32), H % 128 == 0,
 * I % 128 == 0.
 */
int moe_q4_forward(const uint16_t* x, int32_t T, int32_t H,
                   const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                   const q4_weight* experts, int32_t I,
                   void* y, int32_t out_dtype,
                   int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                   void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_ex -- moe_q4_forward with an optional shared expert.
 * Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" and "高效大语言模型推理实践" MoE architecture
 * sections (a shared expert that every token passes through, beside the routed ones).
 *   y[t] = sum_j w[t][j] * o_(t,j) + S(x_t),  S(x) = (SiLU(x . Wg_s^T) * (x . Wu_s^T)) . Wd_s^T,
 * the shared expert a SwiGLU FFN of intermediate I_shared computed like a routed expert (h as a bf16
 * hi/lo pair, fp32 accumulation into the same output sums) with routing weight 1.
 * shared[3] = {gate, up, down} of one expert: gate and up [I_shared][H], down [H][I_shared], the
 * same group and symmetry as the routed experts; NULL (with I_shared ignored) = no shared expert.
 * I_shared % 128 == 0.  Every other argument as moe_q4_forward; the workspace must hold
 * moe_q4_workspace_size_ex(T, H, I, E, topk, I_shared) bytes.
 */
size_t moe_q4_workspace_size_ex(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk, int32_t I_shared);
int moe_q4_forward_ex(const uint16_t* x, int32_t T, int32_t H,
                      const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                      const q4_weight* experts, int32_t I, const q4_weight* shared, int32_t I_shared,
                      void* y, int32_t out_dtype,
                      int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_a8 -- moe_q4_forward with the expert projections on INT8 activation codes (W4A8).
 * Source: the W4A8 page §3.1 (per-token INT8 activations: scale = amax/127, round half to even),
 * §2.3 (INT4 codes widened to INT8, INT8 x INT8 products in INT32, rescale by scale_w * scale_a),
 * §3.2 (the router is not quantized: routing is exactly moe_q4_forward's) and §5.1 (the projections
 * of an FFN take their own precision; the down projection is the first candidate for W4A8).
 *   a8_mask bit 0 (gate/up): xq_t, sa_t = act_quant(x_t) once per token;
 *                g_i = sa_t * sum_g sg[i][g] * P_g, P_g = sum_{k in g} xq_t[k] * (code_g[i][k] - zero_g[i][g])
 *                (exact INT32 partials, fp32 rescale), u likewise;
 *   a8_mask bit 1 (down): h as an fp16 activation (§3.1 quantizes the layer's 16-bit activations) ->
 *                hq, sh = act_quant(fp16(h)) per permuted row (I values), and
 *                o_c = sh * sum_g sd[c][g] * sum_{i in g} hq[i] * (code_d[c][i] - zero_d[c][g]);
 *   a clear bit keeps that projection W4A16 as in moe_q4_forward.  a8_mask in 0..3 (0 = moe_q4_forward).
 *   The INT8 projections take groups 64 and 128 (groups 32 and 256 only with a8_mask 0: Q4_ERR_UNSUPPORTED).
 * Arguments as moe_q4_forward; the workspace must hold moe_q4_workspace_size_a8(T, H, I, E, topk,
 * a8_mask) bytes.  dev_status also receives Q4_ERR_NONFINITE when a quantized row (x or h) holds a
 * non-finite value.
 */
size_t moe_q4_workspace_size_a8(int32_t T, int32_t H, int32_t I, int32_t E, int32_t topk, int32_t a8_mask);
int moe_q4_forward_a8(const uint16_t* x, int32_t T, int32_t H,
                      const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                      const q4_weight* experts, int32_t I, int32_t a8_mask,
                      void* y, int32_t out_dtype,
                      int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_classes -- moe_q4_forward with the experts split into classes, each with its own
 * quantization group size and symmetry.
 * Source: the W4A8 page §5.3 (group size by how often an expert is chosen: smaller groups, i.e. more
 * scales and less error, for the experts most tokens go to, larger groups for rarely chosen ones) and
 * §5.2 (rarely chosen experts can take coarser quantization).
 * Class c holds experts class_begin[c] .. class_begin[c+1]-1 (expert ids as the router numbers them;
 * order the experts so that each class is a contiguous id range); its weights are experts[3c],
 * experts[3c+1], experts[3c+2] = gate [E_c*I][H], up [E_c*I][H], down [E_c*H][I] stacked by the
 * class's experts in id order, with one group (256, 128, 64 or 32) and symmetry shared by the three.
 * class_begin: host array of n_classes + 1 ints, class_begin[0] = 0 < ... < class_begin[n_classes] = E.
 * The layer computes exactly moe_q4_forward's function with each expert's matrices dequantized with
 * its class's parameters.  Every other argument, the workspace size and the limits as moe_q4_forward.
 */
int moe_q4_forward_classes(const uint16_t* x, int32_t T, int32_t H,
                           const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                           int32_t n_classes, const int32_t* class_begin, const q4_weight* experts, int32_t I,
                           void* y, int32_t out_dtype,
                           int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_range -- the part of the MoE layer that one range of experts contributes: the unit of
 * expert parallelism.
 * Source: "大模型之Dense、MoE与量化" 混合专家架构 MoE (the layer is a routing-weighted sum over experts, so
 * it splits into per-expert terms); the W4A8 page §1 (spreading experts over devices trades memory for
 * communication).
 *   y[t] = sum over slots j with e_begin <= ids[t][j] < e_end of w[t][j] * o_(t,j)   (fp32, [T][H])
 * Routing and the permutation are the whole layer's (every token is routed over all E experts);
 * experts[3] = {gate [n*I][H], up [n*I][H], down [n*H][I]} stacked over the n = e_end - e_begin experts
 * of the range.  Ranks that own disjoint ranges covering 0 .. E-1 and sum their y (an all-reduce) obtain
 * moe_q4_forward's output.  0 <= e_begin < e_end <= E; group 32, 64, 128 or 256; everything else as
 * moe_q4_forward (fp32 output only, the workspace of moe_q4_workspace_size).
 */
int moe_q4_forward_range(const uint16_t* x, int32_t T, int32_t H,
                         const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                         int32_t e_begin, int32_t e_end, const q4_weight* experts, int32_t I, float* y,
                         int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * The MoE layer's steps as separate calls: the units of expert parallelism in its all-to-all form (each
 * rank routes its own tokens, sends every routed row to the rank that owns its expert, runs its experts
 * on the rows it receives and sends the results back, where they are combined in token order).
 * Source: "大模型之Dense、MoE与量化" 混合专家架构 MoE and its 缺点 paragraph (tokens are dispatched to
 * different experts, whose outputs are recombined in proportion); the W4A8 page §1 (dispatch and merge
 * cost extra).  Together the three calls compute exactly moe_q4_forward's function.
 *
 * moe_q4_route -- routing (as moe_q4_forward: pinned fp32 logits, top-k with ties to the lower id,
 * softmax over the chosen) and the permutation (stable counting sort of the (token, slot) pairs by expert).
 *   Outputs (required): topk_ids [T][topk] int32, topk_w [T][topk] fp32, offsets [E+1] int32 (the
 *   permuted rows of expert e are offsets[e] .. offsets[e+1]-1), pair_pos [T*topk] int32 (the permuted
 *   position of pair (t, j) at index t*topk + j).  Optional (nullable): x_perm [T*topk][H] bf16 (token rows
 *   in permuted order: the dispatch buffer, whose rows for the experts e0 .. e1-1 are one contiguous block),
 *   row_expert [T*topk] int32 (the expert of each permuted row), perm [T*topk] int32 (value t*topk + j),
 *   expert_counts [E].  workspace: moe_q4_route_workspace_size(T, E, topk) bytes, 256-byte aligned.
 *   Limits as moe_q4_forward (E <= 256, topk <= 16, T * topk <= 2^31 - 1, H % 128 == 0).
 */
size_t moe_q4_route_workspace_size(int32_t T, int32_t E, int32_t topk);
int moe_q4_route(const uint16_t* x, int32_t T, int32_t H, const float* router_w, const float* router_bias,
                 int32_t E, int32_t topk, int32_t* topk_ids, float* topk_w, int32_t* offsets, int32_t* pair_pos,
                 uint16_t* x_perm, int32_t* row_expert, int32_t* perm, int32_t* expert_counts,
                 void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_rows -- the expert FFN on R rows that were routed elsewhere:
 *   y_rows[r] = row_weight[r] * (SiLU(x_r . Wg_e^T) * (x_r . Wu_e^T)) . Wd_e^T,  e = row_expert[r] - e_base,
 * computed exactly as moe_q4_forward's expert GEMMs compute a routed row (h as a bf16 hi/lo pair).
 * x_rows [R][H] bf16; row_expert [R] int32 in [e_base, e_base + E); row_weight [R] fp32 or NULL (1);
 * experts[3] = {gate [E*I][H], up [E*I][H], down [E*H][I]} stacked over the E local experts; y_rows [R][H]
 * fp32.  workspace: moe_q4_rows_workspace_size(R, H, I, E) bytes, 256-byte aligned.  dev_status:
 * Q4_ERR_SHAPE when a row's expert id is outside the range (that row then contributes zeros).
 */
size_t moe_q4_rows_workspace_size(int32_t R, int32_t H, int32_t I, int32_t E);
int moe_q4_forward_rows(const uint16_t* x_rows, int32_t R, int32_t H, const int32_t* row_expert, int32_t e_base,
                        const float* row_weight, int32_t E, const q4_weight* experts, int32_t I, float* y_rows,
                        void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * moe_q4_combine -- the weighted combine in token order: y[t] = sum_j topk_w[t][j] * o_rows[pair_pos[t*topk+j]]
 * (fp32, slot order j, deterministic).  o_rows [P][H] fp32 (the expert outputs in permuted order);
 * pair_pos, topk_w as moe_q4_route returns them; y [T][H] fp32 or bf16.  H % 4 == 0.  dev_status:
 * Q4_ERR_SHAPE when a position is outside [0, P) (that term is left out).
 */
int moe_q4_combine(const float* o_rows, int32_t P, int32_t H, const int32_t* pair_pos, const float* topk_w,
                   int32_t T, int32_t topk, void* y, int32_t out_dtype, int32_t* dev_status, void* stream);

/*
 * moe_q4_forward_noalloc -- moe_q4_forward for callers that cannot allocate device memory.
 * No counterpart in the source pages: this is a library convenience, not part of the method.
 *
 * Some callers have no way to obtain device memory for the workspace: a plugin loaded into a host
 * application that owns all device memory and hands out no allocator, or a latency-critical loop in
 * which a cudaMalloc (which can synchronise the device) is not acceptable.  This entry point takes the
 * same arguments as moe_q4_forward minus the workspace, and uses instead one fixed scratch array that
 * the library holds in device memory (a file-scope __device__ array of Q4_MOE_NOALLOC_SCRATCH_BYTES,
 * 256-byte aligned).  Every GPU on which the library is loaded holds that array until the process
 * exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *   - Sizes whose moe_q4_workspace_size(T, H, I, E, topk) exceeds Q4_MOE_NOALLOC_SCRATCH_BYTES are
 *     rejected with Q4_ERR_WORKSPACE before anything is launched (for H = 2048, I = 1024, E = 64,
 *     top-8 that is T > 453 tokens).
 *   - The first call on a device looks up the array's device address with cudaGetSymbolAddress while
 *     that device is current, and caches it (per device and driver context: after a device reset the
 *     next call looks it up again); make that first call on each device before any stream capture
 *     begins.
 *   - All calls share the one array, which keeps the last call's contents (every call overwrites
 *     what it reads).  Calls that overlap on the GPU (for example on two streams) race on it: keep
 *     them ordered on one stream or serialise them.
 */
#define Q4_MOE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

int moe_q4_forward_noalloc(const uint16_t* x, int32_t T, int32_t H,
                           const float* router_w, const float* router_bias, int32_t E, int32_t topk,
                           const q4_weight* experts, int32_t I,
                           void* y, int32_t out_dtype,
                           int32_t* topk_ids, float* topk_w, int32_t* perm, int32_t* offsets, int32_t* expert_counts,
                           int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
