// Host side of the C ABI: argument validation and dispatch by shape.  See include/q4.h.
#include "q4_common.cuh"

int q4_gemv_w4a16_launch_group(int count, const uint16_t* const* x, int32_t m, const q4_weight* w, void* const* y,
                               int32_t out_dtype, int32_t* dev_status, cudaStream_t stream,
                               const float* const* g = nullptr, const float* const* u = nullptr);
size_t q4_gemm_workspace_bytes(int32_t m, int32_t n, int32_t k);
int q4_gemm_tc_launch(const void* x, const float* scale_a, int32_t m, const q4_weight* w, void* y,
                      int32_t out_dtype, int32_t* acc_dbg, bool int8_path, int32_t* dev_status,
                      cudaStream_t stream, void* workspace);

namespace {
constexpr int kMaxGemvM = 4;

int check_weight(const q4_weight* w, bool need_sym)
{
    if (!w || !w->packed || !w->scales) return Q4_ERR_NULL;
    if (!w->symmetric && !w->zeros) return Q4_ERR_NULL;
    if (w->n < 0 || w->k <= 0 || (w->group != 64 && w->group != 128) || w->k % w->group) return Q4_ERR_SHAPE;
    if (need_sym && !w->symmetric) return Q4_ERR_UNSUPPORTED;
    if (!q4_aligned16(w->packed) || !q4_aligned16(w->scales) || (!w->symmetric && !q4_aligned16(w->zeros)))
        return Q4_ERR_ALIGN;
    return Q4_OK;
}
}  // namespace

extern "C" const char* q4_status_string(int status)
{
    switch (status) {
        case Q4_OK: return "ok";
        case Q4_ERR_NULL: return "null pointer";
        case Q4_ERR_SHAPE: return "bad shape";
        case Q4_ERR_ALIGN: return "pointer not 16-byte aligned";
        case Q4_ERR_UNSUPPORTED: return "unsupported option";
        case Q4_ERR_WORKSPACE: return "workspace too small";
        case Q4_ERR_CUDA: return "CUDA error";
        case Q4_ERR_NONFINITE: return "non-finite input or scale";
        case Q4_ERR_TIMEOUT: return "bounded wait timed out";
        case Q4_ERR_BOUNDS: return "index out of bounds (debug build)";
        default: return "unknown status";
    }
}

extern "C" int q4_version(void) { return 1; }

extern "C" int q4_build_flags(void)
{
#ifdef Q4_DEBUG
    return 1;
#else
    return 0;
#endif
}

static thread_local cudaError_t q4_last_error = cudaSuccess;

void q4_record_cuda_error(cudaError_t e) { q4_last_error = e; }

extern "C" const char* q4_last_cuda_error_string(void)
{
    return q4_last_error == cudaSuccess ? "no error" : cudaGetErrorString(q4_last_error);
}

extern "C" int q4_linear_w4a16_max_gemv_m(void) { return kMaxGemvM; }

extern "C" size_t q4_linear_workspace_size(int32_t m, const q4_weight* w)
{
    if (!w || m < 1 || w->n < 1 || w->k < 1 || w->k % 128) return 0;
    return q4_gemm_workspace_bytes(m, w->n, w->k);   // (a W4A16 call the GEMV serves leaves it unused)
}

namespace {
// a caller workspace (nullable): 256-byte aligned, at least q4_linear_workspace_size bytes
int check_workspace(const void* workspace, size_t bytes, int32_t m, const q4_weight* w)
{
    if (!workspace) return Q4_OK;
    if ((uintptr_t)workspace & 255u) return Q4_ERR_ALIGN;
    return bytes < q4_linear_workspace_size(m, w) ? Q4_ERR_WORKSPACE : Q4_OK;
}
}  // namespace

extern "C" int q4_linear_w4a16(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                               int32_t* dev_status, void* stream)
{
    return q4_linear_w4a16_ws(x, m, w, y, out_dtype, nullptr, 0, dev_status, stream);
}

extern "C" int q4_linear_w4a16_ws(const uint16_t* x, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                                  void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    int rc = check_weight(w, false);
    if (rc) return rc;
    if (m < 0) return Q4_ERR_SHAPE;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    if (m == 0 || w->n == 0) return Q4_OK;   // an empty product reads and writes nothing: x, y may be NULL
    if (!x || !y) return Q4_ERR_NULL;
    if (!q4_aligned16(x) || !q4_aligned16(y)) return Q4_ERR_ALIGN;
    if ((rc = check_workspace(workspace, workspace_bytes, m, w))) return rc;
    if (m <= kMaxGemvM && w->k % 64 == 0) {
        void* ys[1] = {y};
        const int rc = q4_gemv_w4a16_launch_group(1, &x, m, w, ys, out_dtype, dev_status, (cudaStream_t)stream);
        if (rc != Q4_ERR_UNSUPPORTED) return rc;  // shapes the GEMV cannot stage go to the GEMM
    }
    if (w->k % 128) return Q4_ERR_UNSUPPORTED;
    return q4_gemm_tc_launch(x, nullptr, m, w, y, out_dtype, nullptr, false, dev_status, (cudaStream_t)stream,
                             workspace);
}

extern "C" int q4_linear_w4a16_grouped(int32_t count, const uint16_t* const* x, int32_t m, const q4_weight* w,
                                       void* const* y, int32_t out_dtype, int32_t* dev_status, void* stream)
{
    if (!x || !w || !y) return Q4_ERR_NULL;
    if (count < 1 || count > 8 || m < 1 || m > kMaxGemvM) return Q4_ERR_SHAPE;
    for (int i = 0; i < count; i++) {
        const int rc = check_weight(&w[i], false);
        if (rc) return rc;
        if (!x[i] || !y[i]) return Q4_ERR_NULL;
        if (!q4_aligned16(x[i]) || !q4_aligned16(y[i])) return Q4_ERR_ALIGN;
        if (w[i].k != w[0].k || w[i].group != w[0].group || w[i].symmetric != w[0].symmetric) return Q4_ERR_SHAPE;
    }
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    if (w[0].k % 64 || w[0].k > 16384) return Q4_ERR_UNSUPPORTED;
    return q4_gemv_w4a16_launch_group(count, x, m, w, y, out_dtype, dev_status, (cudaStream_t)stream);
}

extern "C" int q4_linear_w4a16_swiglu(const float* gate, const float* up, int32_t m, const q4_weight* w, void* y,
                                      int32_t out_dtype, int32_t* dev_status, void* stream)
{
    int rc = check_weight(w, false);
    if (rc) return rc;
    if (!gate || !up || !y) return Q4_ERR_NULL;
    if (m < 1 || m > kMaxGemvM) return Q4_ERR_SHAPE;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    if (!q4_aligned16(gate) || !q4_aligned16(up) || !q4_aligned16(y)) return Q4_ERR_ALIGN;
    if (w->k % 64 || w->k > 16384) return Q4_ERR_UNSUPPORTED;
    if (w->n == 0) return Q4_OK;
    void* ys[1] = {y};
    const float* gs[1] = {gate};
    const float* us[1] = {up};
    return q4_gemv_w4a16_launch_group(1, nullptr, m, w, ys, out_dtype, dev_status, (cudaStream_t)stream, gs, us);
}

extern "C" int q4_linear_w4a8(const int8_t* xq, const float* scale_a, int32_t m, const q4_weight* w, void* y,
                              int32_t out_dtype, int32_t* acc_dbg, int32_t* dev_status, void* stream)
{
    return q4_linear_w4a8_ws(xq, scale_a, m, w, y, out_dtype, acc_dbg, nullptr, 0, dev_status, stream);
}

extern "C" int q4_linear_w4a8_ws(const int8_t* xq, const float* scale_a, int32_t m, const q4_weight* w, void* y,
                                 int32_t out_dtype, int32_t* acc_dbg, void* workspace, size_t workspace_bytes,
                                 int32_t* dev_status, void* stream)
{
    int rc = check_weight(w, false);
    if (rc) return rc;
    if (m < 0) return Q4_ERR_SHAPE;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    if (m == 0 || w->n == 0) return Q4_OK;   // an empty product: xq, scale_a, y may be NULL
    if (!xq || !scale_a || !y) return Q4_ERR_NULL;
    if (!q4_aligned16(xq) || !q4_aligned16(y) || ((uintptr_t)scale_a & 3u) || ((uintptr_t)acc_dbg & 3u))
        return Q4_ERR_ALIGN;
    if ((rc = check_workspace(workspace, workspace_bytes, m, w))) return rc;
    if (w->k % 128) return Q4_ERR_UNSUPPORTED;
    return q4_gemm_tc_launch(xq, scale_a, m, w, y, out_dtype, acc_dbg, true, dev_status, (cudaStream_t)stream,
                             workspace);
}

int q4_gemv_w4a16_chain_launch(int n_stages, const int32_t* stage_begin, const uint16_t* const* x,
                               const float* const* g, const float* const* u, const q4_weight* w, void* const* y,
                               int32_t out_dtype, uint32_t* sync, int32_t* dev_status, cudaStream_t stream);

extern "C" size_t q4_linear_w4a16_chain_sync_bytes(int32_t n_stages)
{
    return n_stages < 1 ? 0 : (size_t)(n_stages + 1) * 128;   // one 128-byte line per counter
}

extern "C" int q4_linear_w4a16_chain(int32_t n_stages, const int32_t* stage_begin, const uint16_t* const* x,
                                     const float* const* gate, const float* const* up, const q4_weight* w,
                                     void* const* y, int32_t out_dtype, uint32_t* sync, int32_t* dev_status,
                                     void* stream)
{
    if (!stage_begin || !w || !y || !sync) return Q4_ERR_NULL;
    if (n_stages < 1 || n_stages > 128 || stage_begin[0] != 0) return Q4_ERR_SHAPE;
    for (int s = 0; s < n_stages; s++) {
        const int np = stage_begin[s + 1] - stage_begin[s];
        if (np < 1 || np > 8) return Q4_ERR_SHAPE;
    }
    const int count = stage_begin[n_stages];
    if (count > 256) return Q4_ERR_SHAPE;
    if ((uintptr_t)sync & 3u) return Q4_ERR_ALIGN;
    if (out_dtype != Q4_OUT_F32 && out_dtype != Q4_OUT_BF16) return Q4_ERR_UNSUPPORTED;
    for (int i = 0; i < count; i++) {
        const int rc = check_weight(&w[i], false);
        if (rc) return rc;
        if (w[i].group != w[0].group || w[i].symmetric != w[0].symmetric) return Q4_ERR_UNSUPPORTED;
        if (w[i].n < 1) return Q4_ERR_SHAPE;
        if (w[i].k % 64 || w[i].k > 16384) return Q4_ERR_UNSUPPORTED;
        const bool gated = gate && up && gate[i];
        if (gated) {
            if (!up[i]) return Q4_ERR_NULL;
            if (!q4_aligned16(gate[i]) || !q4_aligned16(up[i])) return Q4_ERR_ALIGN;
        } else {
            if (!x || !x[i]) return Q4_ERR_NULL;
            if (!q4_aligned16(x[i])) return Q4_ERR_ALIGN;
        }
        if (!y[i]) return Q4_ERR_NULL;
        if (!q4_aligned16(y[i])) return Q4_ERR_ALIGN;
    }
    // entries of gate/up that are NULL take x (a problem is gated only when both are given)
    const float* gs[256];
    const float* us[256];
    for (int i = 0; i < count; i++) {
        const bool gated = gate && up && gate[i];
        gs[i] = gated ? gate[i] : nullptr;
        us[i] = gated ? up[i] : nullptr;
    }
    return q4_gemv_w4a16_chain_launch(n_stages, stage_begin, x, gs, us, w, y, out_dtype, sync, dev_status,
                                      (cudaStream_t)stream);
}
