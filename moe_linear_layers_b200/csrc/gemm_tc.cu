// Dense INT4 linear layers on the tensor cores (tcgen05): W4A16 with bf16 MMAs and W4A8 with int8 MMAs.
// The kernel itself is tcg::tc_gemm_kernel (tc_gemm.cuh) in Dense mode.
#include "tc_host.cuh"

// m >= 1, k % 128 == 0, group in {64, 128}.
int q4_gemm_tc_launch(const void* x, const float* scale_a, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                      int32_t* acc_dbg, bool int8_path, int32_t* dev_status, cudaStream_t stream)
{
    using namespace tcg;
    if (w->k % KBLK) return Q4_ERR_UNSUPPORTED;
    CUtensorMap mx, mw;
    if (!make_act_map(&mx, x, (uint64_t)w->k, (uint64_t)m, int8_path ? 1 : 2) ||
        !make_packed_map(&mw, w->packed, (uint64_t)w->k, (uint64_t)w->n, BM))
        return Q4_ERR_CUDA;
    Args p = {};
    p.M = m;
    p.N = w->n;
    p.K = w->k;
    p.out_bf16 = out_dtype == Q4_OUT_BF16;
    p.scales_a = reinterpret_cast<const __half*>(w->scales);
    p.zeros_a = reinterpret_cast<const __half*>(w->zeros);
    p.scale_a = scale_a;
    p.y = y;
    p.acc_dbg = acc_dbg;
    p.status = dev_status;
    const int tiles = ((m + BN - 1) / BN) * ((w->n + BM - 1) / BM);
    const int grid = std::min(tiles, q4_num_sms());
    if (int8_path) {
        if (w->group == 128)
            return w->symmetric ? launch<true, 128, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                                : launch<true, 128, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
        return w->symmetric ? launch<true, 64, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                            : launch<true, 64, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
    }
    if (w->group == 128)
        return w->symmetric ? launch<false, 128, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                            : launch<false, 128, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
    return w->symmetric ? launch<false, 64, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                        : launch<false, 64, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
}
