// Dense INT4 linear layers on the tensor cores (tcgen05): W4A16 with bf16 MMAs and W4A8 with int8 MMAs.
// The kernel itself is tcg::tc_gemm_kernel (tc_gemm.cuh) in Dense mode.
#include "tc_host.cuh"

// Split-K choice: a problem of fewer output tiles than half the SMs is split along K into at most
// sms / tiles parts of sps stages each (so splits x tiles <= sms); 1 = no split.
static int choose_splits(int32_t m, int32_t n, int32_t k, int sms, int* sps)
{
    const int tiles = ((m + tcg::BN - 1) / tcg::BN) * ((n + tcg::BM - 1) / tcg::BM);
    const int kblocks = k / tcg::KBLK;
    *sps = kblocks;
    if (tiles < 1 || 2 * tiles > sms || 2 * tiles > 128 || kblocks < 2) return 1;
    const int want = std::min(kblocks, sms / tiles);
    *sps = (kblocks + want - 1) / want;
    return (kblocks + *sps - 1) / *sps;
}

// Workspace of the split-K form: kSplitCounters int32 tile counters at offset 0 (a split shape has at
// most half as many tiles as SMs), then the fp32 partial sums [splits][m][n].  The counters sit at the
// same place for every shape, so a workspace reused across shapes keeps them zero: they must be zero
// before the first call and every completed call leaves them zero.  0 when the shape is not split.
constexpr int kSplitCounters = 128;
constexpr size_t kCounterBytes = kSplitCounters * 4;

size_t q4_gemm_workspace_bytes(int32_t m, int32_t n, int32_t k)
{
    int sps;
    const int splits = choose_splits(m, n, k, q4_num_sms(), &sps);
    if (splits < 2) return 0;
    return kCounterBytes + (((size_t)splits * m * n * 4 + 255) & ~(size_t)255);
}

// m >= 1, k % 128 == 0, group in {64, 128}.  With a workspace, a problem of fewer output tiles than half
// the SMs is split along K so that every SM gets work (the splits meet in the workspace).
int q4_gemm_tc_launch(const void* x, const float* scale_a, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                      int32_t* acc_dbg, bool int8_path, int32_t* dev_status, cudaStream_t stream,
                      void* workspace)
{
    using namespace tcg;
    if (w->k % KBLK) return Q4_ERR_UNSUPPORTED;
    CUtensorMap mx, mw;
    if (!make_act_map(&mx, x, (uint64_t)w->k, (uint64_t)m, int8_path ? 1 : 2, false) ||
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
    const int sms = q4_num_sms();
    p.splits = 1;
    p.sps = w->k / KBLK;
    if (workspace) {
        p.splits = choose_splits(m, w->n, w->k, sms, &p.sps);
        p.tile_ctr = reinterpret_cast<int32_t*>(workspace);
        p.ws = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + kCounterBytes);
    }
    const int grid = std::min(tiles * p.splits, sms);
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
