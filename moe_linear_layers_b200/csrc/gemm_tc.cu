// Dense INT4 linear layers on the tensor cores (tcgen05): W4A16 with bf16 MMAs and W4A8 with int8 MMAs.
// The kernel itself is tcg::tc_gemm_kernel (tc_gemm.cuh) in Dense mode.
#include "tc_host.cuh"

// Split-K: a problem whose output tiles fill fewer than half the SMs is cut along K into splits of sps
// 128-K blocks each (at least two), so that splits x tiles approaches the SM count; 1 = no split.
static int choose_splits(int32_t m, int32_t n, int32_t k, int sms, int* sps)
{
    const int tiles = ((m + tcg::BN - 1) / tcg::BN) * ((n + tcg::BM - 1) / tcg::BM);
    const int kblocks = k / tcg::KBLK;
    *sps = kblocks;
    if (tiles < 1 || 2 * tiles > sms || kblocks < 4) return 1;
    const int want = std::min(std::min(kblocks / 2, sms / tiles), 16);   // (the reduction takes at most 16)
    if (want < 2) return 1;
    *sps = (kblocks + want - 1) / want;
    return (kblocks + *sps - 1) / *sps;
}

size_t q4_gemm_workspace_bytes(int32_t m, int32_t n, int32_t k)
{
    int sps;
    const int splits = choose_splits(m, n, k, q4_num_sms(), &sps);
    return splits < 2 ? 0 : (((size_t)splits * m * n * 4 + 255) & ~(size_t)255);
}

// y = the sum of the splits' partial sums, in split order (the same bits on every run).  Four values a
// thread when m * n % 4 == 0 (16-byte loads; every split's load goes out before the sum), else one.
constexpr int kMaxSplits = 16;

__global__ void split_reduce_kernel(const float* __restrict__ part, int splits, int64_t mn, void* y, int out_bf16)
{
    // launched as a programmatic dependent of the GEMM: the partials are read after its completion
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    if (mn % 4 == 0) {
        const int64_t n4 = mn / 4;
        const float4* p4 = reinterpret_cast<const float4*>(part);
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
            float4 v[kMaxSplits];
#pragma unroll
            for (int sp = 0; sp < kMaxSplits; sp++)
                if (sp < splits) v[sp] = __ldg(p4 + (int64_t)sp * n4 + i);
            float4 a = v[0];
#pragma unroll
            for (int sp = 1; sp < kMaxSplits; sp++)
                if (sp < splits) {
                    a.x += v[sp].x;
                    a.y += v[sp].y;
                    a.z += v[sp].z;
                    a.w += v[sp].w;
                }
            if (out_bf16) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
                reinterpret_cast<uint2*>(y)[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                                            *reinterpret_cast<const uint32_t*>(&hi));
            } else {
                reinterpret_cast<float4*>(y)[i] = a;
            }
        }
        return;
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < mn; i += stride) {
        float v = part[i];
        for (int sp = 1; sp < splits; sp++) v += part[(int64_t)sp * mn + i];
        if (out_bf16) reinterpret_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
        else reinterpret_cast<float*>(y)[i] = v;
    }
}

// m >= 1, k % 128 == 0, group in {64, 128}.  With a workspace of q4_gemm_workspace_bytes, a problem of few
// output tiles is split along K (the splits' partial sums meet in the workspace and a second kernel adds
// them up); without one, or when the shape is not split, one kernel writes y.
int q4_gemm_tc_launch(const void* x, const float* scale_a, int32_t m, const q4_weight* w, void* y, int32_t out_dtype,
                      int32_t* acc_dbg, bool int8_path, int32_t* dev_status, cudaStream_t stream, void* workspace)
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
    const int sms = q4_num_sms();
    p.splits = 1;
    p.sps = w->k / KBLK;
    if (workspace) {
        p.splits = choose_splits(m, w->n, w->k, sms, &p.sps);
        p.part = reinterpret_cast<float*>(workspace);
    }
    if (p.splits < 2) p.splits = 1;
    const int grid = std::min(tiles * p.splits, sms);
    int rc;
    if (int8_path) {
        if (w->group == 128)
            rc = w->symmetric ? launch<true, 128, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                              : launch<true, 128, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
        else
            rc = w->symmetric ? launch<true, 64, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                              : launch<true, 64, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
    } else {
        if (w->group == 128)
            rc = w->symmetric ? launch<false, 128, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                              : launch<false, 128, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
        else
            rc = w->symmetric ? launch<false, 64, true, Mode::Dense>(mx, mw, mw, p, grid, stream)
                              : launch<false, 64, false, Mode::Dense>(mx, mw, mw, p, grid, stream);
    }
    if (rc || p.splits == 1) return rc;
    const int64_t mn = (int64_t)m * w->n;
    cudaLaunchConfig_t cfg = {};
    const int64_t units = mn % 4 == 0 ? mn / 4 : mn;
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, std::min<int64_t>((units + 255) / 256, 4 * sms)));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return q4_cuda_status(cudaLaunchKernelEx(&cfg, split_reduce_kernel, (const float*)p.part, p.splits, mn, y,
                                             (int)(out_dtype == Q4_OUT_BF16)));
}
