// The MoE layer's grouped expert GEMMs with INT8 activations (W4A8): tcg::tc_gemm_kernel in GateUp and
// Down modes with int8 MMAs.  Source: "MoE推理优化实战：4bit存储+INT8计算的W4A8路线解析" §2.3 (INT4
// widened to INT8, INT8 x INT8 into INT32, rescale by scale_w * scale_a), §3.1 (per-token activation
// codes), §5.1 (the projections of an FFN may take different precisions).  Kept in a translation unit of
// its own so that these eight kernel instances compile in parallel with the 16-bit ones.
#include "tc_host.cuh"

namespace {

template <int G, bool SYM>
int gateup(const int8_t* xq, const float* sa, const q4_weight* gate, const q4_weight* up, int P, int H, int I, int E,
           const int32_t* offsets, const int32_t* tiles, __nv_bfloat16* h, bool h_f16, int32_t* status, cudaStream_t s)
{
    using namespace tcg;
    CUtensorMap mx, mg, mu;
    if (!make_act_map(&mx, xq, H, P, 1) || !make_packed_map(&mg, gate->packed, H, (uint64_t)E * I, 64) ||
        !make_packed_map(&mu, up->packed, H, (uint64_t)E * I, 64))
        return Q4_ERR_CUDA;
    Args a = {};
    a.M = P;
    a.N = I;
    a.K = H;
    a.scales_a = reinterpret_cast<const __half*>(gate->scales);
    a.zeros_a = reinterpret_cast<const __half*>(gate->zeros);
    a.scales_b = reinterpret_cast<const __half*>(up->scales);
    a.zeros_b = reinterpret_cast<const __half*>(up->zeros);
    a.scale_a = sa;
    a.status = status;
    a.expert_tiles = tiles;
    a.offsets = offsets;
    a.h = h;
    a.h_f16 = h_f16;
    a.E = E;
    return launch<true, G, SYM, Mode::GateUp>(mx, mg, mu, a, q4_num_sms(), s);
}

template <int G, bool SYM>
int down(const int8_t* hq, const float* sh, const q4_weight* dn, int P, int H, int I, int E, const int32_t* offsets,
         const int32_t* tiles, const int32_t* row_tok, const float* row_w, float* y32, int T, int32_t* status,
         cudaStream_t s)
{
    using namespace tcg;
    CUtensorMap mh, md;
    if (!make_act_map(&mh, hq, I, P, 1) || !make_packed_map(&md, dn->packed, I, (uint64_t)E * H, BM))
        return Q4_ERR_CUDA;
    Args d = {};
    d.M = P;
    d.N = H;
    d.K = I;
    d.scales_a = reinterpret_cast<const __half*>(dn->scales);
    d.zeros_a = reinterpret_cast<const __half*>(dn->zeros);
    d.scale_a = sh;
    d.y = y32;
    d.status = status;
    d.expert_tiles = tiles;
    d.offsets = offsets;
    d.row_tok = row_tok;
    d.row_w = row_w;
    d.E = E;
    d.T = T;
    return launch<true, G, SYM, Mode::Down>(mh, md, md, d, q4_num_sms(), s);
}

}  // namespace

int q4_moe_gateup_a8(const int8_t* xq, const float* sa, const q4_weight* gate, const q4_weight* up, int P, int H,
                     int I, int E, const int32_t* offsets, const int32_t* tiles, __nv_bfloat16* h, bool h_f16,
                     int32_t* status, cudaStream_t s)
{
    if (gate->group == 128)
        return gate->symmetric ? gateup<128, true>(xq, sa, gate, up, P, H, I, E, offsets, tiles, h, h_f16, status, s)
                               : gateup<128, false>(xq, sa, gate, up, P, H, I, E, offsets, tiles, h, h_f16, status, s);
    return gate->symmetric ? gateup<64, true>(xq, sa, gate, up, P, H, I, E, offsets, tiles, h, h_f16, status, s)
                           : gateup<64, false>(xq, sa, gate, up, P, H, I, E, offsets, tiles, h, h_f16, status, s);
}

int q4_moe_down_a8(const int8_t* hq, const float* sh, const q4_weight* dn, int P, int H, int I, int E,
                   const int32_t* offsets, const int32_t* tiles, const int32_t* row_tok, const float* row_w,
                   float* y32, int T, int32_t* status, cudaStream_t s)
{
    if (dn->group == 128)
        return dn->symmetric ? down<128, true>(hq, sh, dn, P, H, I, E, offsets, tiles, row_tok, row_w, y32, T, status, s)
                             : down<128, false>(hq, sh, dn, P, H, I, E, offsets, tiles, row_tok, row_w, y32, T, status, s);
    return dn->symmetric ? down<64, true>(hq, sh, dn, P, H, I, E, offsets, tiles, row_tok, row_w, y32, T, status, s)
                         : down<64, false>(hq, sh, dn, P, H, I, E, offsets, tiles, row_tok, row_w, y32, T, status, s);
}
