// Host helpers of the tensor-core kernels: TMA tensor-map encoding (driver entry point fetched
// through the runtime, so the library does not link libcuda) and kernel launch with the opt-in
// shared-memory size.
#pragma once

#include <cudaTypedefs.h>

#include "tc_gemm.cuh"

namespace tcg {

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode()
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

// 2-D tensor map: `inner` contiguous elements per row, `outer` rows, row pitch in bytes.
inline bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
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

// Activation tile map.  int8 [rows][k]: one 128 x 128 box per stage.  bf16 [rows][k]: viewed as 3-D
// (64 columns, rows, k / 64 column blocks; the last stride is 128 bytes) so that the tile of a stage --
// `blocks` 64-column blocks of 128 rows, each 128-byte swizzled -- is ONE copy (a thread's bulk copies
// are throughput-limited per instruction, not per byte).  blocks = 2: a 128-column stage; blocks = 4:
// the MoE intermediate h, whose rows interleave 64-column blocks of hi and lo values (k = 2 I).
inline bool make_act_map(CUtensorMap* map, const void* base, uint64_t k, uint64_t rows, int elem_bytes, int blocks = 2)
{
    if (elem_bytes == 1)
        return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, k, rows, k, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    auto enc = get_encode();
    if (!enc || k % 64) return false;
    cuuint64_t dims[3] = {64, rows, k / 64};
    cuuint64_t strides[2] = {2 * k, 128};
    cuuint32_t box[3] = {64, BN, (cuuint32_t)blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed weight map: [rows][k/2] bytes, boxes of 64 bytes (one K stage) x box_rows rows, 64-byte swizzle.
inline bool make_packed_map(CUtensorMap* map, const void* base, uint64_t k, uint64_t rows, uint32_t box_rows)
{
    return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, k / 2, rows, k / 2, KBLK / 2, box_rows,
                    CU_TENSOR_MAP_SWIZZLE_64B);
}

template <bool INT8, int G, bool SYM, Mode MODE>
int launch(const CUtensorMap& mx, const CUtensorMap& ma, const CUtensorMap& mb, const Args& p, int grid,
           cudaStream_t s)
{
    auto kern = tc_gemm_kernel<INT8, G, SYM, MODE>;
    constexpr int smem = Cfg<INT8, MODE, !INT8 || !SYM>::SMEM;
    if (const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) return q4_cuda_status(e);
    // The kernel re-partitions its registers between warpgroups (setmaxnreg) assuming a launch
    // allocation of kLaunchRegs per thread; a build that allocated fewer would make the increase wait
    // forever, so it is refused.
    static const int nregs = [&] {
        cudaFuncAttributes fa{};
        return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (nregs != kLaunchRegs) return Q4_ERR_UNSUPPORTED;
    if constexpr (MODE == Mode::Dense) {
        // programmatic dependent launch (see the kernel: only the activation copies wait)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return q4_cuda_status(cudaLaunchKernelEx(&cfg, kern, mx, ma, mb, p));
    } else {
        kern<<<grid, kThreads, smem, s>>>(mx, ma, mb, p);
        return q4_launch_status();
    }
}

}  // namespace tcg
