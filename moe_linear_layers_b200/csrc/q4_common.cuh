// Shared device/host helpers of the CUDA library (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/q4.h"

#define Q4_SM_COUNT_HINT 148

// Record the first device-side error in the caller's status word (nullable).
__device__ __forceinline__ void q4_set_status(int32_t* status, int32_t code)
{
    if (status) atomicCAS(status, 0, code);
}

// Debug build (Q4_DEBUG): a global-memory index a kernel computes is checked against its buffer's extent
// before the access; a failed check records Q4_ERR_BOUNDS and the access is skipped.  In the release build
// the check is the constant true and costs nothing.
__device__ __forceinline__ bool q4_in_bounds(int64_t i, int64_t n, int32_t* status)
{
#ifdef Q4_DEBUG
    if (i >= 0 && i < n) return true;
    q4_set_status(status, Q4_ERR_BOUNDS);
    return false;
#else
    (void)i;
    (void)n;
    (void)status;
    return true;
#endif
}

// (a & b) ^ c in one LOP3.
__device__ __forceinline__ uint32_t lop3_and_xor(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Host side: error mapping for launches.  The last CUDA error is kept per host thread for
// q4_last_cuda_error_string().
void q4_record_cuda_error(cudaError_t e);

static inline int q4_cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return Q4_OK;
    q4_record_cuda_error(e);
    return Q4_ERR_CUDA;
}

static inline int q4_launch_status() { return q4_cuda_status(cudaGetLastError()); }

static inline bool q4_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-token INT8 quantization of bf16 (f16 = false) or fp16 rows, the kernel behind act_quant_per_token
// and act_quant_per_token_f16 (act_quant.cu); same arguments and return codes.
int q4_act_quant_rows(const uint16_t* x, bool f16, int32_t m, int32_t k, int8_t* xq, float* scale_a,
                      int32_t* dev_status, cudaStream_t s);

// The MoE layer's grouped expert GEMMs on int8 activation codes (moe_a8.cu): gate/up with the SwiGLU
// epilogue into h (bf16 hi/lo pairs, or fp16 when h_f16: the activation an INT8 down projection
// quantizes), and down with the weighted reduction into y32.  P permuted rows;
// offsets and tiles as the 16-bit grouped GEMMs take them; sa / sh the per-permuted-row activation scales.
int q4_moe_gateup_a8(const int8_t* xq, const float* sa, const q4_weight* gate, const q4_weight* up, int P, int H,
                     int I, int E, const int32_t* offsets, const int32_t* tiles, __nv_bfloat16* h, bool h_f16,
                     int32_t* status, cudaStream_t s);
int q4_moe_down_a8(const int8_t* hq, const float* sh, const q4_weight* dn, int P, int H, int I, int E,
                   const int32_t* offsets, const int32_t* tiles, const int32_t* row_tok, const float* row_w,
                   float* y32, int T, int32_t* status, cudaStream_t s);

// Number of SMs of the current device (cached per device).
static inline int q4_num_sms()
{
    static int cache[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return Q4_SM_COUNT_HINT;
    if (!cache[dev]) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = Q4_SM_COUNT_HINT;
        cache[dev] = sms;
    }
    return cache[dev];
}
