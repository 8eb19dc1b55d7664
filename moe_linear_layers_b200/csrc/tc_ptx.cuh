// Blackwell (sm_100a) primitives written as inline PTX: mbarriers with bounded waits, TMA tile loads
// (no multicast), tcgen05 TMEM allocation, MMA with the A operand in TMEM, commit, and TMEM
// loads/stores.  Used by the tensor-core GEMM and the MoE expert GEMMs.
#pragma once

#include <cuda.h>

#include "q4_common.cuh"

namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_one_lane() { return (threadIdx.x & 31) == 0; }

// ---------------------------------------------------------------------------------------------- //
// mbarrier
// ---------------------------------------------------------------------------------------------- //

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive without release semantics: the arrival does not wait for this thread's outstanding global
// loads.  For a consumer that read its operands from shared memory (ld.shared has completed once the
// values are in registers) and releases the buffer.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wall-time limit of the kernels' waits.  Long enough that a context time-sliced with other work on a
// shared GPU does not read as stuck, short enough that a wait nothing will satisfy ends the kernel
// with Q4_ERR_TIMEOUT instead of hanging it.
constexpr uint64_t kWaitLimitNs = 10000000000ull;

// True once more than limit_ns of wall time separates now from t0 AND at least min_rounds polls were
// made.  The difference is taken signed, so a global timer stepped back while a wait runs (the timer is
// kept in step with the host clock) cannot make a fresh wait look expired through unsigned wrap-around,
// and the poll count keeps a forward step from ending a wait that has barely started.
__device__ __forceinline__ bool wait_expired(uint64_t t0, uint64_t limit_ns, uint32_t rounds, uint32_t min_rounds)
{
    return rounds >= min_rounds && (int64_t)(globaltimer_ns() - t0) > (int64_t)limit_ns;
}

// Wait for the phase with the given parity to complete.  Gives up after `limit_ns` of wall time:
// records Q4_ERR_TIMEOUT in the status word, raises the CTA's abort flag (nullable) and returns false.
__device__ __forceinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, int32_t* status,
                                               volatile int* abort_flag, uint64_t limit_ns)
{
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; i++) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u) {
            if (abort_flag && *abort_flag) return false;
            if (wait_expired(t0, limit_ns, i >> 8, 64)) {
                q4_set_status(status, Q4_ERR_TIMEOUT);
                if (abort_flag) *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs)
{
#pragma unroll 1
    for (int i = 0; i < 64; i++)
        if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, status, abort_flag, limit_ns);
}

// Wait for three phases at once.  The three tests go out back to back, so a consumer that usually
// finds every phase complete pays one shared-memory round trip instead of three; an incomplete phase
// falls back to mbar_wait.
__device__ __forceinline__ bool mbar_wait3(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                           uint32_t p2, int32_t* status, volatile int* abort_flag)
{
    uint32_t ok0, ok1, ok2;
    asm volatile(
        "{\n\t.reg .pred q0, q1, q2;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 q0, [%3], %4;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 q1, [%5], %6;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 q2, [%7], %8;\n\t"
        "selp.u32 %0, 1, 0, q0;\n\t"
        "selp.u32 %1, 1, 0, q1;\n\t"
        "selp.u32 %2, 1, 0, q2;\n\t}"
        : "=r"(ok0), "=r"(ok1), "=r"(ok2)
        : "r"(smem_u32(b0)), "r"(p0), "r"(smem_u32(b1)), "r"(p1), "r"(smem_u32(b2)), "r"(p2)
        : "memory");
    if (ok0 & ok1 & ok2) return true;
    return (ok0 || mbar_wait(b0, p0, status, abort_flag)) && (ok1 || mbar_wait(b1, p1, status, abort_flag)) &&
           (ok2 || mbar_wait(b2, p2, status, abort_flag));
}

// ---------------------------------------------------------------------------------------------- //
// TMA (tiled, no multicast)
// ---------------------------------------------------------------------------------------------- //

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0, int32_t c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tile load (coordinates innermost first).  No multicast.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t c0, int32_t c1,
                                            int32_t c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------------------------------------- //
// tcgen05: TMEM allocation, MMA, commit, fences, loads and stores
// ---------------------------------------------------------------------------------------------- //

// Whole warp: allocate `ncols` TMEM columns; the base address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T, 16-bit inputs (bf16 or fp16 per the instruction descriptor),
// fp32 accumulate (cta_group::1).
__device__ __forceinline__ void mma_16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, int8 inputs, int32 accumulate (cta_group::1).
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Warp-wide: thread t reads TMEM lane (lane field of taddr) + t, 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Warp-wide: thread t writes TMEM lane (lane field of taddr) + t, 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// ---------------------------------------------------------------------------------------------- //
// progress counters for a thread that issues tcgen05.mma
//
// Any strong memory operation in an MMA-issuing thread -- an mbarrier wait, even on a completed phase,
// or a relaxed / acquire / volatile load -- stalls that thread until the MMAs it issued have retired,
// which leaves the tensor pipe idle (measured: 64 cycles per M128 N128 K16 MMA without, ~155 with one
// such wait per 8 MMAs).  Weak loads do not.  So the issuer polls monotonic counters with weak loads;
// the threads that publish them (converters, epilogue) first complete what the counter announces --
// tcgen05.wait::st / wait::ld, so the TMEM accesses are done, and the mbarrier waits for the data the
// MMA will read -- and then store the counter with a plain shared-memory store: a release (or even a
// relaxed) store would also wait for the publisher's unrelated global loads in flight (the scale
// read-ahead).
// ---------------------------------------------------------------------------------------------- //

// Register re-partition between warpgroups (every warp of a warpgroup executes the same one).  An
// increase waits until other warpgroups have released enough registers of the CTA's launch allocation.
template <uint32_t N> __device__ __forceinline__ void setmaxnreg_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N> __device__ __forceinline__ void setmaxnreg_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

#ifndef Q4_POLL_SLEEP_NS
#define Q4_POLL_SLEEP_NS 0
#endif

__device__ __forceinline__ uint32_t lds_weak(const void* p)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

__device__ __forceinline__ void sts_publish(void* p, uint32_t v)
{
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Spin until each of the n counters at c is >= target.  The fast path makes weak loads only; after a
// few thousand unsuccessful rounds it also watches the wall clock (kWaitLimitNs: Q4_ERR_TIMEOUT, raise
// the abort flag, return false) and the abort flag.
__device__ __forceinline__ bool poll_counters_slow(const uint32_t* c, int n, uint32_t target, int32_t* status,
                                                   volatile int* abort_flag, uint64_t limit_ns = kWaitLimitNs)
{
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t round = 0;; round++) {
        bool ok = true;
        for (int i = 0; i < n; i++) ok &= lds_weak(c + i) >= target;
        if (ok) return true;
        if (abort_flag && *abort_flag) return false;
        if (wait_expired(t0, limit_ns, round, 1u << 16)) {
            q4_set_status(status, Q4_ERR_TIMEOUT);
            if (abort_flag) *abort_flag = 1;
            return false;
        }
    }
}

template <int N>
__device__ __forceinline__ bool poll_counters(const uint32_t* c, uint32_t target, int32_t* status,
                                              volatile int* abort_flag)
{
    for (int round = 0; round < 4096; round++) {
        bool ok = true;
#pragma unroll
        for (int i = 0; i < N; i++) ok &= lds_weak(c + i) >= target;
        if (ok) return true;
#if Q4_POLL_SLEEP_NS > 0
        __nanosleep(Q4_POLL_SLEEP_NS);
#endif
    }
    return poll_counters_slow(c, N, target, status, abort_flag);
}

// ---------------------------------------------------------------------------------------------- //
// packed fp32 pairs (sm_100 f32x2 arithmetic; each half rounds exactly like the scalar instruction)
// ---------------------------------------------------------------------------------------------- //

__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi)
{
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}

__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Warp-wide: thread t fills TMEM lane (lane field of taddr) + t, 32 consecutive columns, with one value.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
        "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};"
        ::"r"(taddr), "r"(v)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with 128-byte swizzle:
// rows of 128 bytes, 8-row atoms 1024 bytes apart (stride byte offset), base 1024-byte aligned.
// Advancing along K inside the 128-byte row adds (bytes >> 4) to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);       // start address, bits [0,14)
    d |= (uint64_t)1u << 16;                        // leading byte offset (unused with swizzle), bits [16,30)
    d |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset, bits [32,46)
    d |= (uint64_t)1u << 46;                        // descriptor version for sm_100, bits [46,48)
    d |= (uint64_t)2u << 61;                        // layout: 128-byte swizzle, bits [61,64)
    return d;
}

// Instruction descriptor: dense, K-major A and B, M = 128, N = n.
//   c_format bits [4,6): 1 = f32, 2 = s32;  a/b_format bits [7,10)/[10,13): f16 = 0, bf16 = 1, s8 = 1 (signed);
//   N >> 3 in bits [17,23);  M >> 4 in bits [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_f16_f32(uint32_t n)
{
    return (1u << 4) | (0u << 7) | (0u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_s8_s32(uint32_t n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

}  // namespace tc
