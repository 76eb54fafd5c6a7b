// Device-side building blocks for sm_100a: shared-memory barriers with bounded
// waits, asynchronous copies and L2 prefetches, programmatic dependent launch,
// element types.
#ifndef PKV_DEVICE_CUH_
#define PKV_DEVICE_CUH_

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pagedkv.h"

namespace pkv {

// One device error word per device (PKV_DEVERR_* bits), read by kv_get_device_error().
// The library's device code is a single translation unit (pagedkv.cu), which defines it.
__device__ unsigned int g_error_word = 0;

// A bounded wait gives up after this many SM clock cycles (about one second at the
// B200's clocks); a healthy wait ends within microseconds.
constexpr long long kWaitLimitCycles = 2000000000LL;

// The limit of the waits through which a warp consumes another's work (mbar_wait_bounded).
// A test build may shorten it (-DPKV_CONSUMER_WAIT_LIMIT_CYCLES=...) to drive the abort
// path, and poll the barrier with the non-blocking test_wait, checking the limit at every
// probe (-DPKV_CONSUMER_WAIT_POLL=1): try_wait may suspend the thread until the phase
// completes, so a healthy wait would never see a short limit run out.  The drain waits for
// copies and MMAs already in flight keep try_wait and kWaitLimitCycles, so no CTA exits, or
// frees tensor memory, with asynchronous writes outstanding.
#ifndef PKV_CONSUMER_WAIT_LIMIT_CYCLES
#define PKV_CONSUMER_WAIT_LIMIT_CYCLES 2000000000LL
#endif
#ifndef PKV_CONSUMER_WAIT_POLL
#define PKV_CONSUMER_WAIT_POLL 0
#endif
constexpr long long kConsumerWaitLimitCycles = PKV_CONSUMER_WAIT_LIMIT_CYCLES;

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait until the phase with the given parity has completed.  Gives up (returns
// false) when *abort is set by another warp, or after kConsumerWaitLimitCycles, in
// which case it sets *abort and PKV_DEVERR_TIMEOUT.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort)
{
#if PKV_CONSUMER_WAIT_POLL
    const long long t_poll = clock64();
    for (;;) {
        if (mbar_test_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t_poll > kConsumerWaitLimitCycles) {
            *abort = 1;
            atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
            return false;
        }
    }
#endif
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 31u) == 0) {
            if (*abort) return false;
            if (clock64() - t0 > kConsumerWaitLimitCycles) {
                *abort = 1;
                atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
                return false;
            }
        }
    }
}

// 16-byte asynchronous global -> shared copy (cp.async, cached in L2 only).
__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// Pull the 128-byte line holding `p` into L2 (no register result, no L1 fill).
__device__ __forceinline__ void prefetch_l2(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Pull the line holding `p` into L2 with the evict-last priority, so that a stream of
// normal-priority lines passing through L2 does not push it out before it is used.
__device__ __forceinline__ void prefetch_l2_evict_last(const void* p)
{
    asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's committed cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// cp_async_wait<n> for a run-time n in 0..8 (n above 8 waits as for 8).
__device__ __forceinline__ void cp_async_wait_upto(int n)
{
    switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    case 7: cp_async_wait<7>(); break;
    default: cp_async_wait<8>(); break;
    }
}

// Programmatic dependent launch: wait for the preceding kernel of the stream to
// finish (and its writes to be visible); allow the next kernel to start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Named barrier for a subset of warps (id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- element types -------------------------------------------------------
template <typename T> struct Elt;

template <> struct Elt<__half> {
    static __device__ __forceinline__ float2 to_float2(uint32_t w)
    {
        __half2 h = *reinterpret_cast<const __half2*>(&w);
        return __half22float2(h);
    }
    static __device__ __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
    static __device__ __forceinline__ __half from_double(double x) { return __double2half(x); }
    static __device__ __forceinline__ double to_double(__half x) { return (double)__half2float(x); }
};

template <> struct Elt<__nv_bfloat16> {
    static __device__ __forceinline__ float2 to_float2(uint32_t w)
    {
        // bfloat16 is the high half of an fp32: widening is a shift / mask.
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_double(double x) { return __double2bfloat16(x); }
    static __device__ __forceinline__ double to_double(__nv_bfloat16 x) { return (double)__bfloat162float(x); }
};

// Dot product of 8 storage elements with fp32 accumulation.  sm_100's mixed-precision
// fma (16-bit multiplicands, fp32 addend and result) rounds exactly like widening both
// operands to fp32 and calling fmaf, since the 16-bit product is exact in fp32.
template <typename T> __device__ __forceinline__ float dot8(const uint4& q, const uint4& k);

#define PKV_DOT8_ASM(TYPE)                                                                                     \
    float a = 0.f, b = 0.f;                                                                                    \
    asm("{ .reg .b16 q0,q1,q2,q3,q4,q5,q6,q7,k0,k1,k2,k3,k4,k5,k6,k7;\n\t"                                      \
        "mov.b32 {q0,q1}, %2; mov.b32 {q2,q3}, %3; mov.b32 {q4,q5}, %4; mov.b32 {q6,q7}, %5;\n\t"                 \
        "mov.b32 {k0,k1}, %6; mov.b32 {k2,k3}, %7; mov.b32 {k4,k5}, %8; mov.b32 {k6,k7}, %9;\n\t"                 \
        "fma.rn.f32." TYPE " %0, q0, k0, %0; fma.rn.f32." TYPE " %1, q1, k1, %1;\n\t"                            \
        "fma.rn.f32." TYPE " %0, q2, k2, %0; fma.rn.f32." TYPE " %1, q3, k3, %1;\n\t"                            \
        "fma.rn.f32." TYPE " %0, q4, k4, %0; fma.rn.f32." TYPE " %1, q5, k5, %1;\n\t"                            \
        "fma.rn.f32." TYPE " %0, q6, k6, %0; fma.rn.f32." TYPE " %1, q7, k7, %1; }"                                \
        : "+f"(a), "+f"(b)                                                                                     \
        : "r"(q.x), "r"(q.y), "r"(q.z), "r"(q.w), "r"(k.x), "r"(k.y), "r"(k.z), "r"(k.w));                    \
    return a + b;

template <> __device__ __forceinline__ float dot8<__half>(const uint4& q, const uint4& k) { PKV_DOT8_ASM("f16") }
template <> __device__ __forceinline__ float dot8<__nv_bfloat16>(const uint4& q, const uint4& k) { PKV_DOT8_ASM("bf16") }
#undef PKV_DOT8_ASM

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8])
{
    float2 a = Elt<T>::to_float2(u.x), b = Elt<T>::to_float2(u.y);
    float2 c = Elt<T>::to_float2(u.z), d = Elt<T>::to_float2(u.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}



}  // namespace pkv

#endif  // PKV_DEVICE_CUH_
