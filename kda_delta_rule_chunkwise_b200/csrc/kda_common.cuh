// Shared device helpers for the KDA kernels: element conversion, bounded
// waits and the device error word protocol.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// The device error area, one per library instance and device, is two 32-bit
// words.  err[0] holds the bits below, reported (and cleared one at a time) by
// kda_check_device_error.  err[1] holds the epoch of the latest launch in which
// a bounded wait gave up: every launch that can wait gets a fresh nonzero
// epoch from the host, and its CTAs stop waiting early only when err[1] holds
// their own epoch.  So a timeout left over from an earlier launch (or from the
// bounded-wait self test), or one in a launch running concurrently on another
// stream, never cuts short the waits of a healthy launch.
enum : uint32_t {
    ERR_WAIT_TIMEOUT = 1u,     // a bounded mbarrier/flag wait gave up
    ERR_SELFTEST = 2u,         // set by the bounded-wait self test
    ERR_BAD_INDEX = 4u,        // an index argument read on the device was out of range
    ERR_INPUT_RANGE = 8u,      // the debug input scan found a log-decay outside [-5, 0]
};

// Record a timeout of the launch with the given epoch.
__device__ __forceinline__ void record_timeout(uint32_t *err, uint32_t epoch) {
    if (!err) return;
    atomicOr(err, ERR_WAIT_TIMEOUT);
    atomicExch(err + 1, epoch);
}

// Upper bound on the wall time of one device-side wait.  Legitimate waits in
// these kernels last microseconds; anything past this bound means a missing
// arrival, and the waiting thread gives up instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s
// A wait longer than this is not a normal hand-off; only then do waiters look at
// the other CTAs' abort word in device memory.
constexpr uint64_t kSlowWaitNs = 50000ull;          // 50 us

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

// One poll of the phase with the given parity; true once that phase completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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

// Bounded wait on the phase with the given parity.  Gives up after
// `limit_ns` nanoseconds of wall time (measured with %globaltimer): it then
// sets ERR_WAIT_TIMEOUT in the error word and returns false; the caller must
// stop issuing work and leave through its normal exit path.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *err,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) break;
    }
    if (err) atomicOr(err, ERR_WAIT_TIMEOUT);
    return false;
}

// As mbar_wait, and also gives up as soon as another thread of the CTA has
// raised the shared abort flag (set here on a timeout), or another CTA of the
// same launch (same epoch) has recorded a timeout, so that one missing arrival
// ends every waiting role of every CTA of the launch within microseconds
// instead of one time limit per CTA.  Timeouts of other launches and the other
// error bits (an out-of-range index) do not stop the work.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t *bar, uint32_t parity,
                                                    uint32_t *err, uint32_t epoch,
                                                    volatile uint32_t *abort,
                                                    uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const volatile uint32_t *gepoch = err ? err + 1 : nullptr;
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        // The device-memory epoch word is read only once a wait has lasted longer
        // than any wait of a healthy launch (tens of microseconds): a global load
        // in every poll would delay noticing a completed phase by its latency.
        const uint64_t dt = globaltimer_ns() - t0;
        if (dt > kSlowWaitNs) {
            if (gepoch && *gepoch == epoch) {   // a CTA of this launch gave up: do not wait out the limit too
                *abort = 1u;
                return false;
            }
            if (dt > limit_ns) break;
        }
    }
    record_timeout(err, epoch);
    *abort = 1u;
    return false;
}

// ---------------------------------------------------------------- ready words
// A 32-bit word in device memory that one CTA sets (release) and another waits
// for (acquire), within one launch.

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// A word in shared memory handed from one thread of the CTA to another.
__device__ __forceinline__ uint32_t ld_acquire_cta_shared(const volatile uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];"
                 : "=r"(v)
                 : "r"(smem_u32(const_cast<const uint32_t *>(p)))
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta_shared(volatile uint32_t *p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(const_cast<uint32_t *>(p))),
                 "r"(v)
                 : "memory");
}

// Eight consecutive words (32-byte aligned) by one acquire load.
__device__ __forceinline__ void ld_acquire_gpu_v8(const uint32_t *p, uint32_t (&w)[8]) {
    asm volatile("ld.acquire.gpu.global.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                   "=r"(w[6]), "=r"(w[7])
                 : "l"(p)
                 : "memory");
}

// Orders this thread's generic-proxy accesses to global memory with its later
// (or, on the writing side, earlier) async-proxy accesses: bulk and TMA copies.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *word == value, with the abort rules of mbar_wait_abortable.
// Polls back off with a short sleep (the word lives in L2).
__device__ __forceinline__ bool word_wait_abortable(const uint32_t *word, uint32_t value,
                                                    uint32_t *err, uint32_t epoch,
                                                    volatile uint32_t *abort,
                                                    uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire_gpu(word) == value) return true;
    const uint64_t t0 = globaltimer_ns();
    const volatile uint32_t *gepoch = err ? err + 1 : nullptr;
    for (;;) {
        __nanosleep(64);
        if (ld_acquire_gpu(word) == value) return true;
        if (*abort) return false;
        const uint64_t dt = globaltimer_ns() - t0;
        if (dt > kSlowWaitNs) {
            if (gepoch && *gepoch == epoch) {
                *abort = 1u;
                return false;
            }
            if (dt > limit_ns) break;
        }
    }
    record_timeout(err, epoch);
    *abort = 1u;
    return false;
}

}  // namespace kda
