// sync.cuh — mbarrier, bulk-copy (TMA) and programmatic-dependent-launch helpers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#define MOE_DEVINL __device__ __forceinline__

namespace moe {

// Device error word bits (word 1 of a workspace; 0 = ok).
//   kErrTimeout: a bounded wait gave up; the call's outputs are not valid, and
//                every later call on the same workspace gives up at its first
//                wait until the word is cleared.
//   kErrRange  : a prefill activation (x or h) outside the fp16 range; the rows
//                of those tokens are not valid, the others are.
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrRange = 2u;
// Bounded waits give up after this long (far above any legitimate wait).
constexpr uint64_t kWaitLimitNs = 500ull * 1000 * 1000;
constexpr uint32_t kMaxPolls = 1u << 24;

MOE_DEVINL uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
MOE_DEVINL uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

MOE_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
MOE_DEVINL void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
MOE_DEVINL void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

MOE_DEVINL void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
// Arrive once `dep` is known: a value computed from everything this warp read
// out of the buffer the arrive releases, so that no read of it is still in
// flight when its producer may overwrite it.
MOE_DEVINL void mbar_arrive_dep(uint64_t* bar, uint32_t dep) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)), "r"(dep)
                 : "memory");
}
MOE_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
MOE_DEVINL bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
MOE_DEVINL bool timed_out(const uint32_t* err) {
    return err && (*reinterpret_cast<const volatile uint32_t*>(err) & kErrTimeout);
}
// Bounded wait: returns false, and sets the timeout bit of *err, if the phase
// does not complete within kWaitLimitNs; returns false as soon as it finds the
// timeout bit already set (another CTA or an earlier kernel gave up).
MOE_DEVINL bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (timed_out(err)) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            if (err) atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

// Bounded wait as mbar_wait, but each poll suspends the thread in hardware
// (up to 20 us) until the phase completes: a waiting warp takes no issue
// slots from the warps that do the work.
MOE_DEVINL bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
// The error word is a global load: it is read every 20 us of waiting, not at
// every poll, so that its latency does not delay the wake-up.
MOE_DEVINL bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t* err) {
    if (mbar_try_wait_suspend(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint64_t check = t0 + 20000;
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity)) return true;
        const uint64_t t = globaltimer_ns();
        if (t >= check) {
            if (timed_out(err)) return false;
            if (t - t0 > kWaitLimitNs) {
                if (err) atomicOr(err, kErrTimeout);
                return false;
            }
            check = t + 20000;
        }
    }
}

// Bounded wait that does not give up early on the error word: used to let
// copies and MMAs still in flight land before the CTA exits.
MOE_DEVINL void mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// Bulk copy global -> shared, completing `bytes` of transaction on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
MOE_DEVINL void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
MOE_DEVINL void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's memory, and
// allow the next grid to start launching.
MOE_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
MOE_DEVINL void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace moe

// Host: launch with the programmatic-stream-serialization attribute; with
// `cooperative`, also as a cooperative launch (every CTA resident at once, or
// the launch fails), for kernels whose CTAs wait on one another.
namespace moe {
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_ex(bool cooperative, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cooperative ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    return launch_pdl_ex(false, kernel, grid, block, smem, s, std::forward<Args>(args)...);
}
}  // namespace moe
