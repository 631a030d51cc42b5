// bulk.cuh -- the 1-D bulk-copy engine and shared-memory barriers (mbarrier) of sm_100a,
// as the decode and encode kernels use them: one thread arms a barrier with the bytes it
// expects and starts a global -> shared copy that completes on it; the consumers wait on
// the barrier's phase with a bounded wait.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dfx {
namespace {

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(unsigned long long* bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
// orders this thread's (and, after a warp barrier, the warp's) earlier generic accesses to
// shared memory before the bulk copies it issues next
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
// arm `bar` for `bytes` and copy them from global `src` to shared `dst` (both 16-byte
// aligned, bytes a multiple of 16)
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}
// Wait for the phase with the given parity of `bar` to complete.  One blocking poll first
// (try_wait, which suspends the warp for at most the 100 us time hint: staged data
// normally lands within it), then non-blocking polls (test_wait) with a sleep of at most
// 128 ns between them (__nanosleep(64) lasts at most twice its argument); a wait that
// never completes gives up after ~0.1 ms + ~0.35 s and the caller reports
// DFX_STATUS_TIMEOUT.
constexpr uint32_t kWaitPolls = 1u << 21;
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity) {
    const uint32_t addr = smem_addr(bar);
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 100000;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    for (uint32_t i = 0; i < kWaitPolls; i++) {
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
        __nanosleep(64);
    }
    return false;
}
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p) : "memory");
}
}  // namespace
}  // namespace dfx
