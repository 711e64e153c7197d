// pipeline.cuh - shared-memory producer/consumer pipelines on sm_100a:
// mbarriers, 1-D bulk copies and 2-D tiled loads (the TMA engine) and waits
// that give up after a bounded number of tries instead of hanging.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace coli {

// device error flags written by kernels into the workspace (bit or)
constexpr int32_t kErrWaitTimeout = 1;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// make initialised barriers visible to the async (bulk copy) proxy
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// arrive once and announce `bytes` of bulk-copy data that will complete the phase
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Each try may suspend the thread for a hardware-chosen time; this many tries
// is well beyond any legitimate wait (seconds), after which the wait is
// abandoned, kErrWaitTimeout is or-ed into *err and false is returned.
constexpr uint32_t kWaitTries = 1u << 22;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err,
                                          uint32_t tries = kWaitTries) {
    for (uint32_t i = 0; i < tries; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    if (err) atomicOr(err, kErrWaitTimeout);
    return false;
}

// Warp-wide wait in which each try may sleep until the phase completes or 20 us
// pass (a suspend-time hint), so that a waiting warp issues almost nothing: for
// kernels with many warps waiting at once.  At most kSleepTries tries (about a
// second), then kErrWaitTimeout as for mbar_wait.
constexpr uint32_t kSleepTries = 1u << 16;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.b32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_warp_sleep(uint64_t* bar, uint32_t parity, int32_t* err) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) {
        ok = 0;
        for (uint32_t i = 0; i < kSleepTries; ++i)
            if (mbar_try_wait_sleep(bar, parity)) { ok = 1; break; }
        if (!ok && err) atomicOr(err, kErrWaitTimeout);
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Warp-wide wait: lane 0 polls the barrier while the other lanes sleep at the
// warp barrier, which then orders their reads after lane 0's acquire.  Keeps the
// mbarrier unit free for the arrivals and transaction counts that make progress
// (every lane polling floods it).  Every lane gets lane 0's result.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, int32_t* err) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// global -> shared bulk copy, completion counted in bytes on `bar`.  Both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// The *_elect variants are executed by every lane of a converged warp with
// warp-uniform operands; one lane elected by elect.sync issues the operation.
// Issued that way the operands stay in uniform registers, which makes the
// async-copy and tensor-core instructions several times cheaper to issue than
// from a lone lane in a divergent branch.
__device__ __forceinline__ void mbar_expect_tx_elect(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n}"
        ::"r"(smem_u32(bar)), "r"(bytes)
        : "memory");
}

__device__ __forceinline__ void bulk_g2s_elect(void* dst, const void* src, uint32_t bytes,
                                               uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n}"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read exactly once (weights streamed into the ring)
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// global -> shared bulk copy with an L2 cache policy (warp-uniform operands;
// one elected lane issues)
__device__ __forceinline__ void bulk_g2s_hint_elect(void* dst, const void* src, uint32_t bytes,
                                                    uint64_t* bar, uint64_t pol) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;\n}"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// 2-D tiled TMA load of the box at (x, y) of `map` into shared memory,
// completion counted in bytes on `bar` (warp-uniform operands; one elected
// lane issues).  x times the element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d_elect(void* dst, const CUtensorMap* map, int x, int y,
                                                  uint64_t* bar) {
    asm volatile(
        "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
        " @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n}"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// barrier among the first `threads` threads of the CTA (named barrier 1)
__device__ __forceinline__ void named_sync(int threads) {
    asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

}  // namespace coli
