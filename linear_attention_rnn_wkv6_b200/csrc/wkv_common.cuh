// wkv_common.cuh -- device helpers shared by the WKV kernels (sm_100a).
//
// Staging uses the Tensor Memory Accelerator: one elected thread issues
// cp.async.bulk.tensor loads of [rows x 64] tiles of the [B,T,C] inputs into
// shared memory and an mbarrier counts the bytes in; consumers wait on the
// barrier's phase.  Every wait is bounded (one second of %globaltimer); a wait
// that runs out records WKV_FAULT_TIMEOUT in g_wkv_faults and the kernel stops.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/wkv.h"

namespace wkv {

extern __device__ unsigned int g_wkv_faults;

constexpr int kHead = 64;                    // compiled head size N
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // bounded waits: 1 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) writes to the same buffers.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the barrier phase with the given parity to complete, for at most
// kWaitLimitNs.  Returns false (and records the fault) if the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_wkv_faults, WKV_FAULT_TIMEOUT);
            return false;
        }
        __nanosleep(64);
    }
}

// After a wait ran out at chunk g: give the copies still in flight (chunk g and,
// if issued, chunk g+1, on a two-stage ring) one more bounded wait each so the
// CTA does not exit while the TMA may still write its shared memory.
__device__ __forceinline__ void drain_two_stage(uint64_t *full, int g, int nchunks) {
    if (threadIdx.x != 0) return;
    mbar_wait_bounded(&full[g & 1], (g >> 1) & 1);
    if (g + 1 < nchunks) mbar_wait_bounded(&full[(g + 1) & 1], ((g + 1) >> 1) & 1);
}

// 3-D tiled TMA load (box described by the tensor map) into shared memory,
// completion counted on `bar`.  Coordinates are (c, t, b); c must be a
// multiple of 16 bytes / element size, t may be negative or past the end
// (those rows are zero filled).
// Tiled TMA store of a shared-memory box to a 3-D map; elements outside the
// tensor are not written.  Completion is tracked with the bulk-group helpers.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c, int t, int b) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c), "r"(t), "r"(b), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The source shared memory of every committed store may be reused.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed store has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c, int t, int b,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c), "r"(t), "r"(b), "r"(smem_u32(bar))
        : "memory");
}

// Prefetch one tile of a 3-D tensor map into L2 (no shared-memory destination,
// no completion to wait for; out-of-range parts are ignored).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *map, int c, int t, int b) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(c), "r"(t), "r"(b)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Index checks of the debug build.  Built with -DWKV_DEVICE_CHECKS=1
// (libwkv_debug.so), every global store of the kernels (and every L2 prefetch of
// an output row) first checks its element index against the size of the array it
// writes; an index out of range skips the access and records WKV_FAULT_INDEX in the fault word (the kernel goes on; nothing
// traps).  In the other builds the check is the constant true and compiles away.
#ifndef WKV_DEVICE_CHECKS
#define WKV_DEVICE_CHECKS 0
#endif
// The check itself, in every build (the debug build's in_range, and the self-test).
__device__ __forceinline__ bool in_range_checked(size_t idx, size_t n) {
    if (idx >= n) {
        atomicOr(&g_wkv_faults, WKV_FAULT_INDEX);
        return false;
    }
    return true;
}
__device__ __forceinline__ bool in_range(size_t idx, size_t n) {
#if WKV_DEVICE_CHECKS
    return in_range_checked(idx, n);
#else
    (void)idx;
    (void)n;
    return true;
#endif
}
// The same check for a vector store of `width` elements starting at idx.
__device__ __forceinline__ bool in_range_vec(size_t idx, int width, size_t n) {
    return in_range(idx, n) && in_range(idx + (size_t)(width - 1), n);
}

// exp(x) for the decay factorisation: exp2 of x*log2(e) on the SFU.
__device__ __forceinline__ float fast_exp(float x) { return exp2f(x * 1.4426950408889634f); }

}  // namespace wkv
