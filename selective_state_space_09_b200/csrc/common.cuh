// common.cuh -- device-side building blocks shared by the scan kernels (sm_100a).
//
//  * TMA tile copies (cp.async.bulk.tensor, no multicast) completing on an mbarrier, and TMA
//    tile stores through bulk groups;
//  * mbarrier waits with an iteration bound: a wait that gives up records LR_ERR_TIMEOUT in the
//    workspace error record and returns false instead of spinning forever;
//  * acquire / release flag accesses for the single-pass chained scan across tiles;
//  * the workspace header (error record and tile tickets).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lrscan.h"

namespace lrs {

// ----------------------------------------------------------------------------- workspace header
// First 256 bytes of every workspace.  Zeroed by the host (cudaMemsetAsync) before each call.
struct WsHeader {
    unsigned int err;       // first device-side error status (0 = none)
    int info;               // kernel-specific detail of that error
    unsigned int ticket[6]; // dynamic tile tickets, one per kernel of a call
    unsigned int pad[56];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// Bounded waits give up after this long (ns of %globaltimer) and record LR_ERR_TIMEOUT.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Records the first error of a call in the workspace header.  A kernel launched as a programmatic
// dependent may run before the kernel ahead of it has finished zeroing that header, so it waits for
// that kernel first (griddepcontrol.wait; immediate in any other launch).  Only failure paths get
// here, and no kernel ahead of another waits on the one behind it.
__device__ __forceinline__ void record_error(WsHeader* hdr, unsigned int code, int info) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (atomicCAS(&hdr->err, 0u, code) == 0u) atomicExch(&hdr->info, info);
}

// ------------------------------------------------------------------------------ numeric I/O
template <typename T> struct IO;
// ld2 / st2: two adjacent elements at an even element index (one 8- or 4-byte access).
template <> struct IO<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
    static __device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }
    static __device__ __forceinline__ void st2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
    static __device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    }
    static __device__ __forceinline__ void st2(__nv_bfloat16* p, float2 v) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __float22bfloat162_rn(v);
    }
};

// ------------------------------------------------------------------------------ smem addresses
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// Bounded wait for phase `parity` of `bar`.  Returns false (and records LR_ERR_TIMEOUT) if the
// phase did not complete within kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr, int info) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    record_error(hdr, LR_ERR_TIMEOUT, info);
    return false;
}

// ------------------------------------------------------------------------------------- TMA
// 3-D tiled load global -> shared, completion counted on `bar` (bytes).  No multicast.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tiled prefetch of a box into L2 (a hint: no shared memory, no barrier; out-of-range parts
// are ignored).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// 3-D tiled store shared -> global (out-of-range rows/columns of the box are clipped).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// 4-D tiled load / store (same conventions as the 3-D forms).
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Contiguous copy global -> shared of `bytes` (multiple of 16, both addresses 16-byte aligned),
// completion counted on `bar`.  No multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem_dst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Arrive on `bar` without expecting bytes (completes a phase that has no copies).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 1-D bulk copy shared -> global (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until at most one bulk group (the most recent) still reads shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// All but the most recent bulk group have completed (their writes performed).
__device__ __forceinline__ void bulk_wait_all_but_1() { asm volatile("cp.async.bulk.wait_group 1;" ::: "memory"); }
// Orders this thread's global accesses through the async proxy (bulk / TMA copies) against its
// generic-proxy accesses (flag stores and loads).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------ programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while the previous kernel of
// the stream is still running.  pdl_launch_dependents lets the next kernel start its independent
// prologue; pdl_wait blocks the calling thread until the previous kernel has completed and its
// writes are visible (it returns at once when there is no such kernel).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------- cross-CTA flag protocol
__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned int* p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// The same between the threads of one CTA, on a shared-memory word.
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta(int* p, int v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Status of a tile's carry record in the chained scan.
enum : unsigned int { kFlagNone = 0, kFlagAgg = 1, kFlagPrefix = 2 };

// Poll `flag` until it is non-zero, for at most kWaitLimitNs.  Returns the flag, or kFlagNone
// after giving up (an error is then recorded).
__device__ __forceinline__ unsigned int wait_flag(const unsigned int* flag, WsHeader* hdr, int info) {
    unsigned int f = ld_acquire(flag);
    if (f != kFlagNone) return f;
    const unsigned long long t0 = global_ns();
    for (int i = 0;; ++i) {
        f = ld_acquire(flag);
        if (f != kFlagNone) return f;
        if (i > 16) __nanosleep(128);
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    record_error(hdr, LR_ERR_TIMEOUT, info);
    return kFlagNone;
}

// Counter protocol: producers add 1 with release semantics, a consumer polls with acquire loads
// until the counter reaches `target` (at most kWaitLimitNs; false after giving up, an error is
// then recorded).  One acquire load covers every producer counted.
__device__ __forceinline__ void red_release_add(unsigned int* p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ bool wait_count(const unsigned int* p, unsigned int target, WsHeader* hdr, int info) {
    if (ld_acquire(p) >= target) return true;
    const unsigned long long t0 = global_ns();
    for (int i = 0;; ++i) {
        if (ld_acquire(p) >= target) return true;
        if (i > 16) __nanosleep(128);
        if (global_ns() - t0 > kWaitLimitNs) break;
    }
    record_error(hdr, LR_ERR_TIMEOUT, info);
    return false;
}

// Dynamic tile ticket: tiles are numbered in the order CTAs start, so that every tile a CTA may
// wait on belongs to a CTA that has already started.
__device__ __forceinline__ unsigned int take_ticket(WsHeader* hdr, int which) {
    return atomicAdd(&hdr->ticket[which], 1u);
}

// ------------------------------------------------------------------------- complex helpers
struct cpx {
    float r, i;
};
__device__ __forceinline__ cpx cmul(cpx a, cpx b) {
    return {fmaf(a.r, b.r, -a.i * b.i), fmaf(a.r, b.i, a.i * b.r)};
}
__device__ __forceinline__ cpx cfma(cpx a, cpx b, cpx c) {  // a*b + c
    return {fmaf(a.r, b.r, fmaf(-a.i, b.i, c.r)), fmaf(a.r, b.i, fmaf(a.i, b.r, c.i))};
}
__device__ __forceinline__ cpx conjc(cpx a) { return {a.r, -a.i}; }

}  // namespace lrs
