// tc.cuh -- 5th-generation tensor-core (tcgen05) building blocks for sm_100a: TMEM allocation,
// shared-memory matrix descriptors for 128-byte-swizzled bf16 tiles, the bf16 x bf16 -> f32 MMA,
// its commit to an mbarrier, and TMEM -> register loads.
//
// Tile format used throughout ("SW128 tile"): a rows x cols bf16 matrix stored as cols/64
// column blocks; each block is rows x 128 bytes, row r at byte r*128, and the 16-byte chunk c of a
// row stored at chunk position c ^ (r % 8).  This is what a TMA box of 64 x rows bf16 with 128-byte
// swizzle writes, and what the MMA reads through a descriptor with 128-byte swizzling:
//   K-major operand (K = the 64-wide column direction): rows are M (or N); one K = 16 step is a
//     32-byte advance of the start address inside the 128-byte row; the next 64 K values are the
//     next column block; stride between 8-row groups (SBO) = 1024 bytes.
//   MN-major operand (MN = the column direction, K = rows): one K = 16 step is 16 rows = 2048
//     bytes; stride between 64-wide MN blocks (LBO) = the block size rows*128; SBO = 1024 bytes.
// Every tile must start on a 1024-byte boundary.
#pragma once

#include "common.cuh"

namespace lrs {
namespace tc {

// element (r, c) of an SW128 tile with `rows` rows: byte offset from the tile start
__host__ __device__ __forceinline__ uint32_t sw128_off(int r, int c, int rows) {
    const int blk = c >> 6, cc = c & 63, chunk = cc >> 3;
    return (uint32_t)(blk * rows * 128 + r * 128 + ((chunk ^ (r & 7)) << 4) + ((cc & 7) << 1));
}

// --------------------------------------------------------------------------- descriptors
__device__ __forceinline__ uint64_t desc_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // descriptor version of this architecture
    d |= (uint64_t)2u << 61;  // 128-byte swizzle
    return d;
}

// Instruction descriptor: bf16 A and B, f32 accumulator, M x N, operand majors (0 = K, 1 = MN).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------------------------ TMEM
// Executed by one whole warp.  Writes the allocated base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] = A * B (+ D if accumulate), issued by one thread.
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                    uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] = A[tmem] * B (+ D if accumulate): A (M = 128 rows = lanes, bf16 pairs packed in 32-bit
// columns, K/2 columns) read from tensor memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 16 columns of 32-bit values: thread l of the warp gets lane (lane base + l).
__device__ __forceinline__ void ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Store 16 32-bit columns of this thread's lane.
__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Descriptor of an SW128 tile at the start of a product: the start address advances by a
// compile-time number of 16-byte units per K = 16 step, so the per-step descriptor is the base
// descriptor plus a small constant (the address field is the low 14 bits and never carries:
// shared memory ends below 256 KB).
//   K-major (mn = 0): +32 bytes per step inside a 64-wide block, +rows * 128 bytes per block;
//   MN-major (mn = 1): +16 rows = 2048 bytes per step.
__device__ __forceinline__ uint64_t tile_desc(uint32_t base, int mn, int rows) {
    return desc_sw128(base, mn ? (uint32_t)rows * 128u : 16u, 1024);
}
__device__ __forceinline__ uint32_t tile_step(int k, int mn, int rows) {
    return mn ? (uint32_t)k * 8u : (uint32_t)(k >> 6) * (uint32_t)rows * 8u + (uint32_t)((k & 63) >> 3);
}

// M = 128 x N x K product with A in tensor memory (a_tmem: K/2 columns) and B an SW128 tile.
__device__ __forceinline__ void mma_ts_tiles(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_base, int b_mn, int b_rows,
                                             int N, int K, uint32_t accumulate_first) {
    const uint32_t idesc = idesc_bf16(128, N, 0, b_mn);
    const uint64_t b0 = tile_desc(b_base, b_mn, b_rows);
#pragma unroll
    for (int k = 0; k < K; k += 16)
        mma_ts(d_tmem, a_tmem + (uint32_t)(k >> 1), b0 + tile_step(k, b_mn, b_rows), idesc,
               (k > 0 || accumulate_first) ? 1u : 0u);
}

// Issue an M x N x K product as K/16 MMAs over SW128 tiles.
//   a: K-major (a_mn = 0: rows = M, 64-wide blocks along K of `a_rows` rows) or MN-major
//      (a_mn = 1: rows = K, blocks along M, block size a_rows*128 where a_rows = K extent)
//   b: same conventions with N in place of M.
__device__ __forceinline__ void mma_tiles(uint32_t d_tmem, uint32_t a_base, int a_mn, int a_rows,
                                          uint32_t b_base, int b_mn, int b_rows, int M, int N, int K,
                                          uint32_t accumulate_first) {
    const uint32_t idesc = idesc_bf16(M, N, a_mn, b_mn);
    const uint64_t a0 = tile_desc(a_base, a_mn, a_rows), b0 = tile_desc(b_base, b_mn, b_rows);
#pragma unroll
    for (int k = 0; k < K; k += 16)
        mma(d_tmem, a0 + tile_step(k, a_mn, a_rows), b0 + tile_step(k, b_mn, b_rows), idesc,
            (k > 0 || accumulate_first) ? 1u : 0u);
}

}  // namespace tc
}  // namespace lrs
