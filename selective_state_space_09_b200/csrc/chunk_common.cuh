// chunk_common.cuh -- pieces shared by the chunked-matmul kernels (chunk.cu, ssd.cu): the chunk
// geometry, the base-2 exponential, CTA-wide prefix sums, row scaling of 128-byte-swizzled tiles,
// vector reductions to global memory, and the TMA map of a [B, L, X, W] bf16 tensor.
#pragma once

#include "common.cuh"
#include "host_common.h"
#include "tc.cuh"

namespace lrs {
namespace chunkc {

constexpr int kQ = 128;        // chunk length (rows of every tile, M of every MMA)
constexpr int kKD = 128;       // key / state-row dimension (N of SSD, K of GLA)
constexpr int kThreads = 128;  // 4 warps: thread i <-> row / TMEM lane i
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ char* smem_base1024() {
    extern __shared__ char dyn_smem[];
    uintptr_t p = reinterpret_cast<uintptr_t>(dyn_smem);
    return reinterpret_cast<char*>((p + 1023) & ~uintptr_t(1023));
}

// Inclusive prefix sum over the 128 threads of the CTA (tmp: 4 floats of shared memory).
__device__ __forceinline__ float cta_inclusive_sum(float x, float* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    float add = 0.0f;
    for (int w = 0; w < warp; ++w) add += tmp[w];
    __syncthreads();
    return x + add;
}

// Inclusive prefix sums of NV values per thread over the 128 threads of the CTA (tmp: 4 * NV
// floats of shared memory).  Same operation order as cta_inclusive_sum for each value.
template <int NV>
__device__ __forceinline__ void cta_inclusive_sum_n(float (&x)[NV], float* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const float y = __shfl_up_sync(0xffffffffu, x[j], o);
            if (lane >= o) x[j] += y;
        }
    }
    if (lane == 31) {
#pragma unroll
        for (int j = 0; j < NV; ++j) tmp[warp * NV + j] = x[j];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        float add = 0.0f;
        for (int w = 0; w < warp; ++w) add += tmp[w * NV + j];
        x[j] += add;
    }
    __syncthreads();
}

// Fire-and-forget vector add of four floats to global memory (relaxed, gpu scope).
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// Scale row r (cols [0, cols)) of an SW128 tile with `rows` rows by w, in place.
__device__ __forceinline__ void scale_row(char* tile, int r, int cols, int rows, float w) {
    for (int c0 = 0; c0 < cols; c0 += 8) {
        uint4 raw = *reinterpret_cast<const uint4*>(tile + tc::sw128_off(r, c0, rows));
        __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(hv[i]);
            hv[i] = __floats2bfloat162_rn(f.x * w, f.y * w);
        }
        *reinterpret_cast<uint4*>(tile + tc::sw128_off(r, c0, rows)) = raw;
    }
}

// rank-4 map of a [B, L, X, W] bf16 tensor (W contiguous) with box [1, 128 rows, 1, 64 cols]
inline bool map4(CUtensorMap* m, const void* p, uint64_t W, uint64_t X, uint64_t L, uint64_t B, bool swz) {
    uint64_t dims[4] = {W, X, L, B};
    uint64_t str[3] = {W * 2, X * W * 2, L * X * W * 2};
    uint32_t box[4] = {64, 1, (uint32_t)kQ, 1};
    return make_tmap(m, p, 2, 4, dims, str, box, swz);
}

}  // namespace chunkc
}  // namespace lrs
