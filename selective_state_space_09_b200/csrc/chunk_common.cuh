// chunk_common.cuh -- pieces shared by the chunked-matmul kernels (ssd.cu, gla.cu, chunk_scan.cuh):
// the chunk geometry, the base-2 exponential, CTA-wide prefix sums, row scaling of
// 128-byte-swizzled tiles, vector reductions to global memory, and the TMA map of a [B, L, X, W]
// bf16 tensor.
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

__device__ __forceinline__ void wg0_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// cta_inclusive_sum_n over the 128 threads of warpgroup 0 (named barrier 1; tmp: 4 * NV floats).
template <int NV>
__device__ __forceinline__ void wg0_inclusive_sum_n(float (&x)[NV], float* tmp) {
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
    wg0_bar();
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        float add = 0.0f;
        for (int w = 0; w < warp; ++w) add += tmp[w * NV + j];
        x[j] += add;
    }
    wg0_bar();
}

// Inclusive prefix sum over the 128 threads of warpgroup 0 (same order as cta_inclusive_sum);
// *total receives the sum of all 128 values.
__device__ __forceinline__ float wg0_inclusive_sum(float x, float* tmp, float* total = nullptr) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    wg0_bar();
    float add = 0.0f;
    for (int w = 0; w < warp; ++w) add += tmp[w];
    if (total) *total = ((tmp[0] + tmp[1]) + tmp[2]) + tmp[3];
    wg0_bar();
    return x + add;
}
// Sums of two values over the 128 threads of warpgroup 0, fixed order, results in every thread.
__device__ __forceinline__ float2 wg0_sum2(float x, float y, float* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, o);
        y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (lane == 0) {
        tmp[8 + warp] = x;
        tmp[12 + warp] = y;
    }
    wg0_bar();
    const float2 s = make_float2((tmp[8] + tmp[9]) + (tmp[10] + tmp[11]), (tmp[12] + tmp[13]) + (tmp[14] + tmp[15]));
    wg0_bar();
    return s;
}

// Pack 8 floats into 8 bf16 (one 16-byte chunk).
__device__ __forceinline__ uint4 pack_bf16x8(const float* f) {
    uint4 r;
    __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) hv[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    return r;
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
