// calib.cu -- throughput probes of the two arithmetic pipes the S6 scan is bound by: the
// special-function unit (ex2.approx, the exponential of every discretisation step) and the fp32
// FMA pipe.  A benchmark times one launch with CUDA events and divides the results produced by
// the time, so the S6 roofline rests on rates measured on the part it runs on, not on a table.
//
// Each thread runs kChains independent dependency chains so that the pipe, not the latency of
// one chain, limits the rate; the chains' final values are summed into `out` so that nothing is
// eliminated.  Values stay bounded: x -> 2^(-x) maps [0, 1] into [0.5, 1], and the FMA chain
// x -> x * c + d with |c| < 1 converges.
#include <cuda_runtime.h>

#include "host_common.h"

namespace lrs {
namespace {

constexpr int kChains = 8;

__global__ void probe_ex2_kernel(float* out, int iters) {
    float v[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) v[k] = 0.001f * (threadIdx.x & 31) + 0.1f * k;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) {
            float y;
            asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-v[k]));
            v[k] = y;
        }
    }
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += v[k];
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void probe_ffma_kernel(float* out, int iters, float c, float d) {
    float v[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) v[k] = 0.001f * (threadIdx.x & 31) + 0.1f * k;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int k = 0; k < kChains; ++k) v[k] = fmaf(v[k], c, d);
    }
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += v[k];
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace
}  // namespace lrs

extern "C" int64_t lr_probe_pipe(int which, float* out, int blocks, int threads, int iters, void* stream) {
    if (!out || blocks < 1 || threads < 32 || threads > 1024 || threads % 32 || iters < 1) return -1;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (which == 0)
        lrs::probe_ex2_kernel<<<blocks, threads, 0, st>>>(out, iters);
    else if (which == 1)
        lrs::probe_ffma_kernel<<<blocks, threads, 0, st>>>(out, iters, 0.999f, 0.0005f);
    else
        return -1;
    if (cudaGetLastError() != cudaSuccess) return -1;
    return (int64_t)blocks * threads * iters * lrs::kChains;
}
