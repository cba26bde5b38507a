// noalloc.cu -- rglru forward pass whose scratch memory is a fixed, library-owned device array,
// for callers that cannot allocate device memory themselves.
//
// Some callers have no way to hand the library a workspace: code running inside a host framework
// that owns every device byte through its own pool (a cudaMalloc behind its back breaks its
// accounting, and the framework exposes no scratch to plug-ins), hosts that only let a plug-in
// run a fixed callback with the tensors they pass in, and latency-critical loops in which a
// cudaMalloc / cudaFree would synchronise the device.  lr_rglru_fwd_noalloc serves them: it runs
// the same rglru forward kernel as lr_scan_fwd, but its carry records and flags live in the
// static array below, so the call allocates nothing (no cudaMalloc, no cudaFree, no allocating
// library routine).
//
// The array is part of the library image: every GPU that loads the library holds these
// kNoAllocScratchBytes until the process exits.  All calls on a device share it and it keeps the
// previous call's contents, so each call first clears the part that must start at zero (flags
// and tile tickets); calls that overlap on the GPU (different streams, no ordering) race on it.
#include <mutex>

#include "common.cuh"
#include "host_common.h"

namespace lrs {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB

// File-scope device array.  In host code `g_noalloc_scratch` is only a host-side handle of the
// symbol, not a device address: its address is obtained with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {nullptr};

// Device address of the array on the current device (looked up once per device).
lr_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LR_ERR_CUDA;
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return LR_OK;
}

}  // namespace
}  // namespace lrs

using namespace lrs;

extern "C" lr_status lr_rglru_fwd_noalloc(const lr_desc* desc, const void* a, const void* b,
                                          void* y, void* ckpt, void* stream, int check) {
    reset_dispatch();
    if (!desc || desc->kind != LR_RGLRU) return LR_ERR_INVALID_ARG;
    if (desc->flags & LR_RGLRU_GATES) return LR_ERR_UNSUPPORTED;  // no gate inputs in this signature
    lr_status s = lr_validate(desc);
    if (s != LR_OK) return s;
    if (!a || !b || !y || !ckpt) return LR_ERR_INVALID_ARG;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al(a) || !al(b) || !al(y) || !al(ckpt)) return LR_ERR_ALIGNMENT;
    const size_t need = diag_ws_bytes(*desc, false);
    if (need > kNoAllocScratchBytes) return LR_ERR_WORKSPACE;  // problem too large for the array
    void* ws = nullptr;
    s = scratch_address(&ws);
    if (s != LR_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    set_launch_stream(st);
    if (cudaMemsetAsync(ws, 0, diag_flag_bytes(*desc, false), st) != cudaSuccess) return LR_ERR_CUDA;
    lr_inputs in{};
    in.a = a;
    in.b = b;
    s = diag_fwd(*desc, in, y, ckpt, static_cast<char*>(ws), st);
    if (s != LR_OK || !check) return s;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LR_ERR_CUDA;
    unsigned int err = 0;
    if (cudaMemcpy(&err, ws, sizeof(err), cudaMemcpyDeviceToHost) != cudaSuccess) return LR_ERR_CUDA;
    return static_cast<lr_status>(err);
}

// The device-side status of the last lr_rglru_fwd_noalloc call on the current device, for callers
// that enqueue with check = 0: synchronises `stream`, reads the error record at the start of the
// array and clears it (the record lr_get_error reads from a caller's workspace).  Each call of
// lr_rglru_fwd_noalloc clears the record when it starts, so a status is lost once the next call
// on the device is enqueued.
extern "C" lr_status lr_rglru_noalloc_error(void* stream, int32_t* info) {
    void* ws = nullptr;
    lr_status s = scratch_address(&ws);
    if (s != LR_OK) return s;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return LR_ERR_CUDA;
    WsHeader h;
    if (cudaMemcpy(&h, ws, 8, cudaMemcpyDeviceToHost) != cudaSuccess) return LR_ERR_CUDA;
    if (cudaMemset(ws, 0, 8) != cudaSuccess) return LR_ERR_CUDA;
    if (info) *info = h.info;
    return static_cast<lr_status>(h.err);
}
