// host_common.h -- host-side helpers shared by the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lrscan.h"

namespace lrs {

// Round up to a multiple of `a`.
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Records the name of a kernel about to be launched on this host thread (fingerprint for
// lr_last_dispatch / lr_last_launch_count).
void note_launch(const char* name);

// Clears this host thread's launch fingerprint (start of an entry-point call).
void reset_dispatch();

// Stream of the current entry-point call (where the timing hook records its events).
void set_launch_stream(cudaStream_t st);

// Converts the last CUDA error into a status.
lr_status check_launch();

// Builds a tiled TMA descriptor of a rank-3 row-major tensor [d2][d1][d0] (d0 contiguous) of
// element size `esize` (4 = f32, 2 = bf16) with box [1][box1][box0].  Returns false if the
// driver rejects the description.
bool make_tmap_3d(CUtensorMap* map, const void* base, int esize, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint32_t box0, uint32_t box1);

// Builds a tiled TMA descriptor of a row-major tensor of rank 2..5 (dims[0] contiguous;
// strides[i] = byte stride of dimension i+1).  swizzle128 selects the 128-byte swizzle (box[0] *
// esize must then be 128).  Returns false if the driver rejects the description.
bool make_tmap(CUtensorMap* map, const void* base, int esize, int rank, const uint64_t* dims,
               const uint64_t* strides, const uint32_t* box, bool swizzle128);

// Launches `kernel` on `st` with programmatic stream serialization (launch_ex: unless
// `programmatic` is false): it may start while the previous kernel of the stream runs and must
// call pdl_wait before touching that kernel's outputs (or anything it reads).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool programmatic, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
// launch_ex with the grid cut into thread-block clusters of `cluster` consecutive blocks along x
// (cluster <= 1: no clusters); the grid's x extent must be a multiple of it.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              bool programmatic, int cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (programmatic) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    return launch_ex(kernel, grid, block, smem, st, true, args...);
}

// Number of SMs of the current device (queried on every call: a process may drive several devices).
inline int device_sm_count() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) ==
                                                      cudaSuccess && v > 0)
        return v;
    return 148;
}

// Byte offset bookkeeping for a workspace: a 256-byte header followed by regions.
struct WsCursor {
    size_t off = 256;
    size_t take(size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    }
};

// Per-kind entry points (defined in the kernel files).  *_supported: whether the library has
// kernels for the (already validated) descriptor.
bool s6_supported(const lr_desc& d);
bool chunk_supported(const lr_desc& d);
size_t diag_ws_bytes(const lr_desc& d, bool bwd);
size_t diag_flag_bytes(const lr_desc& d, bool bwd);
lr_status diag_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                   cudaStream_t st);
lr_status diag_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                   const lr_grads& gr, char* ws, cudaStream_t st);

size_t s6_ws_bytes(const lr_desc& d, bool bwd);
size_t s6_flag_bytes(const lr_desc& d, bool bwd);
lr_status s6_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                 cudaStream_t st);
lr_status s6_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                 const lr_grads& gr, char* ws, cudaStream_t st);

size_t chunk_ws_bytes(const lr_desc& d, bool bwd);
size_t chunk_flag_bytes(const lr_desc& d, bool bwd);
lr_status chunk_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                    cudaStream_t st);
lr_status chunk_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                    const lr_grads& gr, char* ws, cudaStream_t st);

size_t ssd_fwd_ws_bytes(const lr_desc& d);
size_t ssd_fwd_flag_bytes(const lr_desc& d);
lr_status ssd_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws, cudaStream_t st);
size_t gla_ws_bytes(const lr_desc& d, bool bwd);
size_t gla_flag_bytes(const lr_desc& d, bool bwd);
lr_status gla_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws, cudaStream_t st);
lr_status gla_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt, const lr_grads& gr,
                  char* ws, cudaStream_t st);
size_t ssd_bwd_ws_bytes(const lr_desc& d);
size_t ssd_bwd_flag_bytes(const lr_desc& d);
lr_status ssd_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt, const lr_grads& gr,
                  char* ws, cudaStream_t st);

// decode / continuation (step.cu)
bool step_supported(const lr_desc& d);
lr_status step_run(const lr_desc& d, const lr_inputs& in, const float* s_in, float* s_out, void* y,
                   cudaStream_t st);

}  // namespace lrs
