// chunk.cu -- shape rules and dispatch of the chunked-matmul kinds: SSD (ssd.cu) and GLA (gla.cu).
//
// Both kinds are the recurrence S_t = e^{lam_t} S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t with a
// scalar decay per step and head ("mlx-recurrence", Apple Developer Forums thread 840535,
// "Current kernels": ssd_scan, gla_scan), evaluated in 128-step chunks on tcgen05 tensor cores:
// per pass, the chunk states (SSD: one scan kernel; GLA: a chunk-state kernel and an elementwise
// state-passing kernel) and a chunk kernel.
#include "chunk_common.cuh"

namespace lrs {
using namespace chunkc;

bool chunk_supported(const lr_desc& d) {
    if (d.io != LR_BF16) return false;
    if (d.N != kKD || (d.P != 64 && d.P != 128)) return false;
    if (d.segment % kQ != 0 || (d.chunk != 0 && d.chunk != kQ)) return false;  // segments of whole chunks
    // SSD: the decays are kept as chunk-local log sums (with a sign parity for bilinear, whose abar
    // can be negative)
    if (d.kind == LR_SSD && d.P != 64) return false;
    return d.L <= (1 << 28) && d.H <= 4096;
}

size_t chunk_ws_bytes(const lr_desc& d, bool bwd) {
    return d.kind == LR_SSD ? (bwd ? ssd_bwd_ws_bytes(d) : ssd_fwd_ws_bytes(d)) : gla_ws_bytes(d, bwd);
}
size_t chunk_flag_bytes(const lr_desc& d, bool bwd) {
    return d.kind == LR_SSD ? (bwd ? ssd_bwd_flag_bytes(d) : ssd_fwd_flag_bytes(d)) : gla_flag_bytes(d, bwd);
}

lr_status chunk_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws, cudaStream_t st) {
    return d.kind == LR_SSD ? ssd_fwd(d, in, y, ckpt, ws, st) : gla_fwd(d, in, y, ckpt, ws, st);
}

lr_status chunk_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt, const lr_grads& gr,
                    char* ws, cudaStream_t st) {
    return d.kind == LR_SSD ? ssd_bwd(d, in, dy, ckpt, gr, ws, st) : gla_bwd(d, in, dy, ckpt, gr, ws, st);
}

}  // namespace lrs
