// Placeholder entry points for kinds whose kernels are not in this build yet: they report
// LR_ERR_UNSUPPORTED after validation.
#include "common.cuh"
#include "host_common.h"

namespace lrs {
bool chunk_supported(const lr_desc&) { return false; }
size_t chunk_ws_bytes(const lr_desc&, bool) { return 256; }
size_t chunk_flag_bytes(const lr_desc&, bool) { return 256; }
lr_status chunk_fwd(const lr_desc&, const lr_inputs&, void*, void*, char*, cudaStream_t) { return LR_ERR_UNSUPPORTED; }
lr_status chunk_bwd(const lr_desc&, const lr_inputs&, const void*, const void*, const lr_grads&, char*, cudaStream_t) { return LR_ERR_UNSUPPORTED; }
}  // namespace lrs
