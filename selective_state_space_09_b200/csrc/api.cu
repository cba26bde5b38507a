// api.cu -- the extern "C" boundary declared in include/lrscan.h: validation, size queries,
// dispatch by kind, the device error record and the launch fingerprint.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "host_common.h"

namespace lrs {

namespace {
thread_local std::string t_dispatch;
thread_local int t_launches = 0;
thread_local void* const* t_events = nullptr;  // lr_set_launch_events
thread_local int t_nevents = 0;
thread_local cudaStream_t t_stream = nullptr;  // stream of the current entry-point call

int esize(int io) { return io == LR_BF16 ? 2 : 4; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules of the library (also reported by lr_validate).
lr_status validate(const lr_desc* d) {
    if (!d) return LR_ERR_INVALID_ARG;
    if (d->kind < LR_RGLRU || d->kind > LR_GLA) return LR_ERR_INVALID_ARG;
    if (d->io != LR_F32 && d->io != LR_BF16) return LR_ERR_INVALID_ARG;
    if (d->B < 1 || d->L < 1 || d->segment < 1) return LR_ERR_INVALID_ARG;
    if (d->B > (1 << 20) || d->L > (1ll << 30)) return LR_ERR_UNSUPPORTED;
    if ((d->flags & LR_FULL_STATE) && d->kind != LR_RGLRU && d->kind != LR_ROTLRU && d->kind != LR_S6)
        return LR_ERR_UNSUPPORTED;
    if ((d->flags & LR_DELTA_SOFTPLUS) && d->kind != LR_S6 && d->kind != LR_SSD) return LR_ERR_INVALID_ARG;
    if (d->flags & LR_RGLRU_GATES) {
        if (d->kind != LR_RGLRU) return LR_ERR_INVALID_ARG;
        if (d->io != LR_F32 || (d->flags & LR_FULL_STATE)) return LR_ERR_UNSUPPORTED;
    }
    const int es = esize(d->io);
    switch (d->kind) {
        case LR_RGLRU:
        case LR_ROTLRU: {
            if (d->disc != LR_DISC_NONE) return LR_ERR_INVALID_ARG;
            if (d->D < 1) return LR_ERR_INVALID_ARG;
            if (d->kind == LR_ROTLRU && (d->D % 2)) return LR_ERR_INVALID_ARG;
            int64_t inner = d->kind == LR_RGLRU ? d->D : d->D / 2;  // a / g innermost extent
            if ((inner * es) % 16 || (d->D * es) % 16) return LR_ERR_ALIGNMENT;
            if (d->segment > 256) return LR_ERR_UNSUPPORTED;
            if (d->D > (1 << 24)) return LR_ERR_UNSUPPORTED;
            return LR_OK;
        }
        case LR_S6: {
            if (d->disc < LR_DISC_ZOH || d->disc > LR_DISC_ZOH_EULER) return LR_ERR_INVALID_ARG;
            if (d->D < 1 || d->N < 1) return LR_ERR_INVALID_ARG;
            if ((d->D * es) % 16 || (d->N * es) % 16) return LR_ERR_ALIGNMENT;
            return s6_supported(*d) ? LR_OK : LR_ERR_UNSUPPORTED;
        }
        case LR_SSD: {
            if (d->disc < LR_DISC_ZOH || d->disc > LR_DISC_ZOH_EULER) return LR_ERR_INVALID_ARG;
            if (d->H < 1 || d->P < 1 || d->N < 1 || d->G < 1 || d->H % d->G) return LR_ERR_INVALID_ARG;
            if ((d->P * es) % 16 || (d->N * es) % 16) return LR_ERR_ALIGNMENT;
            return chunk_supported(*d) ? LR_OK : LR_ERR_UNSUPPORTED;
        }
        case LR_GLA: {
            if (d->disc != LR_DISC_NONE) return LR_ERR_INVALID_ARG;
            if (d->H < 1 || d->P < 1 || d->N < 1) return LR_ERR_INVALID_ARG;
            if ((d->P * es) % 16 || (d->N * es) % 16) return LR_ERR_ALIGNMENT;
            return chunk_supported(*d) ? LR_OK : LR_ERR_UNSUPPORTED;
        }
    }
    return LR_ERR_INVALID_ARG;
}

size_t state_elems(const lr_desc& d) {
    switch (d.kind) {
        case LR_RGLRU:
        case LR_ROTLRU: return (size_t)d.B * d.D;
        case LR_S6: return (size_t)d.B * d.D * d.N;
        case LR_SSD: return (size_t)d.B * d.H * d.P * d.N;
        case LR_GLA: return (size_t)d.B * d.H * d.N * d.P;
    }
    return 0;
}

size_t ws_bytes(const lr_desc& d, bool bwd) {
    switch (d.kind) {
        case LR_RGLRU:
        case LR_ROTLRU: return diag_ws_bytes(d, bwd);
        case LR_S6: return s6_ws_bytes(d, bwd);
        default: return chunk_ws_bytes(d, bwd);
    }
}

size_t flag_bytes(const lr_desc& d, bool bwd) {
    switch (d.kind) {
        case LR_RGLRU:
        case LR_ROTLRU: return diag_flag_bytes(d, bwd);
        case LR_S6: return s6_flag_bytes(d, bwd);
        default: return chunk_flag_bytes(d, bwd);
    }
}

void begin_call() {
    t_dispatch.clear();
    t_launches = 0;
}

}  // namespace

void reset_dispatch() { begin_call(); }

void note_launch(const char* name) {
    if (!t_dispatch.empty()) t_dispatch += "+";
    t_dispatch += name;
    if (t_events && t_launches < t_nevents && t_events[t_launches])
        cudaEventRecord(static_cast<cudaEvent_t>(t_events[t_launches]), t_stream);
    ++t_launches;
}

void set_launch_stream(cudaStream_t st) { t_stream = st; }

lr_status check_launch() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return encode;
}
// The tensor-map encoder is a driver call and needs a current context on the calling thread; a
// thread whose first CUDA call of the process is this one (a framework's worker thread, say) has
// none yet.  A runtime call binds the current device's primary context to the thread.
bool bind_context() { return cudaFree(nullptr) == cudaSuccess; }
}  // namespace

bool make_tmap(CUtensorMap* map, const void* base, int esize, int rank, const uint64_t* dims,
               const uint64_t* strides, const uint32_t* box, bool swizzle128) {
    auto encode = tmap_encoder();
    if (!encode || rank < 2 || rank > 5) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) s[i] = strides[i];
    auto run = [&] {
        return encode(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank,
                      const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    };
    CUresult r = run();
    if (r == CUDA_ERROR_INVALID_CONTEXT && bind_context()) r = run();
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, int esize_, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint32_t box0, uint32_t box1) {
    auto encode = tmap_encoder();
    if (!encode) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * esize_, d0 * d1 * esize_};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    auto run = [&] {
        return encode(map, esize_ == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    };
    CUresult r = run();
    if (r == CUDA_ERROR_INVALID_CONTEXT && bind_context()) r = run();
    return r == CUDA_SUCCESS;
}

}  // namespace lrs

using namespace lrs;

extern "C" {

int lr_version(void) { return LRSCAN_VERSION; }

lr_status lr_validate(const lr_desc* desc) { return validate(desc); }

size_t lr_ckpt_bytes(const lr_desc* desc) {
    if (validate(desc) != LR_OK) return 0;
    size_t nseg = (desc->flags & LR_FULL_STATE) ? (size_t)desc->L
                                                : (size_t)((desc->L + desc->segment - 1) / desc->segment);
    // SSD, GLA with one chunk per segment: the f32 states are followed by a bf16 copy of each in
    // tensor-core tile order (longer segments: the f32 states only)
    const bool tiles = (desc->kind == LR_SSD || desc->kind == LR_GLA) && desc->segment == 128;
    const size_t per = tiles ? sizeof(float) + 2 : sizeof(float);
    return nseg * state_elems(*desc) * per;
}

size_t lr_workspace_bytes(const lr_desc* desc, int backward) {
    if (validate(desc) != LR_OK) return 0;
    return ws_bytes(*desc, backward != 0);
}

lr_status lr_scan_fwd(const lr_desc* desc, const lr_inputs* in, void* y, void* ckpt, void* ws,
                      size_t ws_size, void* stream) {
    begin_call();
    lr_status s = validate(desc);
    if (s != LR_OK) return s;
    if (!in || !y || !ckpt || !ws) return LR_ERR_INVALID_ARG;
    const lr_desc& d = *desc;
    const void* need[8] = {nullptr};
    int nn = 0;
    switch (d.kind) {
        case LR_RGLRU:
            need[nn++] = in->a; need[nn++] = in->b;
            if (d.flags & LR_RGLRU_GATES) { need[nn++] = in->x; need[nn++] = in->A; }
            break;
        case LR_ROTLRU: need[nn++] = in->b; need[nn++] = in->g; need[nn++] = in->mag; need[nn++] = in->theta; break;
        case LR_S6:
        case LR_SSD:
            need[nn++] = in->x; need[nn++] = in->delta; need[nn++] = in->A; need[nn++] = in->Bm; need[nn++] = in->Cm;
            if (d.flags & LR_HAS_DSKIP) need[nn++] = in->Dskip;
            if (d.flags & LR_HAS_Z) need[nn++] = in->z;
            break;
        case LR_GLA: need[nn++] = in->q; need[nn++] = in->k; need[nn++] = in->v; need[nn++] = in->g; break;
    }
    for (int i = 0; i < nn; ++i) {
        if (!need[i]) return LR_ERR_INVALID_ARG;
        if (!aligned16(need[i])) return LR_ERR_ALIGNMENT;
    }
    if (!aligned16(y) || !aligned16(ckpt) || !aligned16(ws)) return LR_ERR_ALIGNMENT;
    if (ws_size < ws_bytes(d, false)) return LR_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    set_launch_stream(st);
    // the diagonal kinds zero their workspace head in a kernel their scan kernel overlaps
    const bool diag = d.kind == LR_RGLRU || d.kind == LR_ROTLRU;
    if (!diag && cudaMemsetAsync(ws, 0, flag_bytes(d, false), st) != cudaSuccess) return LR_ERR_CUDA;
    switch (d.kind) {
        case LR_RGLRU:
        case LR_ROTLRU: return diag_fwd(d, *in, y, ckpt, (char*)ws, st);
        case LR_S6: return s6_fwd(d, *in, y, ckpt, (char*)ws, st);
        default: return chunk_fwd(d, *in, y, ckpt, (char*)ws, st);
    }
}

lr_status lr_scan_bwd(const lr_desc* desc, const lr_inputs* in, const void* dy, const void* ckpt,
                      lr_grads* gr, void* ws, size_t ws_size, void* stream) {
    begin_call();
    lr_status s = validate(desc);
    if (s != LR_OK) return s;
    if (!in || !dy || !ckpt || !gr || !ws) return LR_ERR_INVALID_ARG;
    const lr_desc& d = *desc;
    const void* need[20] = {nullptr};
    int nn = 0;
    switch (d.kind) {
        case LR_RGLRU:
            need[nn++] = in->a; need[nn++] = in->b; need[nn++] = gr->da; need[nn++] = gr->db;
            if (d.flags & LR_RGLRU_GATES) {  // dA (dLambda) may be NULL
                need[nn++] = in->x; need[nn++] = in->A; need[nn++] = gr->dx;
                if (gr->dA && !aligned16(gr->dA)) return LR_ERR_ALIGNMENT;
            }
            break;
        case LR_ROTLRU:
            need[nn++] = in->b; need[nn++] = in->g; need[nn++] = in->mag; need[nn++] = in->theta;
            need[nn++] = gr->db; need[nn++] = gr->dg; need[nn++] = gr->dmag; need[nn++] = gr->dtheta; break;
        case LR_S6:
        case LR_SSD:
            need[nn++] = in->x; need[nn++] = in->delta; need[nn++] = in->A; need[nn++] = in->Bm; need[nn++] = in->Cm;
            need[nn++] = gr->dx; need[nn++] = gr->ddelta; need[nn++] = gr->dA; need[nn++] = gr->dBm; need[nn++] = gr->dCm;
            if (d.flags & LR_HAS_DSKIP) { need[nn++] = in->Dskip; need[nn++] = gr->dDskip; }
            if (d.flags & LR_HAS_Z) { need[nn++] = in->z; need[nn++] = gr->dz; }
            break;
        case LR_GLA:
            need[nn++] = in->q; need[nn++] = in->k; need[nn++] = in->v; need[nn++] = in->g;
            need[nn++] = gr->dq; need[nn++] = gr->dk; need[nn++] = gr->dv; need[nn++] = gr->dg; break;
    }
    for (int i = 0; i < nn; ++i) {
        if (!need[i]) return LR_ERR_INVALID_ARG;
        if (!aligned16(need[i])) return LR_ERR_ALIGNMENT;
    }
    if (!aligned16(dy) || !aligned16(ckpt) || !aligned16(ws)) return LR_ERR_ALIGNMENT;
    if (ws_size < ws_bytes(d, true)) return LR_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    set_launch_stream(st);
    const bool diag = d.kind == LR_RGLRU || d.kind == LR_ROTLRU;
    if (!diag && cudaMemsetAsync(ws, 0, flag_bytes(d, true), st) != cudaSuccess) return LR_ERR_CUDA;
    switch (d.kind) {
        case LR_RGLRU:
        case LR_ROTLRU: return diag_bwd(d, *in, dy, ckpt, *gr, (char*)ws, st);
        case LR_S6: return s6_bwd(d, *in, dy, ckpt, *gr, (char*)ws, st);
        default: return chunk_bwd(d, *in, dy, ckpt, *gr, (char*)ws, st);
    }
}

lr_status lr_step(const lr_desc* desc, const lr_inputs* in, const void* state_in, void* state_out, void* y,
                  void* stream) {
    begin_call();
    if (!desc || !in || !state_out || !y) return LR_ERR_INVALID_ARG;
    const lr_desc& d = *desc;
    if (d.kind < LR_RGLRU || d.kind > LR_GLA) return LR_ERR_INVALID_ARG;
    if (d.io != LR_F32 && d.io != LR_BF16) return LR_ERR_INVALID_ARG;
    if (d.B < 1 || d.L < 1) return LR_ERR_INVALID_ARG;
    if (d.B > (1 << 20) || d.L > (1ll << 30)) return LR_ERR_UNSUPPORTED;
    if ((d.flags & LR_DELTA_SOFTPLUS) && d.kind != LR_S6 && d.kind != LR_SSD) return LR_ERR_INVALID_ARG;
    if ((d.flags & LR_RGLRU_GATES) && d.kind != LR_RGLRU) return LR_ERR_INVALID_ARG;
    const size_t es = (size_t)esize(d.io);
    struct Need {
        const void* p;
        size_t align;
    } need[10];
    int nn = 0;
    switch (d.kind) {
        case LR_RGLRU:
            if (d.disc != LR_DISC_NONE || d.D < 1) return LR_ERR_INVALID_ARG;
            need[nn++] = {in->a, es};
            need[nn++] = {in->b, es};
            need[nn++] = {y, es};
            if (d.flags & LR_RGLRU_GATES) {
                need[nn++] = {in->x, es};
                need[nn++] = {in->A, 4};
            }
            break;
        case LR_ROTLRU:
            if (d.disc != LR_DISC_NONE || d.D < 2 || d.D % 2) return LR_ERR_INVALID_ARG;
            need[nn++] = {in->b, 2 * es};
            need[nn++] = {in->g, es};
            need[nn++] = {in->mag, 4};
            need[nn++] = {in->theta, 4};
            need[nn++] = {y, 2 * es};
            break;
        case LR_S6:
        case LR_SSD:
            if (d.disc < LR_DISC_ZOH || d.disc > LR_DISC_ZOH_EULER) return LR_ERR_INVALID_ARG;
            if (d.kind == LR_S6 && (d.D < 1 || d.N < 1)) return LR_ERR_INVALID_ARG;
            if (d.kind == LR_SSD && (d.H < 1 || d.P < 1 || d.N < 1 || d.G < 1 || d.H % d.G))
                return LR_ERR_INVALID_ARG;
            need[nn++] = {in->x, es};
            need[nn++] = {in->delta, es};
            need[nn++] = {in->A, 4};
            need[nn++] = {in->Bm, es};
            need[nn++] = {in->Cm, es};
            need[nn++] = {y, es};
            if (d.flags & LR_HAS_DSKIP) need[nn++] = {in->Dskip, 4};
            if (d.flags & LR_HAS_Z) need[nn++] = {in->z, es};
            break;
        case LR_GLA:
            if (d.disc != LR_DISC_NONE || d.H < 1 || d.P < 1 || d.N < 1) return LR_ERR_INVALID_ARG;
            need[nn++] = {in->q, es};
            need[nn++] = {in->k, es};
            need[nn++] = {in->v, es};
            need[nn++] = {in->g, es};
            need[nn++] = {y, es};
            break;
    }
    for (int i = 0; i < nn; ++i) {
        if (!need[i].p) return LR_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(need[i].p) % need[i].align) return LR_ERR_ALIGNMENT;
    }
    if ((reinterpret_cast<uintptr_t>(state_in) | reinterpret_cast<uintptr_t>(state_out)) % 4) return LR_ERR_ALIGNMENT;
    if (!step_supported(d)) return LR_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    set_launch_stream(st);
    return step_run(d, *in, static_cast<const float*>(state_in), static_cast<float*>(state_out), y, st);
}

lr_status lr_get_error(void* ws, void* stream, int32_t* info) {
    if (!ws) return LR_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return LR_ERR_CUDA;
    WsHeader h;
    if (cudaMemcpy(&h, ws, 8, cudaMemcpyDeviceToHost) != cudaSuccess) return LR_ERR_CUDA;
    if (cudaMemset(ws, 0, 8) != cudaSuccess) return LR_ERR_CUDA;
    if (info) *info = h.info;
    return (lr_status)h.err;
}

const char* lr_status_string(lr_status s) {
    switch (s) {
        case LR_OK: return "ok";
        case LR_ERR_INVALID_ARG: return "invalid argument";
        case LR_ERR_UNSUPPORTED: return "unsupported by this library";
        case LR_ERR_ALIGNMENT: return "misaligned pointer or innermost extent";
        case LR_ERR_WORKSPACE: return "workspace too small";
        case LR_ERR_CUDA: return "CUDA runtime error";
        case LR_ERR_TIMEOUT: return "device wait timed out";
        case LR_ERR_DEVICE_CHECK: return "device consistency check failed";
    }
    return "unknown status";
}

const char* lr_last_dispatch(void) { return t_dispatch.c_str(); }

int lr_last_launch_count(void) { return t_launches; }

void lr_set_launch_events(void* const* events, int n) {
    t_events = (events && n > 0) ? events : nullptr;
    t_nevents = t_events ? n : 0;
}

}  // extern "C"
