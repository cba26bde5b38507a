// s6.cu -- selective scan S6 (time-varying diagonal A with per-step dt, B, C), forward and
// backward, fused D skip and silu(z) gate, ZOH, bilinear, dirac or ZOH-Euler discretisation
// (sm_100a).
//
// Definition ("lrnnx: A library for Linear RNNs", ai.info summary, Key Contributions 2-3: time-
// varying layers with ZOH / bilinear / dirac discretisation inside a fused scan and output
// projection; the schemes are named there, the formulas below are this library's readings):
//   per (b, d, n):  abar, beta = disc(dt_t[d], A[d,n])
//     ZOH:       abar = exp(dt A),              beta = (exp(dt A) - 1) / A
//     bilinear:  abar = (1 + dt A/2)/(1 - dt A/2), beta = dt / (1 - dt A/2)
//     dirac:     abar = exp(dt A),              beta = 1
//     ZOH-Euler: abar = exp(dt A),              beta = dt
//   h_t[n] = abar h_{t-1}[n] + beta B_t[n] x_t,   y_t = (sum_n C_t[n] h_t[n] + D x_t) silu(z_t).
// Segment checkpoints and recompute follow the mlx-recurrence post (Apple Developer Forums
// thread 840535, segment checkpointing with recomputation during the backward pass).
//
// Work split.  The scan is bound by the per-(t, d, n) arithmetic (one exp or reciprocal and a
// handful of FMAs per state per step), not by HBM, so the states stay in registers and the
// recurrence never crosses threads: a CTA owns one batch row and 64 channels for the whole
// sequence; kTPC = 4 threads per channel (lanes q, q + 8, q + 16, q + 24 of a warp) hold 4 of its
// 16 states each, so the readout sum over n is two shuffles.  Four threads per channel (rather
// than two) halve the registers a thread needs, so twice the warps fit on an SM; the per-(t, d)
// work that every thread of a channel would repeat -- the silu(z) gate and the softplus step
// length -- is instead split over the four lanes (lane p takes the steps t = p mod 4) and shared
// by shuffles or shared memory.  Steps run in batches of kSub = 8: the exponentials and input
// terms of a batch do not depend on the state, so they are formed first (32 independent
// exponentials per thread), then the 8 dependent state updates.
// Segments of S <= 64 steps are staged in shared memory by TMA (x, dt, z, dy as [S][64] bf16
// tiles, B, C as [S][16]); outputs are written back into the consumed tile slots and stored with
// TMA.  The forward pass double-buffers segments and writes the state entering each segment to the
// checkpoint buffer.
//
// Backward, per segment in reverse order (the adjoint carry G stays in registers across
// segments): the gate terms ds = dy silu(z) and dz / s are formed for the whole tile first; (A)
// from the checkpoint, run the segment forward and keep the state at every 8-step sub-block
// boundary in shared memory; (C) for each sub-block in reverse, recompute its 8 steps keeping h_t
// and abar_t in registers, then run the adjoint recurrence
// G_t[n] = ds_t C_t[n] + abar_{t+1} G_{t+1}[n] backwards through them and form every gradient.
// dB_t[n] and dC_t[n] (sums over channels) are reduced over the 8 channels of a warp with a
// butterfly, then over the CTA's warps in a fixed order once per sub-block, giving one partial per
// 64-channel block; dA and dD partials are per batch row.  A small kernel sums the partials in a
// fixed order (deterministic results).
#include "common.cuh"
#include "host_common.h"

namespace lrs {
namespace {

constexpr int kDB = 64;                // channels per CTA
constexpr int kN = 16;                 // states per channel
constexpr int kTPC = 4;                // threads per channel
constexpr int kNH = kN / kTPC;         // states per thread (4)
constexpr int kCPW = 32 / kTPC;        // channels per warp (8)
constexpr int kThreads = kDB * kTPC;   // 256
constexpr int kWarps = kThreads / 32;  // 8
constexpr int kMaxS = 64;              // segment rows per TMA box
constexpr int kSub = 8;                // step batch (forward) and backward sub-block length
static_assert(2 * kNH == kCPW, "the dB / dC reduce-scatter over a warp's channels leaves one value per lane");
static_assert(kSub == 2 * kTPC, "each lane of a channel takes two steps of a batch for the per-(t, d) work");
static_assert(kSub * 32 == kThreads, "the cross-warp dB / dC reduction gives one (step, lane) pair per thread");
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sigm(float z) { return rcp(1.0f + ex2(-z * kLog2e)); }
__device__ __forceinline__ float bf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// kNH consecutive f32 (this thread's states of a B or C row; one 16-byte access)
__device__ __forceinline__ void ldn(const float* p, float* out) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x;
    out[1] = v.y;
    out[2] = v.z;
    out[3] = v.w;
}
// sum over the kTPC threads of a channel (lanes l, l + kCPW, l + 2 kCPW, ...)
__device__ __forceinline__ float chan_sum(float x) {
#pragma unroll
    for (int o = kCPW; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

struct S6Args {
    int B, L, D, S, nseg, ncb;
    int disc;            // LR_DISC_ZOH / _BILINEAR / _DIRAC / _ZOH_EULER
    int has_z, has_d;
    const float* A;      // [D, N]
    const float* Dskip;  // [D]
    float* ckpt;         // [nseg, B, D, N] (full state: [L, B, D, N])
    WsHeader* hdr;
    float* pdB;          // [ncb, B, L, N]
    float* pdC;          // [ncb, B, L, N]
    float* pdA;          // [B, D, N]
    float* pdD;          // [B, D]
    int softplus;        // LR_DELTA_SOFTPLUS: dt = softplus(delta + bias)
    const float* dbias;  // [D] or null (bias 0)
    float* pdE;          // [B, D] partials of d bias
};

__device__ __forceinline__ float softplus_f(float v) { return v > 20.0f ? v : log1pf(expf(v)); }

// x and dt of the steps t0 .. t0 + kSub - 1 of a tile for channel column `dl` (x = 0 and dt = 0
// beyond `nb` steps: such a step leaves the state unchanged and is never read back).  With the
// softplus front-end (SP) lane part p forms dt of steps p and p + kTPC and the lanes of a channel
// exchange them, instead of all four forming all eight.
template <bool SP>
__device__ __forceinline__ void load_steps(const __nv_bfloat16* X, const __nv_bfloat16* DT, int t0, int nb, int dl,
                                           int part, int q, float bias, float* xs, float* dts) {
#pragma unroll
    for (int i = 0; i < kSub; ++i) xs[i] = i < nb ? bf(X + (t0 + i) * kDB + dl) : 0.0f;
    if constexpr (!SP) {
#pragma unroll
        for (int i = 0; i < kSub; ++i) dts[i] = i < nb ? bf(DT + (t0 + i) * kDB + dl) : 0.0f;
    } else {
        float mine[kSub / kTPC];
#pragma unroll
        for (int r = 0; r < kSub / kTPC; ++r) {
            const int i = part + kTPC * r;
            mine[r] = i < nb ? softplus_f(bf(DT + (t0 + i) * kDB + dl) + bias) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kSub; ++i) dts[i] = __shfl_sync(0xffffffffu, mine[i / kTPC], q + kCPW * (i % kTPC));
    }
}

// Per-thread constants of the discretisation for its kNH states.  The per-step scale of dt
// (log2(e) for the exponential forms, 1/2 for bilinear) is applied once per step, not per state.
struct Disc {
    float A[kNH];
    float ia[kNH];  // ZOH: 1 / A
};

template <int DISC>
__device__ __forceinline__ float dt_scale(float dt) {
    return DISC == LR_DISC_BILINEAR ? 0.5f * dt : dt * kLog2e;
}

// abar and beta of one state; dsc = dt_scale(dt)
template <int DISC>
__device__ __forceinline__ void coef(const Disc& c, int j, float dt, float dsc, float& ab, float& be) {
    if (DISC == LR_DISC_BILINEAR) {
        float r = rcp(fmaf(-dsc, c.A[j], 1.0f));
        ab = fmaf(dsc * c.A[j], r, r);  // (1 + dt A/2) r
        be = dt * r;
    } else {
        ab = ex2(dsc * c.A[j]);
        be = DISC == LR_DISC_ZOH ? fmaf(ab, c.ia[j], -c.ia[j]) : (DISC == LR_DISC_DIRAC ? 1.0f : dt);
    }
}

// beta from abar (cheaper than a second transcendental in the backward sweep)
template <int DISC>
__device__ __forceinline__ float beta_of(const Disc& c, int j, float dt, float ab) {
    if (DISC == LR_DISC_ZOH) return fmaf(ab, c.ia[j], -c.ia[j]);
    if (DISC == LR_DISC_DIRAC) return 1.0f;
    if (DISC == LR_DISC_ZOH_EULER) return dt;
    return dt * 0.5f * (ab + 1.0f);  // bilinear: dt / (1 - dt A/2) = dt (abar + 1) / 2
}

// abar and beta B x of the kSub steps of a batch (state-independent: formed before the updates);
// Bf: the tile's B rows as f32 ([S][16])
template <int DISC>
__device__ __forceinline__ void batch_coefs(const Disc& c, const float* Bf, int t0, int part,
                                            const float* xs, const float* dts, float (&ab)[kSub][kNH],
                                            float (&bx)[kSub][kNH]) {
#pragma unroll
    for (int i = 0; i < kSub; ++i) {
        const float4 B4 = *reinterpret_cast<const float4*>(Bf + (t0 + i) * kN + part * kNH);
        const float Bv[kNH] = {B4.x, B4.y, B4.z, B4.w};
        const float dsc = dt_scale<DISC>(dts[i]);
#pragma unroll
        for (int j = 0; j < kNH; ++j) {
            float be;
            coef<DISC>(c, j, dts[i], dsc, ab[i][j], be);
            bx[i][j] = be * (Bv[j] * xs[i]);
        }
    }
}

// The B and C rows of a tile ([S][16] bf16, as TMA lands them) as f32, by all threads.
__device__ __forceinline__ void widen_bc(const __nv_bfloat16* Bs, const __nv_bfloat16* Cs, float* Bf, float* Cf,
                                         int nt, int tid) {
    for (int e = tid; e < nt * kN / 2; e += kThreads) {
        const float2 b2 = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Bs)[e]);
        const float2 c2 = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Cs)[e]);
        reinterpret_cast<float2*>(Bf)[e] = b2;
        reinterpret_cast<float2*>(Cf)[e] = c2;
    }
}

template <int DISC>
__device__ __forceinline__ void load_disc(Disc& c, const float* A, int d, bool dok, int part) {
#pragma unroll
    for (int j = 0; j < kNH; ++j) {
        float Av = dok ? A[(size_t)d * kN + part * kNH + j] : -1.0f;
        c.A[j] = Av;
        c.ia[j] = DISC == LR_DISC_ZOH ? 1.0f / Av : 0.0f;
    }
}

__device__ __forceinline__ char* smem_base() {
    extern __shared__ char dyn_smem[];
    uintptr_t p = reinterpret_cast<uintptr_t>(dyn_smem);
    return reinterpret_cast<char*>((p + 127) & ~uintptr_t(127));
}

constexpr size_t kTileDT = size_t(kMaxS) * kDB * 2;  // [S][64] bf16
constexpr size_t kTileBC = size_t(kMaxS) * kN * 2;   // [S][16] bf16
constexpr size_t kTileF = size_t(kMaxS) * kDB * 4;   // [S][64] f32

// ----------------------------------------------------------------------------------- forward
// Shared memory per stage: X, DT, Z tiles and B, C tiles.
constexpr size_t kTileBCf = size_t(kMaxS) * kN * 4;  // [S][16] f32
constexpr size_t kFwdStage = 3 * kTileDT + 2 * kTileBC;
constexpr size_t kFwdSmem = 128 + 2 * kFwdStage + 2 * kTileBCf + 128;

template <int DISC, bool FULL, bool SP>
__global__ void __launch_bounds__(kThreads, 2)
s6_fwd_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mDT,
              const __grid_constant__ CUtensorMap mZ, const __grid_constant__ CUtensorMap mB,
              const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mY, S6Args a) {
    char* sm = smem_base();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);  // bar[0], bar[1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int part = lane / kCPW, q = lane % kCPW, dl = warp * kCPW + q;
    const int b = blockIdx.x / a.ncb, cb = blockIdx.x % a.ncb;
    const int d = cb * kDB + dl;
    const bool dok = d < a.D;
    auto stage = [&](int s, int which) -> char* { return sm + 128 + s * kFwdStage + which * kTileDT; };
    auto stageBC = [&](int s, int which) -> __nv_bfloat16* {
        return reinterpret_cast<__nv_bfloat16*>(sm + 128 + s * kFwdStage + 3 * kTileDT + which * kTileBC);
    };
    const uint32_t bytes = (uint32_t)(a.S * kDB * 2 * (a.has_z ? 3 : 2) + 2 * a.S * kN * 2);
    auto issue = [&](int k, int s) {
        mbar_arrive_expect_tx(&bar[s], bytes);
        const int t0 = k * a.S;
        tma_load_3d(stage(s, 0), &mX, &bar[s], cb * kDB, t0, b);
        tma_load_3d(stage(s, 1), &mDT, &bar[s], cb * kDB, t0, b);
        if (a.has_z) tma_load_3d(stage(s, 2), &mZ, &bar[s], cb * kDB, t0, b);
        tma_load_3d(stageBC(s, 0), &mB, &bar[s], 0, t0, b);
        tma_load_3d(stageBC(s, 1), &mC, &bar[s], 0, t0, b);
    };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        issue(0, 0);
    }
    Disc c;
    load_disc<DISC>(c, a.A, d, dok, part);
    const float Dd = (a.has_d && dok) ? a.Dskip[d] : 0.0f;
    const float dbias = (SP && a.dbias && dok) ? a.dbias[d] : 0.0f;
    float* Bf = reinterpret_cast<float*>(sm + 128 + 2 * kFwdStage);  // the stage's B, C rows as f32
    float* Cf = Bf + kMaxS * kN;
    float h[kNH];
#pragma unroll
    for (int j = 0; j < kNH; ++j) h[j] = 0.0f;
    __syncthreads();

    bool ok = true;
    for (int k = 0; k < a.nseg; ++k) {
        const int s = k & 1;
        if (tid == 0 && k + 1 < a.nseg) {
            if (k >= 1) bulk_wait_read_all();  // store of segment k-1 has read stage s^1
            issue(k + 1, s ^ 1);
        }
        ok = ok && mbar_wait(&bar[s], (k >> 1) & 1, a.hdr, 300);
        if (dok && !FULL)
            *reinterpret_cast<float4*>(a.ckpt + (((size_t)k * a.B + b) * a.D + d) * kN + part * kNH) =
                make_float4(h[0], h[1], h[2], h[3]);
        const int nt = min(a.S, a.L - k * a.S);
        __nv_bfloat16* X = reinterpret_cast<__nv_bfloat16*>(stage(s, 0));
        const __nv_bfloat16* DT = reinterpret_cast<const __nv_bfloat16*>(stage(s, 1));
        const __nv_bfloat16* Z = reinterpret_cast<const __nv_bfloat16*>(stage(s, 2));
        widen_bc(stageBC(s, 0), stageBC(s, 1), Bf, Cf, nt, tid);
        __syncthreads();
        for (int t0 = 0; ok && t0 < nt; t0 += kSub) {
            const int nb = min(kSub, nt - t0);
            float xs[kSub], dts[kSub], ab[kSub][kNH], bx[kSub][kNH];
            load_steps<SP>(X, DT, t0, nb, dl, part, q, dbias, xs, dts);
            batch_coefs<DISC>(c, Bf, t0, part, xs, dts, ab, bx);
            float sv[kSub];
#pragma unroll
            for (int i = 0; i < kSub; ++i) {
                float Cv[kNH];
                ldn(Cf + (t0 + i) * kN + part * kNH, Cv);
                if (FULL && dok && i < nb)  // the state entering step k S + t0 + i
                    *reinterpret_cast<float4*>(
                        a.ckpt + ((((size_t)k * a.S + t0 + i) * a.B + b) * a.D + d) * kN + part * kNH) =
                        make_float4(h[0], h[1], h[2], h[3]);
                float acc = 0.0f;
#pragma unroll
                for (int j = 0; j < kNH; ++j) {
                    h[j] = fmaf(ab[i][j], h[j], bx[i][j]);
                    acc = fmaf(Cv[j], h[j], acc);
                }
                sv[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < kSub; ++i) sv[i] = chan_sum(sv[i]);
            // lane part p writes the outputs of steps p and p + kTPC (the gate formed once per (t, d))
#pragma unroll
            for (int r = 0; r < kSub / kTPC; ++r) {
                const int i = part + kTPC * r;
                float yv = 0.0f, xi = 0.0f, si = 0.0f;
#pragma unroll
                for (int u = 0; u < kSub; ++u)  // register select (i is lane-dependent)
                    if (u % kTPC == part % kTPC && u / kTPC == r) { xi = xs[u]; si = sv[u]; }
                if (i < nb) {
                    yv = fmaf(Dd, xi, si);
                    if (a.has_z) {
                        const float zv = bf(Z + (t0 + i) * kDB + dl);
                        yv *= zv * sigm(zv);
                    }
                    X[(t0 + i) * kDB + dl] = __float2bfloat16_rn(yv);
                }
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0 && ok) {
            tma_store_3d(&mY, X, cb * kDB, k * a.S, b);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_read_all();
}

// ---------------------------------------------------------------------------------- backward
// Shared memory: X, DT, Z, DY tiles, B, C tiles (bf16 as TMA lands them, and f32), ds = dy silu(z)
// (f32), sub-block boundary states, per-warp dB / dC of one sub-block.  After the tile's gate
// terms are formed, the Z slot holds dz / s = dy sigma(z) (1 + z (1 - sigma(z))) in bf16 and then
// dz itself.
constexpr size_t kOffX = 128;
constexpr size_t kOffB = kOffX + 4 * kTileDT;
constexpr size_t kOffBf = kOffB + 2 * kTileBC;
constexpr size_t kOffDS = kOffBf + 2 * kTileBCf;
constexpr size_t kOffBnd = kOffDS + kTileF;
constexpr size_t kBndBytes = size_t(kMaxS / kSub) * kThreads * kNH * 4;
constexpr size_t kOffRed = kOffBnd + kBndBytes;
constexpr size_t kRedBytes = size_t(kWarps) * kSub * 32 * 4;  // per-warp dB / dC of one sub-block
constexpr size_t kBwdSmem = kOffRed + kRedBytes + 128;

template <int DISC, bool FULL, bool SP>
__global__ void __launch_bounds__(kThreads, 2)
s6_bwd_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mDT,
              const __grid_constant__ CUtensorMap mZ, const __grid_constant__ CUtensorMap mDY,
              const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mC,
              const __grid_constant__ CUtensorMap mdX, const __grid_constant__ CUtensorMap mdDT,
              const __grid_constant__ CUtensorMap mdZ, S6Args a) {
    char* sm = smem_base();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
    __nv_bfloat16* X = reinterpret_cast<__nv_bfloat16*>(sm + kOffX);
    __nv_bfloat16* DT = reinterpret_cast<__nv_bfloat16*>(sm + kOffX + kTileDT);
    __nv_bfloat16* Z = reinterpret_cast<__nv_bfloat16*>(sm + kOffX + 2 * kTileDT);
    __nv_bfloat16* DY = reinterpret_cast<__nv_bfloat16*>(sm + kOffX + 3 * kTileDT);
    const __nv_bfloat16* Bs = reinterpret_cast<const __nv_bfloat16*>(sm + kOffB);
    const __nv_bfloat16* Cs = reinterpret_cast<const __nv_bfloat16*>(sm + kOffB + kTileBC);
    float* Bf = reinterpret_cast<float*>(sm + kOffBf);    // [S][16] B as f32
    float* Cf = Bf + kMaxS * kN;                           // [S][16] C as f32
    float* DS = reinterpret_cast<float*>(sm + kOffDS);    // [S][64] ds = dy silu(z)
    float* bnd = reinterpret_cast<float*>(sm + kOffBnd);  // [sub-block][thread][kNH]
    float* red = reinterpret_cast<float*>(sm + kOffRed);  // [warp][step of the sub-block][lane]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int part = lane / kCPW, q = lane % kCPW, dl = warp * kCPW + q;
    const int b = blockIdx.x / a.ncb, cb = blockIdx.x % a.ncb;
    const int d = cb * kDB + dl;
    const bool dok = d < a.D;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    Disc c;
    load_disc<DISC>(c, a.A, d, dok, part);
    const float Dd = (a.has_d && dok) ? a.Dskip[d] : 0.0f;
    const float dbias = (SP && a.dbias && dok) ? a.dbias[d] : 0.0f;
    float G[kNH], anext[kNH], dA[kNH];
#pragma unroll
    for (int j = 0; j < kNH; ++j) G[j] = anext[j] = dA[j] = 0.0f;
    float dD = 0.0f, dE = 0.0f;
    const uint32_t bytes = (uint32_t)(a.S * kDB * 2 * (a.has_z ? 4 : 3) + 2 * a.S * kN * 2);
    __syncthreads();

    bool ok = true;
    int phase = 0;
    for (int k = a.nseg - 1; k >= 0; --k, phase ^= 1) {
        const int t0 = k * a.S;
        const int nt = min(a.S, a.L - t0);
        if (tid == 0) {
            bulk_wait_read_all();  // previous segment's gradient tiles have left shared memory
            mbar_arrive_expect_tx(&bar[0], bytes);
            tma_load_3d(X, &mX, &bar[0], cb * kDB, t0, b);
            tma_load_3d(DT, &mDT, &bar[0], cb * kDB, t0, b);
            if (a.has_z) tma_load_3d(Z, &mZ, &bar[0], cb * kDB, t0, b);
            tma_load_3d(DY, &mDY, &bar[0], cb * kDB, t0, b);
            tma_load_3d(const_cast<__nv_bfloat16*>(Bs), &mB, &bar[0], 0, t0, b);
            tma_load_3d(const_cast<__nv_bfloat16*>(Cs), &mC, &bar[0], 0, t0, b);
        }
        float h[kNH];
        if (!FULL && dok) {
            const float4 v = *reinterpret_cast<const float4*>(a.ckpt + (((size_t)k * a.B + b) * a.D + d) * kN + part * kNH);
            h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
        } else {
#pragma unroll
            for (int j = 0; j < kNH; ++j) h[j] = 0.0f;
        }
        ok = ok && mbar_wait(&bar[0], phase, a.hdr, 400);
        // gate terms of the tile, once per (t, d); B and C rows as f32
        for (int e = tid; e < nt * kDB; e += kThreads) {
            const float dyv = bf(DY + e);
            if (a.has_z) {
                const float zv = bf(Z + e);
                const float sg = sigm(zv);
                DS[e] = dyv * zv * sg;
                Z[e] = __float2bfloat16_rn(dyv * sg * fmaf(zv, 1.0f - sg, 1.0f));
            } else {
                DS[e] = dyv;
            }
        }
        widen_bc(Bs, Cs, Bf, Cf, nt, tid);
        __syncthreads();
        const int nsb = (nt + kSub - 1) / kSub;
        // (A) segment forward, keeping sub-block boundary states (not with the full state)
        for (int sb = 0; sb < (FULL ? 0 : nsb); ++sb) {
            *reinterpret_cast<float4*>(bnd + ((size_t)sb * kThreads + tid) * kNH) = make_float4(h[0], h[1], h[2], h[3]);
            if (sb + 1 == nsb) break;  // the last sub-block's end state is not needed
            float xs[kSub], dts[kSub], ab[kSub][kNH], bx[kSub][kNH];
            load_steps<SP>(X, DT, sb * kSub, kSub, dl, part, q, dbias, xs, dts);
            batch_coefs<DISC>(c, Bf, sb * kSub, part, xs, dts, ab, bx);
#pragma unroll
            for (int i = 0; i < kSub; ++i)
#pragma unroll
                for (int j = 0; j < kNH; ++j) h[j] = fmaf(ab[i][j], h[j], bx[i][j]);
        }
        // (C) sub-blocks in reverse: recompute into registers, then the adjoint sweep
        for (int sb = nsb - 1; sb >= 0; --sb) {
            const int tb = sb * kSub;
            const int n = min(kSub, nt - tb);
            // x and dt of the sub-block: kept in registers only with the softplus front-end
            // (its dt is formed, not loaded); otherwise the sweep re-reads them from the tile
            // (step t's row is overwritten with its gradients only after its last use)
            float xs_sp[SP ? kSub : 1], dts_sp[SP ? kSub : 1];
            float h0[kNH], hr[kSub][kNH], ar[kSub][kNH];
            {
                float xs[kSub], dts[kSub];
                load_steps<SP>(X, DT, tb, n, dl, part, q, dbias, xs, dts);
                if constexpr (SP) {
#pragma unroll
                    for (int i = 0; i < kSub; ++i) {
                        xs_sp[i] = xs[i];
                        dts_sp[i] = dts[i];
                    }
                }
                float bx[kSub][kNH];
                batch_coefs<DISC>(c, Bf, tb, part, xs, dts, ar, bx);
                if constexpr (!FULL) {
                    const float4 v = *reinterpret_cast<const float4*>(bnd + ((size_t)sb * kThreads + tid) * kNH);
                    h0[0] = v.x; h0[1] = v.y; h0[2] = v.z; h0[3] = v.w;
#pragma unroll
                    for (int i = 0; i < kSub; ++i)
#pragma unroll
                        for (int j = 0; j < kNH; ++j)
                            hr[i][j] = fmaf(ar[i][j], i > 0 ? hr[i > 0 ? i - 1 : 0][j] : h0[j], bx[i][j]);
                } else {  // the full state: the state entering every step of the sub-block is stored
                    float hs[kSub][kNH];
#pragma unroll
                    for (int i = 0; i < kSub; ++i) {
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (i < n && dok)
                            v = *reinterpret_cast<const float4*>(
                                a.ckpt + ((((size_t)t0 + tb + i) * a.B + b) * a.D + d) * kN + part * kNH);
                        hs[i][0] = v.x; hs[i][1] = v.y; hs[i][2] = v.z; hs[i][3] = v.w;
                    }
#pragma unroll
                    for (int j = 0; j < kNH; ++j) h0[j] = hs[0][j];
#pragma unroll
                    for (int i = 0; i < kSub; ++i)
#pragma unroll
                        for (int j = 0; j < kNH; ++j) hr[i][j] = fmaf(ar[i][j], hs[i][j], bx[i][j]);
                    // the sweep reads the state entering step i > 0 as hr[i - 1], which equals the
                    // stored one up to the rounding of the same operations
                }
            }
#pragma unroll
            for (int i = kSub - 1; i >= 0; --i) {
                if (i < n) {
                    const int t = tb + i;
                    float xv, dt;
                    if constexpr (SP) {
                        xv = xs_sp[i];
                        dt = dts_sp[i];
                    } else {
                        xv = bf(X + t * kDB + dl);
                        dt = bf(DT + t * kDB + dl);
                    }
                    const float ds = DS[t * kDB + dl];
                    float Bv[kNH], Cv[kNH];
                    ldn(Bf + t * kN + part * kNH, Bv);
                    ldn(Cf + t * kN + part * kNH, Cv);
                    float s = 0.0f;
                    if (a.has_z) {  // the readout s is needed only for dz = s (dz / s)
                        float sacc = 0.0f;
#pragma unroll
                        for (int j = 0; j < kNH; ++j) sacc = fmaf(Cv[j], hr[i][j], sacc);
                        s = fmaf(Dd, xv, chan_sum(sacc));
                    }
                    float v[2 * kNH];  // dB (x n), dC (x n) contributions of this channel
                    float dxa = 0.0f, dta = 0.0f;
                    const float hdt = 0.5f * dt;
#pragma unroll
                    for (int j = 0; j < kNH; ++j) {
                        const float ab = ar[i][j];
                        const float hp = i > 0 ? hr[i > 0 ? i - 1 : 0][j] : h0[j];
                        G[j] = fmaf(anext[j], G[j], ds * Cv[j]);
                        v[kNH + j] = ds * hr[i][j];
                        const float xB = xv * Bv[j];
                        if (DISC == LR_DISC_DIRAC) {  // beta = 1
                            v[j] = G[j] * xv;
                            dxa = fmaf(G[j], Bv[j], dxa);
                            const float r = ab * (G[j] * hp);
                            dta = fmaf(r, c.A[j], dta);
                            dA[j] = fmaf(r, dt, dA[j]);
                        } else if (DISC == LR_DISC_ZOH_EULER) {  // beta = dt
                            const float Gb = G[j] * dt;
                            v[j] = Gb * xv;
                            dxa = fmaf(Gb, Bv[j], dxa);
                            const float r = ab * (G[j] * hp);
                            dta = fmaf(r, c.A[j], fmaf(G[j], xB, dta));  // + d loss / d beta
                            dA[j] = fmaf(r, dt, dA[j]);
                        } else if (DISC == LR_DISC_ZOH) {
                            // with dab = G h_{t-1} (d loss / d abar) and w = G B x (d loss / d beta):
                            // d dt = abar (dab A + w) = abar G (h_{t-1} A + B x);
                            // d A = (dt abar G (h_{t-1} A + B x) - w beta) / A, w beta = (G beta x) B;
                            // the 1 / A is applied once, to the sum, at the end
                            const float be = beta_of<DISC>(c, j, dt, ab);
                            const float Gb = G[j] * be;
                            v[j] = Gb * xv;
                            dxa = fmaf(Gb, Bv[j], dxa);
                            const float r = ab * (G[j] * fmaf(hp, c.A[j], xB));
                            dta += r;
                            dA[j] = fmaf(-v[j], Bv[j], fmaf(dt, r, dA[j]));
                        } else {  // bilinear, rr = 1 / (1 - dt A / 2) = (abar + 1) / 2
                            // d dt = rr^2 A (dab + w dt / 2) + w rr;  d A = rr^2 dt (dab + w dt / 2)
                            const float rr = 0.5f * (ab + 1.0f);
                            const float Gb = G[j] * (dt * rr);
                            v[j] = Gb * xv;
                            dxa = fmaf(Gb, Bv[j], dxa);
                            const float rm = (rr * rr) * (G[j] * fmaf(xB, hdt, hp));
                            dta = fmaf(rm, c.A[j], fmaf(G[j] * xB, rr, dta));
                            dA[j] = fmaf(rm, dt, dA[j]);
                        }
                        anext[j] = ab;
                    }
                    dxa = chan_sum(dxa);
                    dta = chan_sum(dta);
                    // dB / dC: sum over the kCPW channels of the warp that hold the same states
                    // (butterfly over lanes differing in the channel bits; lane q ends with the
                    // sum of value q)
#pragma unroll
                    for (int m = kCPW / 2; m >= 1; m >>= 1) {
#pragma unroll
                        for (int i2 = 0; i2 < m; ++i2) {
                            const bool up = (q & m) != 0;
                            const float send = up ? v[i2] : v[i2 + m];
                            const float keep = up ? v[i2 + m] : v[i2];
                            v[i2] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                        }
                    }
                    red[(warp * kSub + i) * 32 + lane] = v[0];
                    if (part == 0) {
                        // softplus: d delta = d dt sigma(delta + bias), and sigma(delta + bias) =
                        // 1 - e^{-dt}
                        const float ddr = SP ? dta * -expm1f(-dt) : dta;
                        dE += ddr;
                        X[t * kDB + dl] = __float2bfloat16_rn(fmaf(ds, Dd, dxa));
                        DT[t * kDB + dl] = __float2bfloat16_rn(ddr);
                        if (a.has_z) Z[t * kDB + dl] = __float2bfloat16_rn(s * bf(Z + t * kDB + dl));
                        dD = fmaf(ds, xv, dD);
                    }
                }
            }
            // this sub-block's dB / dC partial of the CTA: fixed-order sum over the warps, one
            // (step, lane) pair per thread
            __syncthreads();
            {
                const int i = tid >> 5, ln = tid & 31;
                if (i < n) {
                    float sum = 0.0f;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) sum += red[(w * kSub + i) * 32 + ln];
                    const int p = ln / kCPW, qq = ln % kCPW;
                    float* dst = (qq < kNH ? a.pdB : a.pdC) +
                                 (((size_t)cb * a.B + b) * a.L + t0 + tb + i) * kN + p * kNH + (qq % kNH);
                    *dst = sum;
                }
            }
            __syncthreads();
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0 && ok) {
            tma_store_3d(&mdX, X, cb * kDB, t0, b);
            tma_store_3d(&mdDT, DT, cb * kDB, t0, b);
            if (a.has_z) tma_store_3d(&mdZ, Z, cb * kDB, t0, b);
            bulk_commit();
        }
        __syncthreads();
    }
    if (dok) {
        float4 o;
        if (DISC == LR_DISC_ZOH)
            o = make_float4(dA[0] * c.ia[0], dA[1] * c.ia[1], dA[2] * c.ia[2], dA[3] * c.ia[3]);
        else
            o = make_float4(dA[0], dA[1], dA[2], dA[3]);
        *reinterpret_cast<float4*>(a.pdA + ((size_t)b * a.D + d) * kN + part * kNH) = o;
        if (part == 0) a.pdD[(size_t)b * a.D + d] = dD;
        if (part == 0 && SP) a.pdE[(size_t)b * a.D + d] = dE;
    }
    if (tid == 0) bulk_wait_read_all();
}

// Fixed-order sums of the partials: dB, dC over channel blocks; dA, dD over batch rows.
__global__ void s6_reduce_kernel(S6Args a, float* __restrict__ dBm, float* __restrict__ dCm,
                                 float* __restrict__ dAo, float* __restrict__ dDo, float* __restrict__ dEo) {
    const size_t nBC = (size_t)a.B * a.L * kN;
    const size_t nA = (size_t)a.D * kN;
    const size_t n = nBC + nA + a.D + (dEo ? a.D : 0);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        if (i < nBC) {
            float sb = 0.0f, sc = 0.0f;
            for (int cb = 0; cb < a.ncb; ++cb) {
                sb += a.pdB[(size_t)cb * nBC + i];
                sc += a.pdC[(size_t)cb * nBC + i];
            }
            dBm[i] = sb;
            dCm[i] = sc;
        } else if (i < nBC + nA) {
            const size_t j = i - nBC;
            float s = 0.0f;
            for (int bb = 0; bb < a.B; ++bb) s += a.pdA[(size_t)bb * nA + j];
            dAo[j] = s;
        } else if (i < nBC + nA + a.D) {
            if (dDo) {
                const size_t j = i - nBC - nA;
                float s = 0.0f;
                for (int bb = 0; bb < a.B; ++bb) s += a.pdD[(size_t)bb * a.D + j];
                dDo[j] = s;
            }
        } else {  // d bias of the softplus front-end
            const size_t j = i - nBC - nA - a.D;
            float s = 0.0f;
            for (int bb = 0; bb < a.B; ++bb) s += a.pdE[(size_t)bb * a.D + j];
            dEo[j] = s;
        }
    }
}

// ------------------------------------------------------------------------------ host side
struct S6Ws {
    size_t pdB, pdC, pdA, pdD, pdE, end;
};

S6Ws ws_plan(const lr_desc& d) {
    const size_t ncb = (d.D + kDB - 1) / kDB;
    WsCursor c;
    S6Ws w;
    w.pdB = c.take(sizeof(float) * ncb * d.B * d.L * kN);
    w.pdC = c.take(sizeof(float) * ncb * d.B * d.L * kN);
    w.pdA = c.take(sizeof(float) * d.B * d.D * kN);
    w.pdD = c.take(sizeof(float) * d.B * d.D);
    w.pdE = c.take(sizeof(float) * d.B * d.D);
    w.end = c.off;
    return w;
}

S6Args make_args(const lr_desc& d, const lr_inputs& in, void* ckpt, char* ws, bool bwd) {
    S6Args a{};
    a.B = (int)d.B;
    a.L = (int)d.L;
    a.D = (int)d.D;
    a.S = d.segment;
    a.nseg = (int)((d.L + d.segment - 1) / d.segment);
    a.ncb = (int)((d.D + kDB - 1) / kDB);
    a.disc = d.disc;
    a.has_z = (d.flags & LR_HAS_Z) ? 1 : 0;
    a.has_d = (d.flags & LR_HAS_DSKIP) ? 1 : 0;
    a.softplus = (d.flags & LR_DELTA_SOFTPLUS) ? 1 : 0;
    a.dbias = a.softplus ? in.delta_bias : nullptr;
    a.A = in.A;
    a.Dskip = in.Dskip;
    a.ckpt = (float*)ckpt;
    a.hdr = (WsHeader*)ws;
    if (bwd) {
        S6Ws w = ws_plan(d);
        a.pdB = (float*)(ws + w.pdB);
        a.pdC = (float*)(ws + w.pdC);
        a.pdA = (float*)(ws + w.pdA);
        a.pdD = (float*)(ws + w.pdD);
        a.pdE = (float*)(ws + w.pdE);
    }
    return a;
}

template <typename F>
void set_smem(F fn, size_t bytes) {
    cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DISC>
auto fwd_variant(bool full, bool sp) {
    return full ? (sp ? s6_fwd_kernel<DISC, true, true> : s6_fwd_kernel<DISC, true, false>)
                : (sp ? s6_fwd_kernel<DISC, false, true> : s6_fwd_kernel<DISC, false, false>);
}
template <int DISC>
auto bwd_variant(bool full, bool sp) {
    return full ? (sp ? s6_bwd_kernel<DISC, true, true> : s6_bwd_kernel<DISC, true, false>)
                : (sp ? s6_bwd_kernel<DISC, false, true> : s6_bwd_kernel<DISC, false, false>);
}

}  // namespace

bool s6_supported(const lr_desc& d) {
    return d.io == LR_BF16 && d.N == kN && d.segment <= kMaxS && d.segment % kSub == 0 &&
           d.D <= (1 << 24) && d.L <= (1 << 30);
}

size_t s6_ws_bytes(const lr_desc& d, bool bwd) { return bwd ? ws_plan(d).end : 256; }
size_t s6_flag_bytes(const lr_desc&, bool) { return 256; }

lr_status s6_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                 cudaStream_t st) {
    S6Args a = make_args(d, in, ckpt, ws, false);
    CUtensorMap mX, mDT, mZ, mB, mC, mY;
    const uint32_t S = (uint32_t)d.segment;
    bool ok = make_tmap_3d(&mX, in.x, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mDT, in.delta, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mZ, a.has_z ? in.z : in.x, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mB, in.Bm, 2, kN, d.L, d.B, kN, S) &&
              make_tmap_3d(&mC, in.Cm, 2, kN, d.L, d.B, kN, S) &&
              make_tmap_3d(&mY, y, 2, d.D, d.L, d.B, kDB, S);
    if (!ok) return LR_ERR_INVALID_ARG;
    const int grid = a.B * a.ncb;
    auto run = [&](auto kernel, const char* name) {
        set_smem(kernel, kFwdSmem);
        note_launch(name);
        kernel<<<grid, kThreads, kFwdSmem, st>>>(mX, mDT, mZ, mB, mC, mY, a);
    };
    // compile-time variants: LR_FULL_STATE (every step's state checkpointed) and LR_DELTA_SOFTPLUS
    const bool full = (d.flags & LR_FULL_STATE) != 0, sp = a.softplus != 0;
    switch (d.disc) {
        case LR_DISC_ZOH: run(fwd_variant<LR_DISC_ZOH>(full, sp), "s6_fwd_zoh"); break;
        case LR_DISC_BILINEAR: run(fwd_variant<LR_DISC_BILINEAR>(full, sp), "s6_fwd_bilinear"); break;
        case LR_DISC_DIRAC: run(fwd_variant<LR_DISC_DIRAC>(full, sp), "s6_fwd_dirac"); break;
        default: run(fwd_variant<LR_DISC_ZOH_EULER>(full, sp), "s6_fwd_zoh_euler"); break;
    }
    return check_launch();
}

lr_status s6_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                 const lr_grads& gr, char* ws, cudaStream_t st) {
    S6Args a = make_args(d, in, const_cast<void*>(ckpt), ws, true);
    CUtensorMap mX, mDT, mZ, mDY, mB, mC, mdX, mdDT, mdZ;
    const uint32_t S = (uint32_t)d.segment;
    bool ok = make_tmap_3d(&mX, in.x, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mDT, in.delta, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mZ, a.has_z ? in.z : in.x, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mDY, dy, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mB, in.Bm, 2, kN, d.L, d.B, kN, S) &&
              make_tmap_3d(&mC, in.Cm, 2, kN, d.L, d.B, kN, S) &&
              make_tmap_3d(&mdX, gr.dx, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mdDT, gr.ddelta, 2, d.D, d.L, d.B, kDB, S) &&
              make_tmap_3d(&mdZ, a.has_z ? gr.dz : gr.dx, 2, d.D, d.L, d.B, kDB, S);
    if (!ok) return LR_ERR_INVALID_ARG;
    const int grid = a.B * a.ncb;
    auto run = [&](auto kernel, const char* name) {
        set_smem(kernel, kBwdSmem);
        note_launch(name);
        kernel<<<grid, kThreads, kBwdSmem, st>>>(mX, mDT, mZ, mDY, mB, mC, mdX, mdDT, mdZ, a);
    };
    const bool full = (d.flags & LR_FULL_STATE) != 0, sp = a.softplus != 0;  // compile-time variants
    switch (d.disc) {
        case LR_DISC_ZOH: run(bwd_variant<LR_DISC_ZOH>(full, sp), "s6_bwd_zoh"); break;
        case LR_DISC_BILINEAR: run(bwd_variant<LR_DISC_BILINEAR>(full, sp), "s6_bwd_bilinear"); break;
        case LR_DISC_DIRAC: run(bwd_variant<LR_DISC_DIRAC>(full, sp), "s6_bwd_dirac"); break;
        default: run(bwd_variant<LR_DISC_ZOH_EULER>(full, sp), "s6_bwd_zoh_euler"); break;
    }
    lr_status s = check_launch();
    if (s != LR_OK) return s;
    note_launch("s6_param_reduce");
    s6_reduce_kernel<<<4 * 148, 256, 0, st>>>(a, gr.dBm, gr.dCm, gr.dA, a.has_d ? gr.dDskip : nullptr,
                                              a.softplus ? gr.ddelta_bias : nullptr);
    return check_launch();
}

}  // namespace lrs
