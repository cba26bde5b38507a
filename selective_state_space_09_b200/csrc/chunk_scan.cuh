// chunk_scan.cuh -- the chunk-state scan shared by the matrix-state kinds (SSD and GLA) on
// tcgen05: one CTA per (batch row, head, 64 value columns) folds the chunk products
// S_{c+1} = e^{l_Q,c} S_c + R_c^T diag(w) Z_c (or the adjoint in reverse) into a register-resident
// state and writes every chunk's entering state (the checkpoint slots), counting each slot as it
// lands so that the chunk kernels can run beside it.
//
// Recurrence ("mlx-recurrence", Apple Developer Forums thread 840535, "Current kernels": ssd_scan
// and gla_scan, matrix states [B, H, Dh, N] and [B, H, Dh, Dh]; the chunked evaluation of the
// K-Search / mlx-mamba post, paragraph after Table 1).
#pragma once

#include "chunk_common.cuh"

namespace lrs {
using namespace chunkc;
namespace {

constexpr int kScanP = 64;                               // value columns of one scan CTA
constexpr uint32_t kScanTile = kKD * kScanP * 2;         // one 128 x 64 block of a bf16 state tile

// Per-step decay of the scan: SSD with the default kernel variant (ZOH, raw dt), SSD with the
// general one (discretisation and softplus front-end from the arguments), GLA, and SSD with the
// bilinear discretisation (abar may be negative: a sign parity is carried beside the log
// magnitude, see bilinear_step).
enum { kScanSsd = 0, kScanSsdGen = 1, kScanGla = 2, kScanSsdBil = 3 };

// Floor of a step's log decay: e^{-87} is still a normal fp32 number, so products of decays stay
// finite and an exact zero decay (bilinear abar at dt A = -2) enters as e^{-87}.
constexpr float kMinLogDecay = -87.0f;

// Bilinear step (Tustin): u = dt A / 2, abar = (1 + u) / (1 - u), beta = dt / (1 - u).  abar lies
// in (-1, 1] for A < 0 and is negative where dt |A| > 2, so products of decays are carried as a
// log magnitude lam = log|abar| (floored at kMinLogDecay) and a sign: neg = 1 where abar < 0, and
// the sign of a product over steps (s, t] is (-1)^(#neg in (s, t]).
__device__ __forceinline__ void bilinear_step(float dt, float Ah, float& lam, float& beta, float& neg) {
    const float u = 0.5f * dt * Ah;
    const float num = 1.0f + u, den = 1.0f - u;
    lam = fmaxf(__logf(fabsf(num)) - __logf(den), kMinLogDecay);
    beta = dt / den;
    neg = num < 0.0f ? 1.0f : 0.0f;
}
// (-1)^n for an inclusive count n of negative steps (exact small integers in fp32)
__device__ __forceinline__ float parity_sign(float n) { return (__float2int_rn(n) & 1) ? -1.0f : 1.0f; }

struct ScanArgs {
    int B, L, H, G, HpG, nchunk;  // GLA: G = H, HpG = 1
    int halves;                   // 64-column halves of the value width (SSD 1; GLA V / 64)
    int disc;                     // SSD: LR_DISC_ZOH, LR_DISC_DIRAC or LR_DISC_ZOH_EULER
    int softplus;                 // SSD LR_DELTA_SOFTPLUS: dt = softplus(delta + bias_h)
    const float* dbias;           // SSD [H] or null
    const __nv_bfloat16* dt;      // [B, L, H]: SSD raw dt, GLA gate g in (0, 1)
    const float* A;               // SSD [H]
    WsHeader* hdr;
    int withhold;                 // LR_TEST_WITHHOLD_CARRY: slot 0 is never counted (failure-path test)
    int f32_every;                // forward: the f32 state of chunk c is a checkpoint when c % f32_every == 0
                                  // (slot c / f32_every); 0 or 1 = every chunk
    int seg_k;                    // segment mode (dir > 0, recompute): segments of seg_k chunks, each
                                  // restarted from its state in s_init; 0 = one chain over the sequence
    const float* s_init;          // segment mode: f32 state entering each segment [nseg][B*H][kKD][vd]
    int vd;                       // value width of s_init rows
};

// beta of one step inside the sequence (lam = dt A_h): ZOH (e^{lam} - 1) / A_h, dirac 1,
// ZOH-Euler dt.  abar = e^{lam} in all three.
__device__ __forceinline__ float ssd_beta(int disc, float lam, float dt, float Ah) {
    if (disc == LR_DISC_DIRAC) return 1.0f;
    if (disc == LR_DISC_ZOH_EULER) return dt;
    return (ex2(lam * kLog2e) - 1.0f) / Ah;
}

// The kernels come in two variants: the default one (ZOH, raw dt) with both fixed at compile time,
// and the general one (GEN) that takes the discretisation and the softplus front-end from the
// arguments.
template <bool GEN, class Args>
__device__ __forceinline__ int disc_of(const Args& a) {
    if constexpr (GEN) return a.disc;
    return LR_DISC_ZOH;
}
template <bool GEN, class Args>
__device__ __forceinline__ bool softplus_of(const Args& a) {
    if constexpr (GEN) return a.softplus != 0;
    return false;
}

// dt of head h from the raw delta: itself, or softplus(delta + bias_h) (LR_DELTA_SOFTPLUS)
template <bool GEN, class Args>
__device__ __forceinline__ float ssd_dt(const Args& a, float raw, int h) {
    if (!softplus_of<GEN>(a)) return raw;
    const float v = raw + (a.dbias ? a.dbias[h] : 0.0f);
    return v > 20.0f ? v : log1pf(__expf(v));
}

// Barrier of the 128 threads of warpgroup wg (named barrier 1 + wg).
__device__ __forceinline__ void wg_sync(int wg) { asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory"); }

// Inclusive prefix sum over the 128 threads of warpgroup wg (same order as cta_inclusive_sum).
__device__ __forceinline__ float wg_inclusive_sum(float x, float* tmp, int wg) {
    const int lane = threadIdx.x & 31, w = (threadIdx.x >> 5) & 3;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[w] = x;
    wg_sync(wg);
    float add = 0.0f;
    for (int k = 0; k < w; ++k) add += tmp[k];
    wg_sync(wg);
    return x + add;
}

// -------------------------------------------------------------------- chunk states, scanned
// One CTA per (batch row, head, 64-column half of the value width) walks the chunks in order
// (dir > 0) or in reverse (dir < 0).  With R the row operand (SSD: B, C of the head's group; GLA:
// k, q of the head) and Z the value operand (SSD: x, dy; GLA: v, dO):
//   dir > 0: S_0 = 0,      S_{c+1} = e^{l_Q,c} S_c + R_c^T diag(w) Z_c    slot c <- S_c
//            (the f32 checkpoint and its bf16 tile copy);
//   dir < 0: G_{last} = 0, G_{c-1} = e^{l_Q,c} G_c + R_c^T diag(E) Z_c    slot c <- G_c (bf16 tile).
// The per-step log decay and input weight: SSD lam = dt A_h and beta of the discretisation; GLA
// lam = log g_t and beta = 1.
// Only the fold is sequential; the chunk products are independent, so the CTA runs as a pipeline of
// roles joined by mbarriers:
//   warps 0-3 (prep, thread = step t): decays of kScanPrepGroup chunks at a time (inclusive sums of
//     lam), then per chunk, once its tiles are in, row t of Z scaled by w_t (E_t) in place;
//   warp 8 lane 0 (issue): the tcgen05 product of each prepared chunk into one of kScanBufs TMEM
//     buffers;
//   warp 10 lane 0 (load): the TMA loads of the chunk tiles into a ring of NS stages, each stage
//     refilled as soon as the product that reads it has completed;
//   warps 4-7 (fold, thread = state row n, all 64 columns in registers): S <- e^{l_Q} S + product,
//     then S leaves through shared memory (f32: TMA store of two 32-column boxes; bf16 tile: one
//     bulk copy, the tile already in its global format);
//   warp 9: zeroes the dB, dC rows the SSD gradient kernel adds into (backward, by chunk, flagged),
//     then counts the slots whose copies have landed (see below);
//   warp 11 (dt): the raw per-step decay input (SSD dt, GLA g) of every chunk into a ring in shared
//     memory, kDtRing chunks ahead (kept out of the prep warps: their barriers and arrivals would
//     wait for loads in flight).
// No scan CTA waits on another.  Once the copies of a slot have landed the fold tells warp 9 (a counter
// in shared memory), which counts the slot in global memory (ready[slot][b][g], one count per head
// and half of the group, so that a consumer needs one acquire load for all of them), so that the output kernel
// (forward) or the gradient kernel (backward) can start on a chunk before the whole scan has
// finished; the fold itself never waits for a global-scope release.
// NS stages: 3 when the f32 states are staged too (forward), 4 otherwise.
constexpr int kScanBufs = 4, kDecRing = 16, kScanPrepGroup = 4, kDtRing = 8;
constexpr int kScanThreads = 384;
template <int NS, bool F32> struct ScanSmem {
    static constexpr size_t kRt = (size_t)kQ * kKD * 2;            // R tile (B or C), 128 x 128 bf16
    static constexpr size_t kStage = kRt + (size_t)kQ * kScanP * 2;  // then the Z tile
    static constexpr size_t kF32 = (size_t)NS * kStage;             // f32 state staging, 2 boxes
    static constexpr size_t kBf = kF32 + (F32 ? (size_t)kKD * kScanP * 4 : 0);  // bf16 tile staging
    static constexpr size_t kTmp = kBf + kScanTile;                  // prep scan scratch [4][8], l_Q and sign [8]
    static constexpr size_t kDecP = kTmp + 256;                      // e^{l_Q}: prep -> issue [kDecRing]
    static constexpr size_t kDecF = kDecP + 4 * kDecRing;            // e^{l_Q}: issue -> fold [kDecRing]
    static constexpr size_t kDt = kDecF + 4 * kDecRing;              // dt ring [kDtRing][128][8] bf16
    static constexpr size_t kBar = kDt + (size_t)kDtRing * kQ * 16;  // full, scaled, prod, bfree, dt full / empty
    static constexpr size_t kTmem = kBar + 8 * (NS + 3 * kScanBufs + 2 * kDtRing);
    static constexpr size_t kPub = kTmem + 8;                        // puts whose copies landed, minus 1
    static constexpr size_t kEnd = kTmem + 16;
    static constexpr size_t kAlloc = kEnd + 1024;
    static_assert(kStage % 1024 == 0, "stages keep the 1024-byte alignment of SW128 tiles");
    static_assert(kDt % 128 == 0, "dt ring slots are TMA destinations");
    static_assert(kAlloc <= 232448, "scan CTA exceeds the shared memory of one CTA");
    // the prep role writes e^{l_Q} at most NS + kScanPrepGroup chunks ahead of the issuing thread;
    // kScanBufs >= NS keeps every mbarrier at most one phase ahead of its waiters
    static_assert(kScanBufs >= NS && NS + kScanPrepGroup < kDecRing, "ring sizes");
    static_assert(kDtRing % kScanPrepGroup == 0 && kDtRing >= 2 * kScanPrepGroup, "dt ring holds two prep groups");
};

template <int NS, bool F32, int MODE>
__global__ void __launch_bounds__(kScanThreads, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap mR, const __grid_constant__ CUtensorMap mZ,
                  const __grid_constant__ CUtensorMap mS, const __grid_constant__ CUtensorMap mDt, int dt_tma,
                  ScanArgs a, char* __restrict__ tiles, int dir, unsigned int* ready, float* zero0, float* zero1,
                  unsigned int* zready) {
    using SM = ScanSmem<NS, F32>;
    constexpr bool GEN = MODE == kScanSsdGen || MODE == kScanSsdBil;
    char* sm = smem_base1024();
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + SM::kBar);
    uint64_t* scaled = full + NS;
    uint64_t* prod = scaled + kScanBufs;
    uint64_t* bfree = prod + kScanBufs;
    uint64_t* dtfull = bfree + kScanBufs;
    uint64_t* dtempty = dtfull + kDtRing;
    // dt ring: slot s, step t holds the raw dt of heads 8 (h / 8) .. 8 (h / 8) + 7 (a TMA box of
    // the [B, L, H] tensor when H is a multiple of 8; else only head h's entry is written)
    __nv_bfloat16* dtb = reinterpret_cast<__nv_bfloat16*>(sm + SM::kDt);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmem);
    int* pubdone = reinterpret_cast<int*>(sm + SM::kPub);
    float* tmp = reinterpret_cast<float*>(sm + SM::kTmp);
    float* decp = reinterpret_cast<float*>(sm + SM::kDecP);
    float* decf = reinterpret_cast<float*>(sm + SM::kDecF);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = blockIdx.x % a.halves, bh = blockIdx.x / a.halves, b = bh / a.H, h = bh % a.H;
    const int g = h / a.HpG, rsel = MODE == kScanGla ? h : g;  // R: per group (SSD) or head (GLA)
    const int hx = h & 7;  // this head's column of a dt ring row
    const size_t slot_bytes = (size_t)kScanTile * a.halves;  // one bf16 state tile, all halves
    const int BH = a.B * a.H;
    // Segment mode walks the segments from the last to the first (the gradient kernels that wait
    // for the rebuilt states take the chunks from the last one), the chunks of a segment in order;
    // each segment restarts from its checkpointed state and has one product fewer than chunks.
    const int K = a.seg_k > 0 ? a.seg_k : a.nchunk;
    const int nseg = (a.nchunk + K - 1) / K;
    const int nlast = a.nchunk - (nseg - 1) * K;  // chunks of the last segment
    const int nk = a.nchunk - nseg;               // products
    // chunk of product k and of put q (segment mode; otherwise the sequence in order / reversed)
    auto chunk_of = [&](int k) {
        if (!a.seg_k) return dir > 0 ? k : a.nchunk - 1 - k;
        if (k < nlast - 1) return (nseg - 1) * K + k;
        const int kk = k - (nlast - 1);
        return (nseg - 2 - kk / (K - 1)) * K + kk % (K - 1);
    };
    auto slot_of_put = [&](int q) {
        if (!a.seg_k) return dir > 0 ? q : a.nchunk - 1 - q;
        if (q < nlast) return (nseg - 1) * K + q;
        const int qq = q - nlast;
        return (nseg - 2 - qq / K) * K + qq % K;
    };
    auto stage = [&](int k) { return sm + (size_t)(k % NS) * SM::kStage; };
    auto load = [&](int k) {
        char* st = stage(k);
        uint64_t* bar = &full[k % NS];
        const int t0 = chunk_of(k) * kQ;
        mbar_arrive_expect_tx(bar, (uint32_t)SM::kStage);
        for (int j = 0; j < kKD / 64; ++j) tma_load_4d(st + j * kQ * 128, &mR, bar, 64 * j, rsel, t0, b);
        tma_load_4d(st + SM::kRt, &mZ, bar, 64 * half, h, t0, b);
    };
    pdl_launch_dependents();
    if (tid == 256) {
        for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
        for (int i = 0; i < kScanBufs; ++i) {
            mbar_init(&scaled[i], 128);
            mbar_init(&prod[i], 2);  // the product's commit and the issuing thread (e^{l_Q} handed on)
            mbar_init(&bfree[i], 128);
        }
        for (int i = 0; i < kDtRing; ++i) {
            mbar_init(&dtfull[i], dt_tma ? 1 : 32);
            mbar_init(&dtempty[i], 1);
        }
        *pubdone = -1;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 8) tc::tmem_alloc(tmem_slot, 64 * kScanBufs);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp < 4) {
        // ------------------------------------------------------------------------- prep
        constexpr int NG = kScanPrepGroup;
        const int t = tid;
        const float Ah = MODE == kScanGla ? 0.0f : a.A[h];
        for (int k0 = 0; k0 < nk; k0 += NG) {
            // l[j]: log decay of step t of chunk k0 + j; for bilinear l[NG + j]: its negative-step count
            constexpr int NV = MODE == kScanSsdBil ? 2 * NG : NG;
            float l[NV], beta[NG], f[NG];
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const int k = k0 + j;
                ok = ok && mbar_wait(&dtfull[k % kDtRing], (uint32_t)((k / kDtRing) & 1), a.hdr, 745);
                const bool in_seq = chunk_of(k) * kQ + t < a.L;
                const float raw = __bfloat162float(dtb[((k % kDtRing) * kQ + t) * 8 + hx]);
                if constexpr (MODE == kScanGla) {  // lam = log g, beta = 1 (0 past L)
                    l[j] = in_seq ? __logf(raw) : 0.0f;
                    beta[j] = in_seq ? 1.0f : 0.0f;
                } else if constexpr (MODE == kScanSsdBil) {  // log|abar|, sign count (0 past L)
                    l[j] = beta[j] = l[NG + j] = 0.0f;
                    if (in_seq) bilinear_step(ssd_dt<true>(a, raw, h), Ah, l[j], beta[j], l[NG + j]);
                } else {
                    const float dtv = in_seq ? ssd_dt<GEN>(a, raw, h) : 0.0f;  // 0 past L
                    l[j] = dtv * Ah;
                    beta[j] = in_seq ? ssd_beta(disc_of<GEN>(a), l[j], dtv, Ah) : 0.0f;  // no input past L
                }
            }
            wg0_inclusive_sum_n<NV>(l, tmp);  // its barriers: every prep thread has read the dt slots
            if (t == 0) {
#pragma unroll
                for (int j = 0; j < NG; ++j) mbar_arrive(&dtempty[(k0 + j) % kDtRing]);
            }
            if (t == kQ - 1) {
#pragma unroll
                for (int j = 0; j < NV; ++j) tmp[32 + j] = l[j];
            }
            wg_sync(0);
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const float lQ2 = tmp[32 + j] * kLog2e, lt2 = l[j] * kLog2e;
                // signs of the decay products (bilinear): over (t, Q] and over (0, t]
                float sgQ = 1.0f, sgt = 1.0f;
                if constexpr (MODE == kScanSsdBil) {
                    sgQ = parity_sign(tmp[32 + NG + j]);
                    sgt = parity_sign(l[NG + j]);
                }
                f[j] = dir > 0 ? ex2(lQ2 - lt2) * beta[j] * (sgQ * sgt) : ex2(lt2) * sgt;
                if (t == 0) decp[(k0 + j) % kDecRing] = ex2(lQ2) * sgQ;
            }
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const int k = k0 + j;
                if (k >= nk) break;
                ok = ok && mbar_wait(&full[k % NS], (uint32_t)((k / NS) & 1), a.hdr, 740);
                char* z = stage(k) + SM::kRt;
                uint4 raw[kScanP / 8];  // the whole row first: its loads overlap
#pragma unroll
                for (int c = 0; c < kScanP / 8; ++c)
                    raw[c] = *reinterpret_cast<const uint4*>(z + tc::sw128_off(t, 8 * c, kQ));
#pragma unroll
                for (int c = 0; c < kScanP / 8; ++c) {
                    __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&raw[c]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 v = __bfloat1622float2(hv[i]);
                        hv[i] = __floats2bfloat162_rn(v.x * f[j], v.y * f[j]);
                    }
                }
#pragma unroll
                for (int c = 0; c < kScanP / 8; ++c) *reinterpret_cast<uint4*>(z + tc::sw128_off(t, 8 * c, kQ)) = raw[c];
                fence_proxy_async_smem();
                mbar_arrive(&scaled[k % kScanBufs]);
            }
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------------------ issue
        if (lane == 0) {
            for (int k = 0; k < nk; ++k) {
                const int buf = k % kScanBufs, use = k / kScanBufs;
                ok = ok && mbar_wait(&scaled[buf], (uint32_t)(use & 1), a.hdr, 741);
                if (k >= kScanBufs) ok = ok && mbar_wait(&bfree[buf], (uint32_t)((use - 1) & 1), a.hdr, 742);
                tc::fence_after_sync();
                decf[k % kDecRing] = decp[k % kDecRing];
                if (ok)
                    tc::mma_tiles(tmem + 64 * buf, smem_u32(stage(k)), 1, kQ, smem_u32(stage(k) + SM::kRt), 1, kQ,
                                  kKD, kScanP, kQ, 0);
                tc::commit(&prod[buf]);
                mbar_arrive(&prod[buf]);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------------------- load
        if (lane == 0) {
            for (int k = 0; k < nk && k < NS; ++k) load(k);
            for (int k = 0; k + NS < nk; ++k) {  // the product of chunk k has read its stage
                ok = ok && mbar_wait(&prod[k % kScanBufs], (uint32_t)((k / kScanBufs) & 1), a.hdr, 743);
                if (ok) load(k + NS);
            }
        }
    } else if (warp == 11) {
        // --------------------------------------------------------------------------- dt
        // TMA: one box of 8 heads x 128 steps per chunk.  Loads: one prep group (kScanPrepGroup
        // chunks) per batch of loads: an arrival waits for every load of the thread in flight, so
        // the loads of a group are all issued before the first one.
        constexpr int NG = kScanPrepGroup;
        if (dt_tma) {
            if (lane == 0)
                for (int k = 0; k < nk; ++k) {
                    const int slot = k % kDtRing;
                    if (k >= kDtRing)
                        ok = ok && mbar_wait(&dtempty[slot], (uint32_t)(((k / kDtRing) - 1) & 1), a.hdr, 746);
                    mbar_arrive_expect_tx(&dtfull[slot], (uint32_t)(kQ * 16));
                    tma_load_3d(dtb + (size_t)slot * kQ * 8, &mDt, &dtfull[slot], h & ~7, chunk_of(k) * kQ, b);
                }
            // the prep group's chunks past the last product: nothing to load
            if (lane == 0)
                for (int k = nk; k % NG != 0; ++k) {
                    const int slot = k % kDtRing;
                    if (k >= kDtRing)
                        ok = ok && mbar_wait(&dtempty[slot], (uint32_t)(((k / kDtRing) - 1) & 1), a.hdr, 746);
                    mbar_arrive(&dtfull[slot]);
                }
        } else
        for (int k0 = 0; k0 < nk; k0 += NG) {
            if (k0 >= kDtRing) {
#pragma unroll
                for (int j = 0; j < NG; ++j) {
                    const int k = k0 + j;
                    ok = ok && mbar_wait(&dtempty[k % kDtRing], (uint32_t)(((k / kDtRing) - 1) & 1), a.hdr, 746);
                }
            }
            float v[NG][kQ / 32];
#pragma unroll
            for (int j = 0; j < NG; ++j)
#pragma unroll
                for (int i = 0; i < kQ / 32; ++i) {
                    const int k = k0 + j, tt = chunk_of(k) * kQ + lane + 32 * i;
                    v[j][i] = k < nk && tt < a.L ? __bfloat162float(a.dt[((size_t)b * a.L + tt) * a.H + h]) : 0.0f;
                }
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const int slot = (k0 + j) % kDtRing;
#pragma unroll
                for (int i = 0; i < kQ / 32; ++i)
                    dtb[(slot * kQ + lane + 32 * i) * 8 + hx] = __float2bfloat16_rn(v[j][i]);
                mbar_arrive(&dtfull[slot]);
            }
        }
    } else if (warp == 9) {
        // --------------------------------------------------------------- zero, publish
        // backward, several head blocks per group: the dB, dC rows [B, L, G, N] of chunk c, group
        // g are zeroed by head g HpG + (c mod HpG) of the batch row and flagged (zready), for the
        // gradient kernel's reduction-adds
        if (zready) {
            pdl_wait();  // the previous kernel of the stream may still read dB, dC
            const int hg = h - g * a.HpG;
            for (int c = hg; c < a.nchunk; c += a.HpG) {
                const int rows = min(kQ, a.L - c * kQ);
                for (int r = 0; r < rows; ++r) {
                    const size_t off = (((size_t)b * a.L + c * kQ + r) * a.G + g) * kKD + 4 * lane;
                    *reinterpret_cast<float4*>(zero0 + off) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    *reinterpret_cast<float4*>(zero1 + off) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release(&zready[((size_t)c * a.B + b) * a.G + g], 1u);
            }
        }
        // the fold's puts in order (put q writes slot q forward, slot nchunk - 1 - q backward)
        if (ready && lane == 0) {
            int next = 0;
            unsigned long long t0 = global_ns();
            while (next < a.nchunk) {
                const int done = ld_acquire_cta(pubdone);
                if (done >= next) {
                    for (; next <= done; ++next) {
                        const int slot = slot_of_put(next);
                        if (!(a.withhold && slot == 0)) red_release_add(&ready[((size_t)slot * a.B + b) * a.G + g], 1u);
                    }
                    t0 = global_ns();
                    continue;
                }
                if (global_ns() - t0 > kWaitLimitNs) {
                    record_error(a.hdr, LR_ERR_TIMEOUT, 747);
                    break;
                }
                __nanosleep(100);
            }
        }
    } else {
        // ------------------------------------------------------------------------- fold
        const int n = tid - 128, fl = n == 0;  // fl: the thread that issues the copies
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // fl: the last two puts whose copies were issued (pub1 the latest); a put is handed to the
        // publishing warp once the copies of the put after it have been issued, by which time its
        // own have landed
        int nput = 0, pub1 = -1, pub2 = -1;
        auto publish = [&](int q) {  // puts 0 .. q have landed
            fence_proxy_async_global();
            st_release_cta(pubdone, q);
        };
        float S[kScanP];
#pragma unroll
        for (int i = 0; i < kScanP; ++i) S[i] = 0.0f;
        // segment mode: the checkpointed state entering segment sg, row n
        auto load_state = [&](int sg) {
            const float4* src = reinterpret_cast<const float4*>(
                a.s_init + (((size_t)sg * BH + bh) * kKD + n) * a.vd + kScanP * half);
#pragma unroll
            for (int i = 0; i < kScanP / 4; ++i) {
                const float4 v = src[i];
                S[4 * i] = v.x;
                S[4 * i + 1] = v.y;
                S[4 * i + 2] = v.z;
                S[4 * i + 3] = v.w;
            }
        };
        // the previous kernel of the stream may still read the slots; in segment mode the slots are
        // this kernel's own workspace region, which the kernel before it (the backward scan) never
        // touches, so it runs beside that kernel
        if (!a.s_init) pdl_wait();
        // S into slot c through the staging buffers (free: the copies of the previous slot have
        // read them before the first barrier)
        auto put = [&](int c) {
            if (fl) {
                if (ready && pub2 >= 0) {
                    bulk_wait_all_but_1();
                    publish(pub2);
                }
                bulk_wait_read_all();
            }
            wg_sync(1);
            const int every = a.f32_every > 1 ? a.f32_every : 1;
            const bool f32_slot = F32 && c % every == 0;  // a checkpoint slot (forward)
            if (f32_slot) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    char* box = sm + SM::kF32 + j * (kKD * 128);  // columns 32 j .. 32 j + 31
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<float4*>(box + n * 128 + ((i ^ (n & 7)) << 4)) =
                            make_float4(S[32 * j + 4 * i], S[32 * j + 4 * i + 1], S[32 * j + 4 * i + 2],
                                        S[32 * j + 4 * i + 3]);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<uint4*>(sm + SM::kBf + tc::sw128_off(n, 8 * i, kKD)) = pack_bf16x8(S + 8 * i);
            fence_proxy_async_smem();
            wg_sync(1);
            if (fl) {
                if (f32_slot) {
                    tma_store_4d(&mS, sm + SM::kF32, 64 * half, 0, bh, c / every);
                    tma_store_4d(&mS, sm + SM::kF32 + kKD * 128, 64 * half + 32, 0, bh, c / every);
                }
                bulk_store(tiles + (size_t)c * BH * slot_bytes + (size_t)bh * slot_bytes + (size_t)half * kScanTile,
                           sm + SM::kBf, kScanTile);
                bulk_commit();
            }
            pub2 = pub1;
            pub1 = nput++;
        };
        // one product folded into S, then S put into the slot of the next chunk
        auto fold = [&](int k) {
            const int buf = k % kScanBufs;
            ok = ok && mbar_wait(&prod[buf], (uint32_t)((k / kScanBufs) & 1), a.hdr, 744);
            tc::fence_after_sync();
            float v[kScanP];
#pragma unroll
            for (int j = 0; j < kScanP; j += 16) tc::ld16(tmem + 64 * buf + j + lane_off, v + j);
            tc::wait_ld();
            tc::fence_before_sync();
            mbar_arrive(&bfree[buf]);
            const float d = decf[k % kDecRing];
#pragma unroll
            for (int i = 0; i < kScanP; ++i) S[i] = fmaf(d, S[i], v[i]);
            put(chunk_of(k) + dir);
        };
        if (!a.seg_k) {
            put(dir > 0 ? 0 : a.nchunk - 1);
            for (int k = 0; k < nk; ++k) fold(k);
        } else {
            int k = 0;
            for (int sg = nseg - 1; sg >= 0; --sg) {
                load_state(sg);
                put(sg * K);
                const int nc = sg == nseg - 1 ? nlast : K;
                for (int j = 0; j + 1 < nc; ++j) fold(k++);
            }
        }
        if (fl) {
            bulk_wait_all();
            if (ready) publish(pub1);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 8) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 64 * kScanBufs);
    }
}

// TMA map of f32 state slots [nslot][B*H][128][VD], boxes of 32 columns x 128 rows (128-byte
// swizzle), written by the scan kernel.
inline bool map_states_vd(CUtensorMap* m, void* base, int64_t BH, int64_t nslot, int VD) {
    uint64_t dims[4] = {(uint64_t)VD, (uint64_t)kKD, (uint64_t)BH, (uint64_t)nslot};
    uint64_t str[3] = {(uint64_t)VD * 4, (uint64_t)kKD * VD * 4, (uint64_t)BH * kKD * VD * 4};
    uint32_t box[4] = {32, (uint32_t)kKD, 1, 1};
    return make_tmap(m, base, 4, 4, dims, str, box, true);
}

// TMA map of a per-step, per-head [B, L, H] bf16 tensor (SSD dt, GLA g) with boxes of 8 heads x
// 128 steps (16-byte rows): only when a row of H heads spans a multiple of 16 bytes (H a multiple
// of 8); false otherwise.
inline bool map_dt(CUtensorMap* m, int64_t B, int64_t L, int64_t H, const void* dt) {
    if (H % 8 != 0) return false;
    return make_tmap_3d(m, dt, 2, (uint64_t)H, (uint64_t)L, (uint64_t)B, 8, (uint32_t)kQ);
}

}  // namespace
}  // namespace lrs
