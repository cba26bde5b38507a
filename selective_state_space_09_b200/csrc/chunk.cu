// chunk.cu -- chunked-matmul chassis: ssd_scan and gla_scan on tcgen05 tensor cores (sm_100a).
//
// Both kinds are the recurrence S_t = e^{lam_t} S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t with a
// scalar decay per step and head ("mlx-recurrence", Apple Developer Forums thread 840535,
// "Current kernels": ssd_scan state [B, H, Dh, N], gla_scan state [B, H, Dh, Dh]):
//   gla:  q, k, v per head, lam = log g, beta = 1;
//   ssd:  q = C_t, k = B_t (shared by the heads of a group), v = x_t, lam = dt A_h,
//         beta = (e^{dt A_h} - 1) / A_h (ZOH), y = o + D_h x.
// The chunked form evaluates a chunk of Q = 128 steps with dense products (chunk-local cumulative
// log decay l_t):
//   o_t = sum_{s<=t} e^{l_t - l_s} beta_s (q_t . k_s) v_s  +  e^{l_t} q_t S_in
//   S_out = e^{l_Q} S_in + sum_s e^{l_Q - l_s} beta_s k_s v_s^T
// and chunks compose with the associative operator of the K-Search / mlx-mamba post (techtrendfeed
// repost, paragraph after Table 1) -- here with a scalar coefficient e^{l_Q} and a matrix state.
//
// Forward tile = (batch row, head, chunk).  TMA brings q, k (128 x 128) and v (128 x V) into
// 128-byte-swizzled shared-memory tiles; tcgen05 computes, with fp32 accumulators in TMEM,
//   G1: Sqk = Q K^T                 (128 x 128 x K)
//   G2: Y   = P V                   (P = masked, decayed, beta-scaled Sqk, written as bf16)
//   G4: Sl  = K^T (w . V)           (w_s = e^{l_Q - l_s} beta_s; the chunk's own state increment)
//   G3: Y2  = Q S_in                (S_in as bf16)
// and y = Y + e^{l_t} Y2 (+ D x).  The state entering each chunk comes from a single-pass
// decoupled look-back: a tile publishes its aggregate (e^{l_Q}, Sl) as soon as G4 is done, walks
// back to the nearest chunk that has published its inclusive state, and folds the aggregates in
// chain order (deterministic).  The inclusive states are the checkpoints: the checkpoint segment
// equals the chunk (128 steps), slot c = state entering chunk c.
#include "chunk_common.cuh"

namespace lrs {
using namespace chunkc;
namespace {

struct ChunkArgs {
    int kind;                 // LR_SSD / LR_GLA
    int B, L, H, G, nchunk;   // G = groups (SSD), H heads
    int VD;                   // value dim (SSD P, GLA V)
    const __nv_bfloat16* lam; // SSD: dt [B, L, H]; GLA: g [B, L, H]
    const float* A;           // SSD [H]
    const float* Dskip;       // SSD [H] or null
    float* ckpt;              // [nchunk, B, H, KD, VD] f32
    WsHeader* hdr;
    unsigned int* flags;      // [B*H*nchunk]
    float* agg;               // [B*H*nchunk][KD][VD]
    float* aggA;              // [B*H*nchunk] chunk decay e^{l_Q}
    unsigned int dflags;
};

// Per-step log decay and beta of row t (t >= L gives no decay, no input).
__device__ __forceinline__ void step_coef(const ChunkArgs& a, int b, int h, int t, float& lam, float& beta) {
    lam = 0.0f;
    beta = 0.0f;
    if (t >= a.L) return;
    const float v = __bfloat162float(a.lam[((size_t)b * a.L + t) * a.H + h]);
    if (a.kind == LR_SSD) {
        const float Ah = a.A[h];
        lam = v * Ah;
        beta = (ex2(lam * kLog2e) - 1.0f) / Ah;
    } else {
        lam = __logf(v);
        beta = 1.0f;
    }
}

// Nearest chunk, walking from `c` in direction `dir`, whose inclusive record is published
// (flags read four at a time; an unpublished flag is waited for, with a bound).  Returns `stop`
// (-1 or nchunk) if the walk leaves the row.  A wait that gives up counts as published (the
// error is recorded and the caller proceeds with whatever the record holds).
__device__ __forceinline__ int find_prefix(const unsigned int* flags, int c, int dir, int nchunk,
                                           WsHeader* hdr, int info) {
    int j = c + dir;
    const int stop = dir < 0 ? -1 : nchunk;
    while (j != stop) {
        unsigned int f[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int jj = j + k * dir;
            f[k] = (jj >= 0 && jj < nchunk) ? ld_acquire(&flags[jj]) : kFlagPrefix;
        }
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
            const int jj = j + k * dir;
            if (jj < 0 || jj >= nchunk) return stop;
            unsigned int fk = f[k];
            if (fk == kFlagNone) fk = wait_flag(&flags[jj], hdr, info);
            if (fk != kFlagAgg) return jj;  // prefix (or a wait that gave up)
        }
        j += 4 * dir;
    }
    return stop;
}

// x[0..16) = fold in chain order of the aggregates first .. last (x <- a_i x + agg_i) starting
// from the 16 values at `pre` (or zero).  agg_row0 points at the caller's row inside record 0;
// records are `rec_stride` floats apart and indexed row0 + i.  dir = +1 folds i = first .. last-1
// upwards, dir = -1 folds i = first .. last+1 downwards.  Loads of up to three records are issued
// together.
__device__ __forceinline__ void fold_chain(float* x, const float* pre, const float* agg_row0, size_t rec_stride,
                                           const float* aggA, size_t row0, int first, int last, int dir) {
    float4 p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = pre ? __ldcg(reinterpret_cast<const float4*>(pre) + e) : make_float4(0, 0, 0, 0);
    int i = first;
    while (i != last) {
        float4 r[3][4];
        float ar[3];
        int n = 0;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int ii = i + k * dir;
            const bool live = dir > 0 ? ii < last : ii > last;
            if (live) {
                const float* src = agg_row0 + (row0 + ii) * rec_stride;
#pragma unroll
                for (int e = 0; e < 4; ++e) r[k][e] = __ldcg(reinterpret_cast<const float4*>(src) + e);
                ar[k] = __ldcg(&aggA[row0 + ii]);
                n = k + 1;
            }
        }
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            if (k < n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    p[e].x = fmaf(ar[k], p[e].x, r[k][e].x);
                    p[e].y = fmaf(ar[k], p[e].y, r[k][e].y);
                    p[e].z = fmaf(ar[k], p[e].z, r[k][e].z);
                    p[e].w = fmaf(ar[k], p[e].w, r[k][e].w);
                }
            }
        }
        i += n * dir;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[4 * e] = p[e].x;
        x[4 * e + 1] = p[e].y;
        x[4 * e + 2] = p[e].z;
        x[4 * e + 3] = p[e].w;
    }
}

// Shared-memory plan of the forward tile (offsets from a 1024-aligned base).  P lives in tensor
// memory, K is rescaled in place once Q K^T is done, and the output is staged in the Q tile after
// the last product that reads Q, so the SSD tile (V = 64) needs under 100 KB: two CTAs per SM.
template <int VD>
struct FwdSmem {
    static constexpr size_t kQt = 0;                       // 128 x 128 bf16 (q / C), then y staging
    static constexpr size_t kKt = kQt + kQ * kKD * 2;      // 128 x 128 (k / B), then diag(w) K
    static constexpr size_t kVt = kKt + kQ * kKD * 2;      // 128 x VD (v / x)
    static constexpr size_t kSt = kVt + kQ * VD * 2;       // KD x VD (S_in bf16)
    static constexpr size_t kL2 = kSt + kKD * VD * 2;      // l * log2e [128]
    static constexpr size_t kBeta = kL2 + kQ * 4;          // beta [128]
    static constexpr size_t kTmp = kBeta + kQ * 4;         // scan scratch, misc
    static constexpr size_t kBar = kTmp + 64;              // mbarriers
    static constexpr size_t kTmem = kBar + 64;             // TMEM base address
    static constexpr size_t kEnd = kTmem + 64;
    static constexpr size_t kAlloc = kEnd + 1024;          // + alignment slack
    static constexpr uint32_t kTmemCols = VD <= 64 ? 256 : 512;
    static constexpr int kMinBlocks = VD <= 64 ? 2 : 1;
    static_assert(kAlloc <= 232448, "forward tile exceeds the shared memory of one CTA");
};

// TMEM columns of the forward tile: Q K^T (f32, 128 columns), overwritten in place by P (bf16
// pairs, 64 columns) and later by Y2; Y; Sl.
constexpr uint32_t kColS1 = 0;
constexpr uint32_t kColY = 128;
template <int VD> constexpr uint32_t col_sl() { return 128 + VD; }

template <int VD>
__global__ void __launch_bounds__(kThreads, FwdSmem<VD>::kMinBlocks)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                 const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mY,
                 ChunkArgs a) {
    using SM = FwdSmem<VD>;
    constexpr uint32_t kColSl = col_sl<VD>();
    char* sm = smem_base1024();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::kBar);  // 0 load, 1 G1, 2 G2, 3 G4, 4 G3
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmem);
    float* l2 = reinterpret_cast<float*>(sm + SM::kL2);
    float* betas = reinterpret_cast<float*>(sm + SM::kBeta);
    float* tmp = reinterpret_cast<float*>(sm + SM::kTmp);
    int* misc = reinterpret_cast<int*>(sm + SM::kTmp + 32);
    const uint32_t sQ = smem_u32(sm + SM::kQt), sK = smem_u32(sm + SM::kKt), sV = smem_u32(sm + SM::kVt),
                   sS = smem_u32(sm + SM::kSt);
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    if (tid == 0) {
        const unsigned int tk = take_ticket(a.hdr, 0);
        const int per = a.B * a.H;
        misc[0] = tk / per;           // chunk
        misc[1] = (tk % per) / a.H;   // batch row
        misc[2] = tk % a.H;           // head
        for (int i = 0; i < 6; ++i) mbar_init(&bar[i], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, SM::kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int c = misc[0], b = misc[1], h = misc[2];
    const int t0 = c * kQ;
    const int qk_head = a.kind == LR_SSD ? h / (a.H / a.G) : h;
    const size_t tile = ((size_t)b * a.H + h) * a.nchunk + c;  // record index of this tile

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], (uint32_t)(2 * kQ * kKD * 2 + kQ * VD * 2));
        for (int j = 0; j < kKD / 64; ++j) {
            tma_load_4d(sm + SM::kQt + j * kQ * 128, &mQ, &bar[0], 64 * j, qk_head, t0, b);
            tma_load_4d(sm + SM::kKt + j * kQ * 128, &mK, &bar[0], 64 * j, qk_head, t0, b);
        }
        for (int j = 0; j < VD / 64; ++j) tma_load_4d(sm + SM::kVt + j * kQ * 128, &mV, &bar[0], 64 * j, h, t0, b);
    }
    // decays of this chunk: l_t inclusive cumulative log decay, beta_t
    float lam, beta;
    step_coef(a, b, h, t0 + tid, lam, beta);
    const float lt = cta_inclusive_sum(lam, tmp);
    l2[tid] = lt * kLog2e;
    betas[tid] = beta;
    __syncthreads();
    const float lQ2 = l2[kQ - 1];  // l_Q log2e

    bool ok = mbar_wait(&bar[0], 0, a.hdr, 500);
    if (tid == 0 && ok) {  // G1: Q K^T
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kColS1, sQ, 0, kQ, sK, 0, kQ, kQ, kQ, kKD, 0);
        tc::commit(&bar[1]);
    }
    __syncwarp();
    ok = ok && mbar_wait(&bar[1], 0, a.hdr, 501);
    tc::fence_after_sync();
    {
        // P[t, s] = Sqk[t, s] e^{l_t - l_s} beta_s (s <= t) as bf16 pairs, written over the Sqk
        // columns it has already read (32 f32 columns in, 16 packed columns out, lower addresses)
        const int t = tid;
        const float lt2 = l2[t];
#pragma unroll 1
        for (int s0 = 0; s0 < kQ; s0 += 32) {
            uint32_t pk[16];
            if (s0 > warp * 32 + 31) {  // every row of this warp is above the diagonal block
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = 0u;
                tc::st16(tmem + kColS1 + lane_off + (s0 >> 1), pk);
                continue;
            }
            float v[32];
            tc::ld16(tmem + kColS1 + lane_off + s0, v);
            tc::ld16(tmem + kColS1 + lane_off + s0 + 16, v + 16);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s = s0 + 2 * i;
                const float p0 = (s <= t) ? v[2 * i] * ex2(lt2 - l2[s]) * betas[s] : 0.0f;
                const float p1 = (s + 1 <= t) ? v[2 * i + 1] * ex2(lt2 - l2[s + 1]) * betas[s + 1] : 0.0f;
                __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                pk[i] = *reinterpret_cast<uint32_t*>(&pr);
            }
            tc::st16(tmem + kColS1 + lane_off + (s0 >> 1), pk);
        }
        tc::wait_st();
        // K rows scaled by w_s = e^{l_Q - l_s} beta_s (the A operand of G4); G1 is complete
        scale_row(sm + SM::kKt, t, kKD, kQ, ex2(lQ2 - l2[t]) * betas[t]);
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        tc::fence_after_sync();
        tc::mma_ts_tiles(tmem + kColY, tmem + kColS1, sV, 1, kQ, VD, kQ, 0);  // G2: Y = P V
        tc::commit(&bar[2]);
        tc::mma_tiles(tmem + kColSl, sK, 1, kQ, sV, 1, kQ, kKD, VD, kQ, 0);   // G4: Sl = (w K)^T V
        tc::commit(&bar[3]);
    }
    __syncwarp();
    ok = ok && mbar_wait(&bar[3], 0, a.hdr, 502);
    tc::fence_after_sync();

    // publish the aggregate (e^{l_Q}, Sl) of this chunk
    const int kd = tid;  // state row / TMEM lane
    const bool has_succ = c + 1 < a.nchunk;
    float* myagg = a.agg + tile * kKD * VD + (size_t)kd * VD;
    if (c > 0 && has_succ) {
        for (int v0 = 0; v0 < VD; v0 += 16) {
            float v[16];
            tc::ld16(tmem + kColSl + lane_off + v0, v);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                __stcg(reinterpret_cast<float4*>(myagg + v0 + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
        }
        if (tid == 0) __stcg(&a.aggA[tile], ex2(lQ2));
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release(&a.flags[tile], kFlagAgg);
    }

    // look-back: state entering this chunk (row kd), deterministic fold in chain order
    const size_t row0 = ((size_t)b * a.H + h) * a.nchunk;
    const int j = find_prefix(a.flags + row0, c, -1, a.nchunk, a.hdr, 503);
    // j: nearest earlier chunk with a published inclusive state (checkpoint slot j + 1), or -1.
    // For every 16 columns: fold (prefix, aggregates j+1 .. c-1) into the entering state S_in
    // (checkpoint slot c, written by the predecessor as its inclusive state; chunk 0 writes the
    // zero slot), its bf16 copy (MN-major B of G3), and the inclusive state
    // S_out = e^{l_Q} S_in + Sl into slot c + 1.
    float* ck_in = a.ckpt + ((((size_t)c * a.B + b) * a.H + h) * kKD + kd) * VD;
    float* ck_out = a.ckpt + ((((size_t)(c + 1) * a.B + b) * a.H + h) * kKD + kd) * VD;
    const float* pre_row = j >= 0 ? a.ckpt + ((((size_t)(j + 1) * a.B + b) * a.H + h) * kKD + kd) * VD : nullptr;
    const float aq = ex2(lQ2);
    char* St = sm + SM::kSt;
#pragma unroll 1
    for (int v0 = 0; v0 < VD; v0 += 16) {
        float x[16];
        fold_chain(x, pre_row ? pre_row + v0 : nullptr, a.agg + (size_t)kd * VD + v0, (size_t)kKD * VD,
                   a.aggA, row0, j + 1, c, +1);
        if (c == 0) {  // slot 0 (zero state); later slots are written by the predecessor
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(ck_in + v0 + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        }
        __align__(16) __nv_bfloat16 pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = __float2bfloat16_rn(x[i]);
        *reinterpret_cast<uint4*>(St + tc::sw128_off(kd, v0, kKD)) = *reinterpret_cast<uint4*>(&pk[0]);
        *reinterpret_cast<uint4*>(St + tc::sw128_off(kd, v0 + 8, kKD)) = *reinterpret_cast<uint4*>(&pk[8]);
        if (has_succ) {
            float v[16];
            tc::ld16(tmem + kColSl + lane_off + v0, v);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                __stcg(reinterpret_cast<float4*>(ck_out + v0 + i),
                       make_float4(fmaf(aq, x[i], v[i]), fmaf(aq, x[i + 1], v[i + 1]), fmaf(aq, x[i + 2], v[i + 2]),
                                   fmaf(aq, x[i + 3], v[i + 3])));
        }
    }
    const bool withhold = (a.dflags & LR_TEST_WITHHOLD_CARRY) && c == 0;
    if (has_succ) __threadfence();
    ok = ok && mbar_wait(&bar[2], 0, a.hdr, 504);  // G2 done: P's columns can take Y2
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && has_succ && !withhold) st_release(&a.flags[tile], kFlagPrefix);
    if (tid == 0 && ok && c > 0) {  // G3: Y2 = Q S_in (in the Sqk / P columns)
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kColS1, sQ, 0, kQ, sS, 1, kKD, kQ, VD, kKD, 0);
        tc::commit(&bar[4]);
    }
    __syncwarp();
    if (c > 0) ok = ok && mbar_wait(&bar[4], 0, a.hdr, 505);
    tc::fence_after_sync();

    // output rows: y_t = Y_t + e^{l_t} Y2_t (+ D x_t), staged in the Q tile (G3 is complete)
    {
        const int t = tid;
        const float Et = ex2(l2[t]);
        const float Dh = (a.kind == LR_SSD && a.Dskip) ? a.Dskip[h] : 0.0f;
        char* Yo = sm + SM::kQt;
        const char* V = sm + SM::kVt;
        for (int v0 = 0; v0 < VD; v0 += 16) {
            float y1[16], y2[16];
            tc::ld16(tmem + kColY + lane_off + v0, y1);
            if (c > 0) tc::ld16(tmem + kColS1 + lane_off + v0, y2);
            tc::wait_ld();
            __align__(16) __nv_bfloat16 pk[16];
#pragma unroll
            for (int i = 0; i < 16; i += 8) {
                uint4 raw = *reinterpret_cast<const uint4*>(V + tc::sw128_off(t, v0 + i, kQ));
                const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float yv = y1[i + e] + (c > 0 ? Et * y2[i + e] : 0.0f);
                    yv = fmaf(Dh, __bfloat162float(xv[e]), yv);
                    pk[i + e] = __float2bfloat16_rn(yv);
                }
            }
            *reinterpret_cast<uint4*>(Yo + tc::sw128_off(t, v0, kQ)) = *reinterpret_cast<uint4*>(&pk[0]);
            *reinterpret_cast<uint4*>(Yo + tc::sw128_off(t, v0 + 8, kQ)) = *reinterpret_cast<uint4*>(&pk[8]);
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        for (int jj = 0; jj < VD / 64; ++jj) tma_store_4d(&mY, sm + SM::kQt + jj * kQ * 128, 64 * jj, h, t0, b);
        bulk_commit();
        bulk_wait_read_all();
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, SM::kTmemCols);
    }
}

// ------------------------------------------------------------------------------ host side
struct ChunkWs {
    size_t flags, agg, aggA, end;
};

ChunkWs ws_plan(const lr_desc& d) {
    const size_t tiles = (size_t)d.B * d.H * ((d.L + kQ - 1) / kQ);
    const size_t VD = (size_t)d.P;
    WsCursor c;
    ChunkWs w;
    w.flags = c.take(sizeof(unsigned int) * tiles);
    w.aggA = c.take(sizeof(float) * tiles);
    w.agg = c.take(sizeof(float) * tiles * kKD * VD);
    w.end = c.off;
    return w;
}

}  // namespace

bool chunk_supported(const lr_desc& d) {
    if (d.io != LR_BF16) return false;
    if (d.N != kKD || (d.P != 64 && d.P != 128)) return false;
    if (d.segment != kQ || (d.chunk != 0 && d.chunk != kQ)) return false;
    if (d.kind == LR_SSD && (d.disc != LR_DISC_ZOH || (d.flags & LR_HAS_Z) || d.P != 64)) return false;
    return d.L <= (1 << 28) && d.H <= 4096;
}

size_t chunk_bwd_ws_end(const lr_desc& d, bool flags_only);
size_t chunk_ws_bytes(const lr_desc& d, bool bwd) {
    if (d.kind == LR_SSD) return bwd ? ssd_bwd_ws_bytes(d) : ssd_fwd_ws_bytes(d);
    if (d.kind == LR_GLA) return gla_ws_bytes(d, bwd);
    return bwd ? chunk_bwd_ws_end(d, false) : ws_plan(d).end;
}
size_t chunk_flag_bytes(const lr_desc& d, bool bwd) {
    if (d.kind == LR_SSD) return bwd ? ssd_bwd_flag_bytes(d) : ssd_fwd_flag_bytes(d);
    if (d.kind == LR_GLA) return gla_flag_bytes(d, bwd);
    return bwd ? chunk_bwd_ws_end(d, true) : ws_plan(d).aggA;
}

lr_status chunk_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                    cudaStream_t st) {
    if (d.kind == LR_SSD) return ssd_fwd(d, in, y, ckpt, ws, st);
    if (d.kind == LR_GLA) return gla_fwd(d, in, y, ckpt, ws, st);
    ChunkWs w = ws_plan(d);
    ChunkArgs a{};
    a.kind = d.kind;
    a.B = (int)d.B;
    a.L = (int)d.L;
    a.H = (int)d.H;
    a.G = d.kind == LR_SSD ? (int)d.G : (int)d.H;
    a.nchunk = (int)((d.L + kQ - 1) / kQ);
    a.VD = (int)d.P;
    a.lam = (const __nv_bfloat16*)(d.kind == LR_SSD ? in.delta : in.g);
    a.A = in.A;
    a.Dskip = (d.kind == LR_SSD && (d.flags & LR_HAS_DSKIP)) ? in.Dskip : nullptr;
    a.ckpt = (float*)ckpt;
    a.hdr = (WsHeader*)ws;
    a.flags = (unsigned int*)(ws + w.flags);
    a.agg = (float*)(ws + w.agg);
    a.aggA = (float*)(ws + w.aggA);
    a.dflags = d.flags;
    CUtensorMap mQ, mK, mV, mY;
    const void* q = d.kind == LR_SSD ? in.Cm : in.q;
    const void* k = d.kind == LR_SSD ? in.Bm : in.k;
    const void* v = d.kind == LR_SSD ? in.x : in.v;
    const uint64_t QX = d.kind == LR_SSD ? (uint64_t)d.G : (uint64_t)d.H;
    bool ok = map4(&mQ, q, kKD, QX, d.L, d.B, true) && map4(&mK, k, kKD, QX, d.L, d.B, true) &&
              map4(&mV, v, d.P, d.H, d.L, d.B, true) && map4(&mY, y, d.P, d.H, d.L, d.B, true);
    if (!ok) return LR_ERR_INVALID_ARG;
    const int grid = a.B * a.H * a.nchunk;
    if (d.P == 64) {
        using SM = FwdSmem<64>;
        cudaFuncSetAttribute(chunk_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
        note_launch(d.kind == LR_SSD ? "ssd_fwd_chunk" : "gla_fwd_chunk");
        chunk_fwd_kernel<64><<<grid, kThreads, SM::kAlloc, st>>>(mQ, mK, mV, mY, a);
    } else {
        using SM = FwdSmem<128>;
        cudaFuncSetAttribute(chunk_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
        note_launch(d.kind == LR_SSD ? "ssd_fwd_chunk" : "gla_fwd_chunk");
        chunk_fwd_kernel<128><<<grid, kThreads, SM::kAlloc, st>>>(mQ, mK, mV, mY, a);
    }
    return check_launch();
}

// =========================================================================================
// Backward.  Tile = (batch row, head, chunk), chunks taken in reverse order.  With the chunk's
// entering state S_in (checkpoint slot c), its inclusive state S_out (slot c + 1), the upstream
// gradient dO and the adjoint dS_out of S_out, the chunk's gradients are (l: chunk-local
// cumulative log decay, E_t = e^{l_t}, W_s = e^{l_Q - l_s}, a = e^{l_Q}):
//   dq  = Pd K + diag(E) dO S_in^T            Pd[t,s] = (dO V^T)[t,s] e^{l_t - l_s} beta_s, s <= t
//   dk  = Pd^T Q + diag(W beta) V dS_out^T
//   dv  = P^T dO + diag(W beta) K dS_out       P[t,s]  = (Q K^T)[t,s] e^{l_t - l_s} beta_s, s <= t
//   dS_in = a dS_out + Q^T diag(E) dO         (the adjoint handed to the previous chunk)
//   dl_t  = q_t . dq_t - k_t . dk_t  (+ <dS_out, S_out> at the chunk's last step)
//   d lam_r = sum_{t >= r} dl_t ;   d beta_s = k_s . dk_s / beta_s
// (gla: dg = d lam / g; ssd: d dt = d lam A + d beta abar, dA = sum(d lam dt + d beta
// (dt abar - beta) / A), dx = dv + D dy, dB / dC = sums of dk / dq over the heads of a group.)
// The adjoint carry dS_out comes from a reverse decoupled look-back over per-chunk records
// (aggregate (a, Q^T diag(E) dO), inclusive dS_in), folded in chain order.
// =========================================================================================
namespace {

template <int VD>
struct BwdSmem {
    static constexpr size_t kQt = 0;                      // Q (never scaled); dq staging at the end
    static constexpr size_t kKt = kQt + kQ * kKD * 2;     // K, then diag(W beta) K; dk staging
    static constexpr size_t kVt = kKt + kQ * kKD * 2;     // V, then diag(W beta) V; dv / dx staging
    static constexpr size_t kOt = kVt + kQ * VD * 2;      // dO, then diag(E) dO
    static constexpr size_t kPt = kOt + kQ * VD * 2;      // P, then dS_out (bf16, KD x VD)
    static constexpr size_t kPdt = kPt + kQ * kQ * 2;     // Pd, then S_in (bf16, KD x VD)
    static constexpr size_t kYt = kPdt + kQ * kQ * 2;     // dy, unscaled (ssd, V = 64: dx = dv + D dy)
    static constexpr size_t kL2 = kYt + (VD <= 64 ? kQ * VD * 2 : 0);  // l log2e [128]
    static constexpr size_t kBeta = kL2 + kQ * 4;         // beta [128]
    static constexpr size_t kLam = kBeta + kQ * 4;        // raw per-step input (dt or g) [128]
    static constexpr size_t kRed = kLam + kQ * 4;         // reduction scratch [128]
    static constexpr size_t kTmp = kRed + kQ * 4;         // scan scratch, misc
    static constexpr size_t kBar = kTmp + 64;
    static constexpr size_t kTmem = kBar + 64;
    static constexpr size_t kEnd = kTmem + 64;
    static constexpr size_t kAlloc = kEnd + 1024;
    static_assert(kAlloc <= 232448, "backward tile exceeds the shared memory of one CTA");
};

constexpr uint32_t kR0 = 0, kR1 = 128, kR2 = 256, kR3 = 384;

struct ChunkBwdArgs {
    ChunkArgs f;              // shapes, decays, checkpoints (read), header
    const __nv_bfloat16* kg;  // k (GLA) / B (SSD) in global memory, for the k . dk row dots
    const __nv_bfloat16* dy;  // upstream gradient [B, L, H, VD]
    __nv_bfloat16* dlam;      // GLA dg / SSD ddt [B, L, H]
    float* dBm;               // SSD [B, L, G, N] (accumulated over heads)
    float* dCm;
    unsigned int* flags;      // reverse-chain records
    float* agg;
    float* aggA;
    float* pre;
    float* pdA;               // SSD per-tile partials
    float* pdD;
};

template <int VD>
__global__ void __launch_bounds__(kThreads, 1)
chunk_bwd_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                 const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mO,
                 const __grid_constant__ CUtensorMap mdQ, const __grid_constant__ CUtensorMap mdK,
                 const __grid_constant__ CUtensorMap mdV, ChunkBwdArgs bw) {
    using SM = BwdSmem<VD>;
    const ChunkArgs& a = bw.f;
    char* sm = smem_base1024();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::kBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmem);
    float* l2 = reinterpret_cast<float*>(sm + SM::kL2);
    float* betas = reinterpret_cast<float*>(sm + SM::kBeta);
    float* red = reinterpret_cast<float*>(sm + SM::kRed);
    float* tmp = reinterpret_cast<float*>(sm + SM::kTmp);
    int* misc = reinterpret_cast<int*>(sm + SM::kTmp + 32);
    const uint32_t sQ = smem_u32(sm + SM::kQt), sK = smem_u32(sm + SM::kKt), sV = smem_u32(sm + SM::kVt),
                   sO = smem_u32(sm + SM::kOt), sP = smem_u32(sm + SM::kPt), sPd = smem_u32(sm + SM::kPdt);
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const bool ssd = a.kind == LR_SSD;
    const uint32_t colDv = kR1, colDSl = ssd ? kR1 + 64 : kR0;

    if (tid == 0) {
        // Tiles are numbered along diagonals key = (nchunk - 1 - c) + h, so that tiles running at
        // the same time sit at different chunks of different heads (SSD's dB / dC sums over heads
        // then do not collide), while every tile's reverse-chain dependency (c + 1, key - 1) has
        // a smaller number.
        unsigned int tk = take_ticket(a.hdr, 1);
        int key = 0, lo = 0, n = 0;
        for (;; ++key) {
            lo = max(0, key - (a.nchunk - 1));
            const int hi = min(a.H - 1, key);
            n = hi - lo + 1;
            if (tk < (unsigned int)(a.B * n)) break;
            tk -= a.B * n;
        }
        const int hh = lo + (int)(tk % n);
        misc[0] = a.nchunk - 1 - (key - hh);
        misc[1] = (int)(tk / n);
        misc[2] = hh;
        for (int i = 0; i < 6; ++i) mbar_init(&bar[i], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int c = misc[0], b = misc[1], h = misc[2];
    const int t0 = c * kQ;
    const int gq = ssd ? h / (a.H / a.G) : h;
    const size_t row0 = ((size_t)b * a.H + h) * a.nchunk;
    const size_t tile = row0 + c;
    const bool last = c + 1 >= a.nchunk;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], (uint32_t)(2 * kQ * kKD * 2 + (ssd ? 3 : 2) * kQ * VD * 2));
        for (int j = 0; j < kKD / 64; ++j) {
            tma_load_4d(sm + SM::kQt + j * kQ * 128, &mQ, &bar[0], 64 * j, gq, t0, b);
            tma_load_4d(sm + SM::kKt + j * kQ * 128, &mK, &bar[0], 64 * j, gq, t0, b);
        }
        for (int j = 0; j < VD / 64; ++j) {
            tma_load_4d(sm + SM::kVt + j * kQ * 128, &mV, &bar[0], 64 * j, h, t0, b);
            tma_load_4d(sm + SM::kOt + j * kQ * 128, &mO, &bar[0], 64 * j, h, t0, b);
            if (ssd) tma_load_4d(sm + SM::kYt + j * kQ * 128, &mO, &bar[0], 64 * j, h, t0, b);
        }
    }
    const int r = tid;  // this thread's row (time step in the chunk, or state row kd)
    const int tr = t0 + r;
    float lam, beta;
    step_coef(a, b, h, tr, lam, beta);
    const float lt = cta_inclusive_sum(lam, tmp);
    l2[r] = lt * kLog2e;
    betas[r] = beta;
    __syncthreads();
    const float lQ2 = l2[kQ - 1];

    bool ok = mbar_wait(&bar[0], 0, a.hdr, 600);
    if (tid == 0 && ok) {
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kR0, sQ, 0, kQ, sK, 0, kQ, kQ, kQ, kKD, 0);  // Q K^T
        tc::mma_tiles(tmem + kR1, sO, 0, kQ, sV, 0, kQ, kQ, kQ, VD, 0);   // dO V^T
        tc::commit(&bar[1]);
    }
    __syncwarp();
    ok = ok && mbar_wait(&bar[1], 0, a.hdr, 601);
    tc::fence_after_sync();
    {  // P and Pd (bf16), row r
        const float lr2 = l2[r];
        char* P = sm + SM::kPt;
        char* Pd = sm + SM::kPdt;
        for (int s0 = 0; s0 < kQ; s0 += 16) {
            float qk[16], dv[16];
            tc::ld16(tmem + kR0 + lane_off + s0, qk);
            tc::ld16(tmem + kR1 + lane_off + s0, dv);
            tc::wait_ld();
            __align__(16) __nv_bfloat16 pk[16], pd[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s = s0 + i;
                const float f = (s <= r) ? ex2(lr2 - l2[s]) * betas[s] : 0.0f;
                pk[i] = __float2bfloat16_rn(qk[i] * f);
                pd[i] = __float2bfloat16_rn(dv[i] * f);
            }
            *reinterpret_cast<uint4*>(P + tc::sw128_off(r, s0, kQ)) = *reinterpret_cast<uint4*>(&pk[0]);
            *reinterpret_cast<uint4*>(P + tc::sw128_off(r, s0 + 8, kQ)) = *reinterpret_cast<uint4*>(&pk[8]);
            *reinterpret_cast<uint4*>(Pd + tc::sw128_off(r, s0, kQ)) = *reinterpret_cast<uint4*>(&pd[0]);
            *reinterpret_cast<uint4*>(Pd + tc::sw128_off(r, s0 + 8, kQ)) = *reinterpret_cast<uint4*>(&pd[8]);
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kR2, sPd, 0, kQ, sK, 1, kQ, kQ, kKD, kQ, 0);  // dq  = Pd K
        tc::mma_tiles(tmem + kR3, sPd, 1, kQ, sQ, 1, kQ, kQ, kKD, kQ, 0);  // dk  = Pd^T Q
        tc::mma_tiles(tmem + colDv, sP, 1, kQ, sO, 1, kQ, kQ, VD, kQ, 0);  // dv  = P^T dO
        tc::commit(&bar[2]);
    }
    __syncwarp();
    ok = ok && mbar_wait(&bar[2], 0, a.hdr, 602);
    float dD_part = 0.0f;
    {
        // D-skip gradient part (ssd): sum_v dy x of row r, before V is rescaled
        char* V = sm + SM::kVt;
        char* O = sm + SM::kOt;
        if (ssd) {
            for (int v0 = 0; v0 < VD; v0 += 8) {
                uint4 xr = *reinterpret_cast<const uint4*>(V + tc::sw128_off(r, v0, kQ));
                uint4 orw = *reinterpret_cast<const uint4*>(O + tc::sw128_off(r, v0, kQ));
                const __nv_bfloat16* xv = reinterpret_cast<const __nv_bfloat16*>(&xr);
                const __nv_bfloat16* ov = reinterpret_cast<const __nv_bfloat16*>(&orw);
#pragma unroll
                for (int e = 0; e < 8; ++e) dD_part = fmaf(__bfloat162float(xv[e]), __bfloat162float(ov[e]), dD_part);
            }
        }
        const float E = ex2(l2[r]);
        const float wb = ex2(lQ2 - l2[r]) * betas[r];
        scale_row(O, r, VD, kQ, E);                   // diag(E) dO
        scale_row(V, r, VD, kQ, wb);                  // diag(W beta) V
        // S_in (checkpoint slot c) as bf16, rows kd x cols v, in the Pd region
        const float* sin = a.ckpt + ((((size_t)c * a.B + b) * a.H + h) * kKD + r) * VD;
        char* St = sm + SM::kPdt;
        for (int v0 = 0; v0 < VD; v0 += 8) {
            const float4 f0 = __ldcg(reinterpret_cast<const float4*>(sin + v0));
            const float4 f1 = __ldcg(reinterpret_cast<const float4*>(sin + v0 + 4));
            __align__(16) __nv_bfloat162 pk[4] = {__floats2bfloat162_rn(f0.x, f0.y), __floats2bfloat162_rn(f0.z, f0.w),
                                                  __floats2bfloat162_rn(f1.x, f1.y), __floats2bfloat162_rn(f1.z, f1.w)};
            *reinterpret_cast<uint4*>(St + tc::sw128_off(r, v0, kKD)) = *reinterpret_cast<uint4*>(pk);
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kR2, sO, 0, kQ, sPd, 0, kKD, kQ, kKD, VD, 1);   // dq += diag(E) dO S_in^T
        tc::mma_tiles(tmem + colDSl, sQ, 1, kQ, sO, 1, kQ, kKD, VD, kQ, 0);  // dSl = Q^T diag(E) dO
        tc::commit(&bar[3]);
    }
    __syncwarp();
    ok = ok && mbar_wait(&bar[3], 0, a.hdr, 603);
    tc::fence_after_sync();

    // reverse chain: aggregate (a, dSl) of this chunk
    const float aq = ex2(lQ2);
    float* myagg = bw.agg + tile * kKD * VD + (size_t)r * VD;
    if (c > 0 && !last) {
        for (int v0 = 0; v0 < VD; v0 += 16) {
            float v[16];
            tc::ld16(tmem + colDSl + lane_off + v0, v);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                __stcg(reinterpret_cast<float4*>(myagg + v0 + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
        }
        if (tid == 0) __stcg(&bw.aggA[tile], aq);
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release(&bw.flags[tile], kFlagAgg);
    }
    // dS_out: nearest later chunk with an inclusive adjoint, then the fold in chain order
    const int j = find_prefix(bw.flags + row0, c, +1, a.nchunk, a.hdr, 604);
    float xdot = 0.0f;  // <dS_out, S_out> restricted to row r
    float* mypre = bw.pre + tile * kKD * VD + (size_t)r * VD;
    char* dSt = sm + SM::kPt;
    const float* sout = a.ckpt + ((((size_t)(c + 1) * a.B + b) * a.H + h) * kKD + r) * VD;
    const float* pre_row = j < a.nchunk ? bw.pre + (row0 + j) * kKD * VD + (size_t)r * VD : nullptr;
#pragma unroll 1
    for (int v0 = 0; v0 < VD; v0 += 16) {
        float4 so[4];
        if (!last) {
#pragma unroll
            for (int e = 0; e < 4; ++e) so[e] = __ldcg(reinterpret_cast<const float4*>(sout + v0) + e);
        }
        float x[16];
        fold_chain(x, pre_row ? pre_row + v0 : nullptr, bw.agg + (size_t)r * VD + v0, (size_t)kKD * VD, bw.aggA,
                   row0, j - 1, c, -1);
        if (!last) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                xdot = fmaf(x[4 * e], so[e].x, fmaf(x[4 * e + 1], so[e].y, fmaf(x[4 * e + 2], so[e].z, fmaf(x[4 * e + 3], so[e].w, xdot))));
        }
        __align__(16) __nv_bfloat16 pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = __float2bfloat16_rn(x[i]);
        *reinterpret_cast<uint4*>(dSt + tc::sw128_off(r, v0, kKD)) = *reinterpret_cast<uint4*>(&pk[0]);
        *reinterpret_cast<uint4*>(dSt + tc::sw128_off(r, v0 + 8, kKD)) = *reinterpret_cast<uint4*>(&pk[8]);
        if (c > 0) {  // inclusive adjoint handed to chunk c - 1: a dS_out + dSl
            float v[16];
            tc::ld16(tmem + colDSl + lane_off + v0, v);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                __stcg(reinterpret_cast<float4*>(mypre + v0 + i),
                       make_float4(fmaf(aq, x[i], v[i]), fmaf(aq, x[i + 1], v[i + 1]), fmaf(aq, x[i + 2], v[i + 2]),
                                   fmaf(aq, x[i + 3], v[i + 3])));
        }
    }
    const bool withhold = (a.dflags & LR_TEST_WITHHOLD_CARRY) && last;
    if (c > 0) {
        __threadfence();
        __syncthreads();
        if (tid == 0 && !withhold) st_release(&bw.flags[tile], kFlagPrefix);
    }
    red[r] = xdot;
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok && !last) {
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kR3, sV, 0, kQ, sP, 0, kKD, kQ, kKD, VD, 1);     // dk += diag(W b) V dS_out^T
        tc::mma_tiles(tmem + colDSl, sK, 0, kQ, sP, 1, kKD, kQ, VD, kKD, 0);  // K dS_out (dSl is consumed)
        tc::commit(&bar[4]);
    }
    __syncwarp();
    if (!last) ok = ok && mbar_wait(&bar[4], 0, a.hdr, 605);
    tc::fence_after_sync();
    float X = 0.0f;  // <dS_out, S_out>
    for (int i = 0; i < kQ; ++i) X += red[i];

    // final epilogue, row r: dq, dk, dv (dx), dl
    const bool valid = tr < a.L;
    float qdq = 0.0f, kdk = 0.0f;
    {
        char* Q = sm + SM::kQt;
        char* K = sm + SM::kKt;
        for (int k0 = 0; k0 < kKD; k0 += 16) {
            float dq[16], dk[16];
            tc::ld16(tmem + kR2 + lane_off + k0, dq);
            tc::ld16(tmem + kR3 + lane_off + k0, dk);
            tc::wait_ld();
            __align__(16) __nv_bfloat16 oq[16], ok2[16];
#pragma unroll
            for (int i = 0; i < 16; i += 8) {
                uint4 qr = *reinterpret_cast<const uint4*>(Q + tc::sw128_off(r, k0 + i, kQ));
                uint4 kr = *reinterpret_cast<const uint4*>(K + tc::sw128_off(r, k0 + i, kQ));
                const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(&qr);
                const __nv_bfloat16* kv = reinterpret_cast<const __nv_bfloat16*>(&kr);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    qdq = fmaf(__bfloat162float(qv[e]), dq[i + e], qdq);
                    kdk = fmaf(__bfloat162float(kv[e]), dk[i + e], kdk);
                    oq[i + e] = __float2bfloat16_rn(dq[i + e]);
                    ok2[i + e] = __float2bfloat16_rn(dk[i + e]);
                }
            }
            if (ssd) {
                if (valid) {
                    float* dC = bw.dCm + (((size_t)b * a.L + tr) * a.G + gq) * kKD + k0;
                    float* dB = bw.dBm + (((size_t)b * a.L + tr) * a.G + gq) * kKD + k0;
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        red_add4(dC + i, dq[i], dq[i + 1], dq[i + 2], dq[i + 3]);
                        red_add4(dB + i, dk[i], dk[i + 1], dk[i + 2], dk[i + 3]);
                    }
                }
            } else {
                *reinterpret_cast<uint4*>(Q + tc::sw128_off(r, k0, kQ)) = *reinterpret_cast<uint4*>(&oq[0]);
                *reinterpret_cast<uint4*>(Q + tc::sw128_off(r, k0 + 8, kQ)) = *reinterpret_cast<uint4*>(&oq[8]);
                *reinterpret_cast<uint4*>(K + tc::sw128_off(r, k0, kQ)) = *reinterpret_cast<uint4*>(&ok2[0]);
                *reinterpret_cast<uint4*>(K + tc::sw128_off(r, k0 + 8, kQ)) = *reinterpret_cast<uint4*>(&ok2[8]);
            }
        }
        // dv (gla) / dx = dv + D dy (ssd) into the V region
        char* V = sm + SM::kVt;
        const float Dh = (ssd && a.Dskip) ? a.Dskip[h] : 0.0f;
        const char* Yt = sm + SM::kYt;
        const float wbr = ex2(lQ2 - l2[r]) * betas[r];
        for (int v0 = 0; v0 < VD; v0 += 16) {
            float dv[16], dvi[16];
            tc::ld16(tmem + colDv + lane_off + v0, dv);
            if (!last) tc::ld16(tmem + colDSl + lane_off + v0, dvi);
            tc::wait_ld();
            if (!last) {
#pragma unroll
                for (int i = 0; i < 16; ++i) dv[i] = fmaf(wbr, dvi[i], dv[i]);
            }
            __align__(16) __nv_bfloat16 o[16];
#pragma unroll
            for (int i = 0; i < 16; i += 8) {
                uint4 yr = ssd ? *reinterpret_cast<const uint4*>(Yt + tc::sw128_off(r, v0 + i, kQ)) : make_uint4(0, 0, 0, 0);
                const __nv_bfloat16* yv = reinterpret_cast<const __nv_bfloat16*>(&yr);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[i + e] = __float2bfloat16_rn(fmaf(Dh, __bfloat162float(yv[e]), dv[i + e]));
            }
            *reinterpret_cast<uint4*>(V + tc::sw128_off(r, v0, kQ)) = *reinterpret_cast<uint4*>(&o[0]);
            *reinterpret_cast<uint4*>(V + tc::sw128_off(r, v0 + 8, kQ)) = *reinterpret_cast<uint4*>(&o[8]);
        }
    }
    // decay and beta gradients
    float dl = qdq - kdk + (r == kQ - 1 ? X : 0.0f);
    if (!valid) dl = 0.0f;
    const float incl = cta_inclusive_sum(dl, tmp);
    if (tid == kQ - 1) red[0] = incl;  // total
    __syncthreads();
    const float dlam = red[0] - incl + dl;  // sum over t >= r
    float dA_part = 0.0f;
    if (valid) {
        const float raw = __bfloat162float(a.lam[((size_t)b * a.L + tr) * a.H + h]);
        float out;
        if (ssd) {
            const float Ah = a.A[h];
            const float ab = ex2(raw * Ah * kLog2e);
            const float dbeta = beta != 0.0f ? kdk / beta : 0.0f;
            out = dlam * Ah + dbeta * ab;
            dA_part = dlam * raw + dbeta * (raw * ab - beta) / Ah;
        } else {
            out = dlam / raw;
        }
        bw.dlam[((size_t)b * a.L + tr) * a.H + h] = __float2bfloat16_rn(out);
    }
    if (ssd) {  // per-tile partials of dA_h and dD_h (fixed-order sums)
        __syncthreads();
        red[r] = dA_part;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int i = 0; i < kQ; ++i) s += red[i];
            bw.pdA[tile] = s;
        }
        __syncthreads();
        red[r] = dD_part;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int i = 0; i < kQ; ++i) s += red[i];
            bw.pdD[tile] = s;
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        if (!ssd) {
            for (int jj = 0; jj < kKD / 64; ++jj) {
                tma_store_4d(&mdQ, sm + SM::kQt + jj * kQ * 128, 64 * jj, h, t0, b);
                tma_store_4d(&mdK, sm + SM::kKt + jj * kQ * 128, 64 * jj, h, t0, b);
            }
        }
        for (int jj = 0; jj < VD / 64; ++jj) tma_store_4d(&mdV, sm + SM::kVt + jj * kQ * 128, 64 * jj, h, t0, b);
        bulk_commit();
        bulk_wait_read_all();
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// Fixed-order sums of the per-tile SSD parameter partials over batch rows and chunks.
__global__ void ssd_param_reduce(const float* __restrict__ pdA, const float* __restrict__ pdD, int B, int H,
                                 int nchunk, float* __restrict__ dA, float* __restrict__ dD) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float sa = 0.0f, sd = 0.0f;
    for (int b = 0; b < B; ++b)
        for (int c = 0; c < nchunk; ++c) {
            const size_t t = ((size_t)b * H + h) * nchunk + c;
            sa += pdA[t];
            sd += pdD[t];
        }
    dA[h] = sa;
    if (dD) dD[h] = sd;
}

struct ChunkBwdWs {
    size_t flags, aggA, pdA, pdD, agg, pre, end;
};

ChunkBwdWs bwd_plan(const lr_desc& d) {
    const size_t tiles = (size_t)d.B * d.H * ((d.L + kQ - 1) / kQ);
    const size_t VD = (size_t)d.P;
    WsCursor c;
    ChunkBwdWs w;
    w.flags = c.take(sizeof(unsigned int) * tiles);
    w.aggA = c.take(sizeof(float) * tiles);
    w.pdA = c.take(sizeof(float) * tiles);
    w.pdD = c.take(sizeof(float) * tiles);
    w.agg = c.take(sizeof(float) * tiles * kKD * VD);
    w.pre = c.take(sizeof(float) * tiles * kKD * VD);
    w.end = c.off;
    return w;
}

}  // namespace

size_t chunk_bwd_ws_end(const lr_desc& d, bool flags_only) {
    ChunkBwdWs w = bwd_plan(d);
    return flags_only ? w.aggA : w.end;
}

lr_status chunk_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                    const lr_grads& gr, char* ws, cudaStream_t st) {
    if (d.kind == LR_SSD) return ssd_bwd(d, in, dy, ckpt, gr, ws, st);
    if (d.kind == LR_GLA) return gla_bwd(d, in, dy, ckpt, gr, ws, st);
    ChunkBwdWs w = bwd_plan(d);
    ChunkBwdArgs bw{};
    ChunkArgs& a = bw.f;
    a.kind = d.kind;
    a.B = (int)d.B;
    a.L = (int)d.L;
    a.H = (int)d.H;
    a.G = d.kind == LR_SSD ? (int)d.G : (int)d.H;
    a.nchunk = (int)((d.L + kQ - 1) / kQ);
    a.VD = (int)d.P;
    a.lam = (const __nv_bfloat16*)(d.kind == LR_SSD ? in.delta : in.g);
    a.A = in.A;
    a.Dskip = (d.kind == LR_SSD && (d.flags & LR_HAS_DSKIP)) ? in.Dskip : nullptr;
    a.ckpt = (float*)const_cast<void*>(ckpt);
    a.hdr = (WsHeader*)ws;
    a.dflags = d.flags;
    bw.kg = (const __nv_bfloat16*)(d.kind == LR_SSD ? in.Bm : in.k);
    bw.dy = (const __nv_bfloat16*)dy;
    bw.dlam = (__nv_bfloat16*)(d.kind == LR_SSD ? gr.ddelta : gr.dg);
    bw.dBm = gr.dBm;
    bw.dCm = gr.dCm;
    bw.flags = (unsigned int*)(ws + w.flags);
    bw.agg = (float*)(ws + w.agg);
    bw.aggA = (float*)(ws + w.aggA);
    bw.pre = (float*)(ws + w.pre);
    bw.pdA = (float*)(ws + w.pdA);
    bw.pdD = (float*)(ws + w.pdD);
    const bool ssd = d.kind == LR_SSD;
    if (ssd) {
        const size_t n = (size_t)d.B * d.L * d.G * kKD * sizeof(float);
        if (cudaMemsetAsync(gr.dBm, 0, n, st) != cudaSuccess || cudaMemsetAsync(gr.dCm, 0, n, st) != cudaSuccess)
            return LR_ERR_CUDA;
    }
    CUtensorMap mQ, mK, mV, mO, mdQ, mdK, mdV;
    const void* q = ssd ? in.Cm : in.q;
    const void* k = ssd ? in.Bm : in.k;
    const void* v = ssd ? in.x : in.v;
    const uint64_t QX = ssd ? (uint64_t)d.G : (uint64_t)d.H;
    bool okm = map4(&mQ, q, kKD, QX, d.L, d.B, true) && map4(&mK, k, kKD, QX, d.L, d.B, true) &&
               map4(&mV, v, d.P, d.H, d.L, d.B, true) && map4(&mO, dy, d.P, d.H, d.L, d.B, true) &&
               map4(&mdV, ssd ? gr.dx : gr.dv, d.P, d.H, d.L, d.B, true) &&
               map4(&mdQ, ssd ? gr.dx : gr.dq, ssd ? d.P : kKD, d.H, d.L, d.B, true) &&
               map4(&mdK, ssd ? gr.dx : gr.dk, ssd ? d.P : kKD, d.H, d.L, d.B, true);
    if (!okm) return LR_ERR_INVALID_ARG;
    const int grid = a.B * a.H * a.nchunk;
    if (d.P == 64) {
        using SM = BwdSmem<64>;
        cudaFuncSetAttribute(chunk_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
        note_launch(ssd ? "ssd_bwd_chunk" : "gla_bwd_chunk");
        chunk_bwd_kernel<64><<<grid, kThreads, SM::kAlloc, st>>>(mQ, mK, mV, mO, mdQ, mdK, mdV, bw);
    } else {
        using SM = BwdSmem<128>;
        cudaFuncSetAttribute(chunk_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
        note_launch(ssd ? "ssd_bwd_chunk" : "gla_bwd_chunk");
        chunk_bwd_kernel<128><<<grid, kThreads, SM::kAlloc, st>>>(mQ, mK, mV, mO, mdQ, mdK, mdV, bw);
    }
    lr_status s = check_launch();
    if (s != LR_OK || !ssd) return s;
    note_launch("ssd_param_reduce");
    ssd_param_reduce<<<(a.H + 127) / 128, 128, 0, st>>>(bw.pdA, bw.pdD, a.B, a.H, a.nchunk, gr.dA,
                                                         (d.flags & LR_HAS_DSKIP) ? gr.dDskip : nullptr);
    return check_launch();
}

}  // namespace lrs
