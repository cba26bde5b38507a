// gla.cu -- gated linear attention scan (gla_scan of the mlx-recurrence post: state [B, H, Dh, Dh])
// on tcgen05, one head per CTA.
//
// Recurrence per head ("mlx-recurrence", Apple Developer Forums thread 840535, "Current kernels":
// gla_scan with a scalar gate g_t per step and head):
//   S_t = g_t S_{t-1} + k_t v_t^T,  o_t = S_t^T q_t
// With 128-step chunks, lam_t = log g_t, l_t the chunk-local inclusive cumulative log decay,
// w_t = e^{l_Q - l_t}, E_t = e^{l_t}, M = Q K^T, Lmask[t, s] = e^{l_t - l_s} (s <= t):
//   S_out = e^{l_Q} S_in + Sl,  Sl = K^T diag(w) V
//   O     = (M o Lmask) V + diag(E) Q S_in
// (the chunked evaluation of the K-Search / mlx-mamba post, paragraph after Table 1, with a
// scalar decay and a matrix state).  Forward = chunk_scan_kernel (chunk_scan.cuh: one CTA per (row,
// head, 64 value columns) folding Sl = K^T diag(w) V into the entering states, checkpoints and
// bf16 tiles) and gla_out_kernel beside it.  Backward = chunk_scan_kernel in reverse (adjoint
// states G from U = Q^T diag(E) dO) and gla_grad_kernel beside it.  The chunk kernels wait for the
// scan's per-slot flags, not for the whole scan.
#include "chunk_scan.cuh"

namespace lrs {
using namespace chunkc;
namespace {

struct GlaArgs {
    int B, L, H, nchunk;
    const __nv_bfloat16* g;   // [B, L, H] gate in (0, 1)
    WsHeader* hdr;
    int withhold;             // LR_TEST_WITHHOLD_CARRY (the scan never counts slot 0)
};

// log decay of step t of head h (0 past L)
__device__ __forceinline__ float gla_lam(const GlaArgs& a, int b, int h, int t) {
    if (t >= a.L) return 0.0f;
    return __logf(__bfloat162float(a.g[((size_t)b * a.L + t) * a.H + h]));
}

// ---------------------------------------------------------------------------------- outputs
template <int VD>
struct GOutSmem {
    static constexpr size_t kQt = 0;                     // q, then diag(E) q
    static constexpr size_t kKt = kQt + kQ * kKD * 2;    // k, then the S_in tile (128 x VD bf16)
    static constexpr size_t kVt = kKt + kQ * kKD * 2;    // v, then the output rows
    static constexpr size_t kL2 = kVt + kQ * VD * 2;     // l log2e [128]
    static constexpr size_t kCf = kL2 + kQ * 4;          // column factors [4 warps][128]
    static constexpr size_t kTmp = kCf + 4 * kQ * 4;     // scan scratch
    static constexpr size_t kBar = kTmp + 64;            // 0 q/k, 1 v, 2 M, 3 S_in, 4 O
    static constexpr size_t kTmem = kBar + 64;
    static constexpr size_t kEnd = kTmem + 64;
    static constexpr size_t kAlloc = kEnd + 1024;
    static_assert(2 * (kAlloc + 1024) <= 233472, "two output CTAs per SM");
};

// One CTA per (chunk, batch row, head).  TMEM: M = Q K^T (f32, columns 0..127), rewritten in place
// as P = M o Lmask (bf16 pairs, columns 0..63); O (f32, columns 64 .. 64 + VD) accumulates
// P V (A from TMEM) and diag(E) Q S_in (q rows scaled by E in place once M is done).
template <int VD>
__global__ void __launch_bounds__(kThreads, 2)
gla_out_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
               const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mO, GlaArgs a,
               const char* stiles, const unsigned int* ready, int halves) {
    using SM = GOutSmem<VD>;
    constexpr uint32_t kColO = 64;
    char* sm = smem_base1024();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::kBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmem);
    float* l2s = reinterpret_cast<float*>(sm + SM::kL2);
    float* tmp = reinterpret_cast<float*>(sm + SM::kTmp);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float* cfw = reinterpret_cast<float*>(sm + SM::kCf) + warp * kQ;
    int idx = blockIdx.x;
    const int h = idx % a.H;
    idx /= a.H;
    const int b = idx % a.B;
    const int c = idx / a.B;
    const int t0 = c * kQ;
    const bool has_in = c > 0;
    pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(&bar[i], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0) tc::tmem_alloc(tmem_slot, 256);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], (uint32_t)(2 * kQ * kKD * 2));
        for (int j = 0; j < kKD / 64; ++j) {
            tma_load_4d(sm + SM::kQt + j * kQ * 128, &mQ, &bar[0], 64 * j, h, t0, b);
            tma_load_4d(sm + SM::kKt + j * kQ * 128, &mK, &bar[0], 64 * j, h, t0, b);
        }
        mbar_arrive_expect_tx(&bar[1], (uint32_t)(kQ * VD * 2));
        for (int j = 0; j < VD / 64; ++j) tma_load_4d(sm + SM::kVt + j * kQ * 128, &mV, &bar[1], 64 * j, h, t0, b);
    }
    // the S_in tile of slot c: written by the scan kernel, which counts each 64-column half once its
    // copies have landed; polled here by a thread with no copies in flight, so that the poll's
    // latency hides behind the loads above (slot 0, the zero state, is waited for too: the scan
    // counts it only after the kernels before it are done, and no global write of this kernel
    // comes before the barrier below)
    // (a timeout is recorded in the workspace; the kernel finishes)
    if (tid == 32) wait_count(&ready[((size_t)c * a.B + b) * a.H + h], (unsigned int)halves, a.hdr, 813);
    const float lt2 = cta_inclusive_sum(gla_lam(a, b, h, t0 + tid), tmp) * kLog2e;
    l2s[tid] = lt2;
    __syncthreads();
    const float E = ex2(lt2);
    const float l0 = l2s[32 * warp];
    for (int s = lane; s < 32 * warp; s += 32) cfw[s] = ex2(l0 - l2s[s]);
    __syncwarp();
    bool ok = mbar_wait(&bar[0], 0, a.hdr, 810);
    if (tid == 0 && ok) {
        tc::fence_after_sync();
        tc::mma_tiles(tmem, smem_u32(sm + SM::kQt), 0, kQ, smem_u32(sm + SM::kKt), 0, kQ, kQ, kQ, kKD, 0);  // Q K^T
        tc::commit(&bar[2]);
    }
    ok = ok && mbar_wait(&bar[2], 0, a.hdr, 811);
    tc::fence_after_sync();
    if (tid == 0 && ok && has_in) {  // k is consumed: its slot takes the S_in tile
        fence_proxy_async_global();  // the copy comes after the count polled above
        mbar_arrive_expect_tx(&bar[3], (uint32_t)(kKD * VD * 2));
        bulk_load(sm + SM::kKt, stiles + (((size_t)c * a.B + b) * a.H + h) * (size_t)(kKD * VD * 2),
                  (uint32_t)(kKD * VD * 2), &bar[3]);
    }
    {  // P = M o Lmask as bf16 pairs over the columns of M already read
        const float rf = ex2(lt2 - l0);
#pragma unroll 1
        for (int sb = 0; sb < 4; ++sb) {
            uint32_t pk[16];
            if (sb > warp) {
#pragma unroll
                for (int q = 0; q < 16; ++q) pk[q] = 0u;
                tc::st16(tmem + lane_off + 16 * sb, pk);
                continue;
            }
            float v[32];
            tc::ld16(tmem + lane_off + 32 * sb, v);
            tc::ld16(tmem + lane_off + 32 * sb + 16, v + 16);
            tc::wait_ld();
            if (sb < warp) {
                const float* cfb = cfw + 32 * sb;
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    __nv_bfloat162 pr = __floats2bfloat162_rn(v[2 * q] * (rf * cfb[2 * q]), v[2 * q + 1] * (rf * cfb[2 * q + 1]));
                    pk[q] = *reinterpret_cast<uint32_t*>(&pr);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int s = 32 * sb + 2 * q;
                    const float p0 = s <= tid ? v[2 * q] * ex2(lt2 - l2s[s]) : 0.0f;
                    const float p1 = s + 1 <= tid ? v[2 * q + 1] * ex2(lt2 - l2s[s + 1]) : 0.0f;
                    __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                    pk[q] = *reinterpret_cast<uint32_t*>(&pr);
                }
            }
            tc::st16(tmem + lane_off + 16 * sb, pk);
        }
        tc::wait_st();
    }
    if (has_in) scale_row(sm + SM::kQt, tid, kKD, kQ, E);  // q is consumed by Q K^T: diag(E) q
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        ok = mbar_wait(&bar[1], 0, a.hdr, 812);
        if (has_in) ok = ok && mbar_wait(&bar[3], 0, a.hdr, 813);
        tc::fence_after_sync();
        tc::mma_ts_tiles(tmem + kColO, tmem, smem_u32(sm + SM::kVt), 1, kQ, VD, kQ, 0);  // P V
        if (has_in)  // + diag(E) Q S_in
            tc::mma_tiles(tmem + kColO, smem_u32(sm + SM::kQt), 0, kQ, smem_u32(sm + SM::kKt), 1, kKD, kQ, VD, kKD, 1);
        tc::commit(&bar[4]);
    }
    ok = ok && mbar_wait(&bar[4], 0, a.hdr, 814);
    tc::fence_after_sync();
    {  // output row t into the v tile (v is consumed), then a TMA store
        char* Ot = sm + SM::kVt;
#pragma unroll
        for (int v0 = 0; v0 < VD; v0 += 16) {
            float o[16];
            tc::ld16(tmem + kColO + lane_off + v0, o);
            tc::wait_ld();
            *reinterpret_cast<uint4*>(Ot + tc::sw128_off(tid, v0, kQ)) = pack_bf16x8(o);
            *reinterpret_cast<uint4*>(Ot + tc::sw128_off(tid, v0 + 8, kQ)) = pack_bf16x8(o + 8);
        }
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {
        for (int j = 0; j < VD / 64; ++j) tma_store_4d(&mO, sm + SM::kVt + j * kQ * 128, 64 * j, h, t0, b);
        bulk_commit();
        bulk_wait_read_all();
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------------------- gradients
// With G the adjoint of the chunk's outgoing state (bf16 tile), S_in its entering state, S2 = dO V^T,
// P = M o Lmask, Pd = S2 o Lmask, R = Pd o M:
//   dq = Pd K + diag(E) dO S_in^T      dk = Pd^T Q + diag(w) V G^T      dv = P^T dO + diag(w) K G
//   dl_t = rowsum_t R + E_t dO_t . (Q S_in)_t - colsum_t R - w_t v_t . (K G)_t (+ X at t = Q - 1)
//   X = <G, S_out> = e^{l_Q} <G, S_in> + sum_s w_s v_s . (K G)_s
//   d lam_r = sum_{t >= r} dl_t,  dg = d lam / g.
template <int VD>
struct GGradSmem {
    static constexpr size_t kQt = 0;                       // q
    static constexpr size_t kKt = kQt + kQ * kKD * 2;      // k
    static constexpr size_t kVt = kKt + kQ * kKD * 2;      // v, then diag(w) v
    static constexpr size_t kOt = kVt + kQ * VD * 2;       // dO, then diag(E) dO
    static constexpr size_t kPt = kOt + kQ * VD * 2;       // P, then the S_in tile
    static constexpr size_t kPdt = kPt + kQ * kQ * 2;      // Pd, then the G tile
    static constexpr size_t kL2 = kPdt + kQ * kQ * 2;      // l log2e [128]
    static constexpr size_t kCf = kL2 + kQ * 4;            // column factors [4][128]
    static constexpr size_t kRowp = kCf + 4 * kQ * 4;      // row sums of R [2][128]
    static constexpr size_t kColp = kRowp + 2 * kQ * 4;    // column sums of R [4][128]
    static constexpr size_t kQdq = kColp + 4 * kQ * 4;     // E dO . Y2 [2][128]
    static constexpr size_t kKdk = kQdq + 2 * kQ * 4;      // w v . KG [2][128]
    static constexpr size_t kGs = kKdk + 2 * kQ * 4;       // <G, S_in> partials [256]
    static constexpr size_t kTmp = kGs + 256 * 4;          // scan scratch
    static constexpr size_t kBar = kTmp + 256;             // 0 loads, 1 A, 2 B, 3 S_in/G, 4 C, 5 D
    static constexpr size_t kTmem = kBar + 64;
    static constexpr size_t kTicket = kTmem + 8;
    static constexpr size_t kEnd = kTmem + 64;
    static constexpr size_t kAlloc = kEnd + 1024;
    static_assert(kAlloc <= 232448, "gradient CTA exceeds the shared memory of one CTA");
};

struct GlaGradArgs {
    GlaArgs a;
    const char* stiles;      // [nchunk][B][H] bf16 tiles of the entering states
    const char* gtiles;      // [nchunk][B][H] bf16 tiles of the adjoint states
    const unsigned int* gready;  // [nchunk][B][H]: halves of the slot's G tile written (by the scan kernel)
    const unsigned int* sready;  // [nchunk][B][H]: halves of the recomputed S_in tile written, or null (one
                                 // chunk per segment: the tiles come with the checkpoint)
    int halves;
    __nv_bfloat16* dq;       // [B, L, H, K]
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;       // [B, L, H, V]
    __nv_bfloat16* dg;       // [B, L, H]
};

// One CTA per (chunk, batch row, head), 256 threads: warpgroup wg takes columns [64 wg, ...) (or
// [VD/2 wg, ...)) of TMEM lane / row 32 wq + lane.  TMEM: phase A M (0), S2 (128); phase B dq (0),
// dk (128), P^T dO (256); phase C adds the S_in / G terms to dq, dk and K G (256 + VD); phase D
// Q S_in (256).
template <int VD>
__global__ void __launch_bounds__(256, 1)
gla_grad_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mO, GlaGradArgs ga) {
    using SM = GGradSmem<VD>;
    constexpr uint32_t kCdq = 0, kCdk = 128, kCdv = 256, kCkg = 256 + VD, kCy2 = 256;
    constexpr int kHalf = VD / 2;  // value columns per warpgroup
    const GlaArgs& a = ga.a;
    char* sm = smem_base1024();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::kBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM::kTmem);
    float* l2s = reinterpret_cast<float*>(sm + SM::kL2);
    float* cf = reinterpret_cast<float*>(sm + SM::kCf);
    float* rowp = reinterpret_cast<float*>(sm + SM::kRowp);
    float* colp = reinterpret_cast<float*>(sm + SM::kColp);
    float* qdqp = reinterpret_cast<float*>(sm + SM::kQdq);
    float* kdkp = reinterpret_cast<float*>(sm + SM::kKdk);
    float* gsp = reinterpret_cast<float*>(sm + SM::kGs);
    float* tmp = reinterpret_cast<float*>(sm + SM::kTmp);
    const uint32_t sQ = smem_u32(sm + SM::kQt), sK = smem_u32(sm + SM::kKt), sV = smem_u32(sm + SM::kVt),
                   sO = smem_u32(sm + SM::kOt), sP = smem_u32(sm + SM::kPt), sPd = smem_u32(sm + SM::kPdt);
    const int tid = threadIdx.x, wg = tid >> 7, wq = (tid >> 5) & 3, lane = tid & 31;
    const int row = tid & 127;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // tile from a ticket taken at the start, chunks from the last (whose adjoint the scan kernel
    // writes first)
    unsigned int* ticket = reinterpret_cast<unsigned int*>(sm + SM::kTicket);
    if (tid == 0) *ticket = take_ticket(a.hdr, 0);
    pdl_launch_dependents();

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bar[i], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (tid < 32) tc::tmem_alloc(tmem_slot, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    int idx = (int)*ticket;
    const int h = idx % a.H;
    idx /= a.H;
    const int b = idx % a.B;
    const int c = a.nchunk - 1 - idx / a.B;
    const int t0 = c * kQ;
    const bool has_in = c > 0, has_out = c + 1 < a.nchunk;
    const bool vrow = t0 + row < a.L;
    const size_t tok = ((size_t)b * a.L + (vrow ? t0 + row : 0)) * a.H + h;  // token index of this row
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], (uint32_t)(2 * kQ * kKD * 2 + 2 * kQ * VD * 2));
        for (int j = 0; j < kKD / 64; ++j) {
            tma_load_4d(sm + SM::kQt + j * kQ * 128, &mQ, &bar[0], 64 * j, h, t0, b);
            tma_load_4d(sm + SM::kKt + j * kQ * 128, &mK, &bar[0], 64 * j, h, t0, b);
        }
        for (int j = 0; j < VD / 64; ++j) {
            tma_load_4d(sm + SM::kVt + j * kQ * 128, &mV, &bar[0], 64 * j, h, t0, b);
            tma_load_4d(sm + SM::kOt + j * kQ * 128, &mO, &bar[0], 64 * j, h, t0, b);
        }
    }
    // the G tile of slot c: written by the scan kernel, which counts each 64-column half once its
    // copies have landed (the last chunk's zero adjoint too, counted only after the kernels before
    // the scan are done); polled here by a thread of warpgroup 1, idle while warpgroup 0 forms the
    // decays, and no global write of this kernel comes before the barrier below
    // (a timeout is recorded in the workspace; the kernel finishes)
    if (tid == 224) {
        wait_count(&ga.gready[((size_t)c * a.B + b) * a.H + h], (unsigned int)ga.halves, a.hdr, 828);
        if (ga.sready) wait_count(&ga.sready[((size_t)c * a.B + b) * a.H + h], (unsigned int)ga.halves, a.hdr, 830);
    }
    // decays (warpgroup 0), column factors cf[w][s] = e^{l_{32 w} - l_s} (s < 32 w); the row's
    // gate stays in a register for dg = d lam / g at the end (its load is not repeated there)
    float gself = 1.0f;
    if (wg == 0) {
        if (vrow) gself = __bfloat162float(a.g[tok]);
        l2s[row] = wg0_inclusive_sum(vrow ? __logf(gself) : 0.0f, tmp) * kLog2e;
    }
    __syncthreads();
#pragma unroll
    for (int k = tid; k < 4 * kQ; k += 256) {
        const int w = k >> 7, s = k & 127;
        if (s < 32 * w) cf[k] = ex2(l2s[32 * w] - l2s[s]);
    }
    bool ok = mbar_wait(&bar[0], 0, a.hdr, 820);
    __syncthreads();
    if (tid == 0 && ok) {  // phase A
        tc::fence_after_sync();
        tc::mma_tiles(tmem, sQ, 0, kQ, sK, 0, kQ, kQ, kQ, kKD, 0);         // M  = Q K^T
        tc::mma_tiles(tmem + 128, sO, 0, kQ, sV, 0, kQ, kQ, kQ, VD, 0);   // S2 = dO V^T
        tc::commit(&bar[1]);
    }
    ok = ok && mbar_wait(&bar[1], 0, a.hdr, 821);
    tc::fence_after_sync();
    // ---- E1: P, Pd (bf16 tiles) and the fp32 row / column sums of R = Pd o M
    {
        char* Pt = sm + SM::kPt;
        char* Pdt = sm + SM::kPdt;
        const float l2r = l2s[row];
        const float rf = ex2(l2r - l2s[32 * wq]);
        float rsum = 0.0f;
#pragma unroll 1
        for (int sb = wg; sb < 4; sb += 2) {
            const int s0 = 32 * sb;
            if (sb > wq) {  // above the diagonal
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int k = 0; k < 32; k += 8) {
                    *reinterpret_cast<uint4*>(Pt + tc::sw128_off(row, s0 + k, kQ)) = z;
                    *reinterpret_cast<uint4*>(Pdt + tc::sw128_off(row, s0 + k, kQ)) = z;
                }
                colp[wq * kQ + s0 + lane] = 0.0f;
                continue;
            }
            float m[32], s2[32];
            tc::ld16(tmem + lane_off + s0, m);
            tc::ld16(tmem + lane_off + s0 + 16, m + 16);
            tc::ld16(tmem + 128 + lane_off + s0, s2);
            tc::ld16(tmem + 128 + lane_off + s0 + 16, s2 + 16);
            tc::wait_ld();
            float rr[32];
            if (sb < wq) {
                const float* cfb = cf + wq * kQ + s0;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float f = rf * cfb[k];
                    const float mk = m[k];
                    m[k] = mk * f;
                    s2[k] *= f;
                    rr[k] = s2[k] * mk;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int s = s0 + k;
                    const float f = s <= row ? ex2(l2r - l2s[s]) : 0.0f;
                    const float mk = m[k];
                    m[k] = mk * f;
                    s2[k] *= f;
                    rr[k] = s2[k] * mk;
                }
            }
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
                *reinterpret_cast<uint4*>(Pt + tc::sw128_off(row, s0 + k, kQ)) = pack_bf16x8(m + k);
                *reinterpret_cast<uint4*>(Pdt + tc::sw128_off(row, s0 + k, kQ)) = pack_bf16x8(s2 + k);
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) rsum += rr[k];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {  // lane l ends with column s0 + l
                const bool up = (lane & off) != 0;
#pragma unroll
                for (int k = 0; k < off; ++k) {
                    const float send = up ? rr[k] : rr[k + off];
                    const float keep = up ? rr[k + off] : rr[k];
                    rr[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
            colp[wq * kQ + s0 + lane] = rr[0];
        }
        rowp[wg * kQ + row] = rsum;
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {  // phase B
        tc::fence_after_sync();
        tc::mma_tiles(tmem + kCdq, sPd, 0, kQ, sK, 1, kQ, kQ, kKD, kQ, 0);  // dq  = Pd K
        tc::mma_tiles(tmem + kCdk, sPd, 1, kQ, sQ, 1, kQ, kQ, kKD, kQ, 0);  // dk  = Pd^T Q
        tc::mma_tiles(tmem + kCdv, sP, 1, kQ, sO, 1, kQ, kQ, VD, kQ, 0);    // dv1 = P^T dO
        tc::commit(&bar[2]);
    }
    ok = ok && mbar_wait(&bar[2], 0, a.hdr, 822);
    tc::fence_after_sync();
    if (tid == 0) {  // P, Pd are consumed: their slots take S_in and G
        fence_proxy_async_global();  // the copies below come after the count polled above
        const size_t tile = (((size_t)c * a.B + b) * a.H + h) * (size_t)(kKD * VD * 2);
        const uint32_t bytes = (has_in ? kKD * VD * 2 : 0u) + (has_out ? kKD * VD * 2 : 0u);
        if (bytes == 0) {
            mbar_arrive(&bar[3]);
        } else {
            mbar_arrive_expect_tx(&bar[3], bytes);
            if (has_in) bulk_load(sm + SM::kPt, ga.stiles + tile, (uint32_t)(kKD * VD * 2), &bar[3]);
            if (has_out) bulk_load(sm + SM::kPdt, ga.gtiles + tile, (uint32_t)(kKD * VD * 2), &bar[3]);
        }
    }
    // dO rows scaled by E, v rows by w (their unscaled uses are done)
    const float l2r = l2s[row];
    const float E = ex2(l2r), w = ex2(l2s[kQ - 1] - l2r);
    {
        char* Vt = sm + SM::kVt;
        char* Ot = sm + SM::kOt;
#pragma unroll
        for (int c0 = 0; c0 < kHalf; c0 += 8) {
            const uint32_t off = tc::sw128_off(row, kHalf * wg + c0, kQ);
            uint4 vr = *reinterpret_cast<const uint4*>(Vt + off), orr = *reinterpret_cast<const uint4*>(Ot + off);
            __nv_bfloat162* vv = reinterpret_cast<__nv_bfloat162*>(&vr);
            __nv_bfloat162* ov = reinterpret_cast<__nv_bfloat162*>(&orr);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 vf = __bfloat1622float2(vv[e]), of = __bfloat1622float2(ov[e]);
                vv[e] = __floats2bfloat162_rn(vf.x * w, vf.y * w);
                ov[e] = __floats2bfloat162_rn(of.x * E, of.y * E);
            }
            *reinterpret_cast<uint4*>(Vt + off) = vr;
            *reinterpret_cast<uint4*>(Ot + off) = orr;
        }
    }
    ok = ok && mbar_wait(&bar[3], 0, a.hdr, 823);
    {  // <G, S_in> partial over this thread's row (state row k) and columns
        float gs = 0.0f;
        if (has_in && has_out) {
#pragma unroll
            for (int c0 = 0; c0 < kHalf; c0 += 8) {
                const uint32_t off = tc::sw128_off(row, kHalf * wg + c0, kKD);
                uint4 sr = *reinterpret_cast<const uint4*>(sm + SM::kPt + off);
                uint4 gr = *reinterpret_cast<const uint4*>(sm + SM::kPdt + off);
                const __nv_bfloat162* sv = reinterpret_cast<const __nv_bfloat162*>(&sr);
                const __nv_bfloat162* gv = reinterpret_cast<const __nv_bfloat162*>(&gr);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 sf = __bfloat1622float2(sv[e]), gf = __bfloat1622float2(gv[e]);
                    gs = fmaf(sf.x, gf.x, fmaf(sf.y, gf.y, gs));
                }
            }
        }
        gsp[tid] = gs;
    }
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {  // phase C
        tc::fence_after_sync();
        if (has_in) tc::mma_tiles(tmem + kCdq, sO, 0, kQ, sP, 0, kKD, kQ, kKD, VD, 1);    // dq += (E dO) S_in^T
        if (has_out) {
            tc::mma_tiles(tmem + kCdk, sV, 0, kQ, sPd, 0, kKD, kQ, kKD, VD, 1);           // dk += (w V) G^T
            tc::mma_tiles(tmem + kCkg, sK, 0, kQ, sPd, 1, kKD, kQ, VD, kKD, 0);           // K G
        }
        tc::commit(&bar[4]);
    }
    ok = ok && mbar_wait(&bar[4], 0, a.hdr, 824);
    tc::fence_after_sync();
    {  // E2a: dv = P^T dO + w K G, kdk = (w v) . K G
        const char* Vt = sm + SM::kVt;
        float kdk = 0.0f;
#pragma unroll
        for (int v0 = 0; v0 < kHalf; v0 += 16) {
            const int col = kHalf * wg + v0;
            float dv[16], kg[16];
            tc::ld16(tmem + kCdv + lane_off + col, dv);
            if (has_out) tc::ld16(tmem + kCkg + lane_off + col, kg);
            tc::wait_ld();
            if (has_out) {
#pragma unroll
                for (int hh = 0; hh < 16; hh += 8) {
                    uint4 vr = *reinterpret_cast<const uint4*>(Vt + tc::sw128_off(row, col + hh, kQ));
                    const __nv_bfloat162* vv = reinterpret_cast<const __nv_bfloat162*>(&vr);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 vf = __bfloat1622float2(vv[e]);
                        kdk = fmaf(vf.x, kg[hh + 2 * e], fmaf(vf.y, kg[hh + 2 * e + 1], kdk));
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) dv[e] = fmaf(w, kg[e], dv[e]);
            }
            if (vrow) {
                *reinterpret_cast<uint4*>(ga.dv + tok * VD + col) = pack_bf16x8(dv);
                *reinterpret_cast<uint4*>(ga.dv + tok * VD + col + 8) = pack_bf16x8(dv + 8);
            }
        }
        kdkp[wg * kQ + row] = kdk;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0 && ok) {  // phase D
        tc::fence_after_sync();
        if (has_in) tc::mma_tiles(tmem + kCy2, sQ, 0, kQ, sP, 1, kKD, kQ, VD, kKD, 0);   // Q S_in
        tc::commit(&bar[5]);
    }
    {  // dq, dk rows (their products are complete): columns [64 wg, 64 wg + 64)
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            __nv_bfloat16* dst = (which == 0 ? ga.dq : ga.dk) + tok * kKD + 64 * wg;
            const uint32_t col = (which == 0 ? kCdq : kCdk) + 64 * wg;
#pragma unroll
            for (int v0 = 0; v0 < 64; v0 += 16) {
                float v[16];
                tc::ld16(tmem + col + lane_off + v0, v);
                tc::wait_ld();
                if (vrow) {
                    *reinterpret_cast<uint4*>(dst + v0) = pack_bf16x8(v);
                    *reinterpret_cast<uint4*>(dst + v0 + 8) = pack_bf16x8(v + 8);
                }
            }
        }
    }
    ok = ok && mbar_wait(&bar[5], 0, a.hdr, 825);
    tc::fence_after_sync();
    {  // E2b: (E dO) . Q S_in
        const char* Ot = sm + SM::kOt;
        float qdq = 0.0f;
        if (has_in) {
#pragma unroll
            for (int v0 = 0; v0 < kHalf; v0 += 16) {
                const int col = kHalf * wg + v0;
                float y2[16];
                tc::ld16(tmem + kCy2 + lane_off + col, y2);
                tc::wait_ld();
#pragma unroll
                for (int hh = 0; hh < 16; hh += 8) {
                    uint4 orr = *reinterpret_cast<const uint4*>(Ot + tc::sw128_off(row, col + hh, kQ));
                    const __nv_bfloat162* ov = reinterpret_cast<const __nv_bfloat162*>(&orr);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 of = __bfloat1622float2(ov[e]);
                        qdq = fmaf(of.x, y2[hh + 2 * e], fmaf(of.y, y2[hh + 2 * e + 1], qdq));
                    }
                }
            }
        }
        qdqp[wg * kQ + row] = qdq;
    }
    __syncthreads();
    if (wg == 0) {  // dl, d lam (reverse cumulative sum), dg
        const int t = row;
        const float cs = (colp[t] + colp[kQ + t]) + (colp[2 * kQ + t] + colp[3 * kQ + t]);
        const float rs = rowp[t] + rowp[kQ + t];
        const float qi = qdqp[t] + qdqp[kQ + t];
        const float ki = kdkp[t] + kdkp[kQ + t];  // w_t v_t . (K G)_t (v was scaled by w)
        const float2 kg = wg0_sum2(ki, gsp[t] + gsp[kQ + t], tmp);
        const float X = ex2(l2s[kQ - 1]) * kg.y + kg.x;
        float dl = rs + qi - cs - ki + (t == kQ - 1 ? X : 0.0f);
        if (!vrow) dl = 0.0f;
        float total;
        const float incl = wg0_inclusive_sum(dl, tmp, &total);
        const float dlam = total - incl + dl;
        if (vrow) ga.dg[tok] = __float2bfloat16_rn(dlam / gself);
    }
    __syncthreads();
    if (tid < 32) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// Chunks per checkpoint segment.  With one chunk per segment the checkpoint buffer also holds the
// bf16 tile copy of every state; with longer segments it holds the f32 segment states only, the
// forward pass keeps the tiles of every chunk in its workspace and the backward pass recomputes
// them from the segment states.
int chunks_per_segment(const lr_desc& d) { return d.segment / kQ; }

struct GlaWs {
    size_t ready, sready, flags_end, gtiles, stiles, end;  // the slot flags first (reset every call)
};
GlaWs gla_plan(const lr_desc& d, bool bwd) {
    const size_t nchunk = (size_t)((d.L + kQ - 1) / kQ);
    const size_t tiles = (size_t)d.B * d.H * nchunk;
    const bool seg = chunks_per_segment(d) > 1;
    WsCursor cur;
    GlaWs w{};
    w.ready = cur.take(sizeof(unsigned int) * tiles * (size_t)(d.P / kScanP));
    if (bwd && seg) w.sready = cur.take(sizeof(unsigned int) * tiles);
    w.flags_end = cur.off;
    if (bwd) w.gtiles = cur.take((size_t)2 * tiles * kKD * d.P);
    if (seg) w.stiles = cur.take((size_t)2 * tiles * kKD * d.P);
    w.end = cur.off;
    return w;
}

GlaArgs gla_args(const lr_desc& d, const lr_inputs& in, char* ws) {
    GlaArgs a{};
    a.B = (int)d.B;
    a.L = (int)d.L;
    a.H = (int)d.H;
    a.nchunk = (int)((d.L + kQ - 1) / kQ);
    a.g = (const __nv_bfloat16*)in.g;
    a.hdr = (WsHeader*)ws;
    a.withhold = (d.flags & LR_TEST_WITHHOLD_CARRY) ? 1 : 0;
    return a;
}

// The scan kernel's view of the problem (chunk_scan.cuh): per-head rows (G = H), decay log g.
ScanArgs scan_args(const GlaArgs& a, int VD) {
    ScanArgs s{};
    s.B = a.B;
    s.L = a.L;
    s.H = a.H;
    s.G = a.H;
    s.HpG = 1;
    s.nchunk = a.nchunk;
    s.halves = VD / kScanP;
    s.dt = a.g;
    s.hdr = a.hdr;
    s.withhold = a.withhold;
    s.f32_every = 1;
    return s;
}

// The chunk-state scan over (row, head, 64 value columns): dir > 0 folds K^T diag(w) V into the
// entering states (f32 checkpoint slots every `kseg` chunks, bf16 tiles of every chunk); dir < 0
// folds Q^T diag(E) dO into the adjoint states (bf16 tiles).  With `recompute` (dir > 0, kseg > 1)
// one CTA per (row, head, half) rebuilds the tiles of every chunk from the f32 segment states in
// `ckpt`, the last segment first.  Each slot half is flagged in `ready` once written.
template <int VD>
lr_status gla_scan(const lr_desc& d, const GlaArgs& a, const CUtensorMap& mR, const CUtensorMap& mZ, void* ckpt,
                   char* tiles, int dir, unsigned int* ready, int kseg, bool recompute, cudaStream_t st) {
    const int nseg = (a.nchunk + kseg - 1) / kseg;
    CUtensorMap mS, mDt;
    if (dir > 0 && !recompute && !map_states_vd(&mS, ckpt, (int64_t)a.B * a.H, nseg, VD)) return LR_ERR_INVALID_ARG;
    if (dir < 0 || recompute) mS = mR;  // no f32 states written
    const int dt_tma = map_dt(&mDt, d.B, d.L, d.H, a.g) ? 1 : 0;
    if (!dt_tma) mDt = mR;  // not read
    ScanArgs sa = scan_args(a, VD);
    cudaError_t e;
    if (recompute) {
        sa.seg_k = kseg;
        sa.s_init = (const float*)ckpt;
        sa.vd = VD;
        using SR = ScanSmem<4, false>;
        cudaFuncSetAttribute(chunk_scan_kernel<4, false, kScanGla>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SR::kAlloc);
        note_launch("gla_state_recompute");
        e = launch_pdl(chunk_scan_kernel<4, false, kScanGla>, dim3((unsigned)(a.B * a.H * sa.halves)),
                       dim3(kScanThreads), SR::kAlloc, st, mR, mZ, mS, mDt, dt_tma, sa, tiles, +1, ready,
                       (float*)nullptr, (float*)nullptr, (unsigned int*)nullptr);
        if (e != cudaSuccess) return LR_ERR_CUDA;
        return check_launch();
    }
    const dim3 grid((unsigned)(a.B * a.H * sa.halves));
    note_launch("gla_state_scan");
    if (dir > 0) {
        sa.f32_every = kseg;  // f32 checkpoints at segment starts only
        using SF = ScanSmem<3, true>;
        cudaFuncSetAttribute(chunk_scan_kernel<3, true, kScanGla>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SF::kAlloc);
        e = launch_pdl(chunk_scan_kernel<3, true, kScanGla>, grid, dim3(kScanThreads), SF::kAlloc, st, mR, mZ, mS,
                       mDt, dt_tma, sa, tiles, +1, ready, (float*)nullptr, (float*)nullptr, (unsigned int*)nullptr);
    } else {
        using SB = ScanSmem<4, false>;
        cudaFuncSetAttribute(chunk_scan_kernel<4, false, kScanGla>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SB::kAlloc);
        e = launch_pdl(chunk_scan_kernel<4, false, kScanGla>, grid, dim3(kScanThreads), SB::kAlloc, st, mR, mZ, mS,
                       mDt, dt_tma, sa, tiles, -1, ready, (float*)nullptr, (float*)nullptr, (unsigned int*)nullptr);
    }
    if (e != cudaSuccess) return LR_ERR_CUDA;
    return check_launch();
}

template <int VD>
lr_status gla_fwd_t(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws, cudaStream_t st) {
    const GlaWs w = gla_plan(d, false);
    GlaArgs a = gla_args(d, in, ws);
    CUtensorMap mQ, mK, mV, mO;
    if (!(map4(&mQ, in.q, kKD, d.H, d.L, d.B, true) && map4(&mK, in.k, kKD, d.H, d.L, d.B, true) &&
          map4(&mV, in.v, VD, d.H, d.L, d.B, true) && map4(&mO, y, VD, d.H, d.L, d.B, true)))
        return LR_ERR_INVALID_ARG;
    const int kseg = chunks_per_segment(d);
    char* stiles = kseg == 1 ? (char*)ckpt + (size_t)a.nchunk * a.B * a.H * kKD * VD * sizeof(float) : ws + w.stiles;
    unsigned int* ready = (unsigned int*)(ws + w.ready);
    lr_status s = gla_scan<VD>(d, a, mK, mV, ckpt, stiles, +1, ready, kseg, false, st);
    if (s != LR_OK) return s;
    cudaFuncSetAttribute(gla_out_kernel<VD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GOutSmem<VD>::kAlloc);
    note_launch("gla_chunk_out");
    if (launch_pdl(gla_out_kernel<VD>, dim3(a.nchunk * a.B * a.H), dim3(kThreads), GOutSmem<VD>::kAlloc, st, mQ, mK,
                   mV, mO, a, (const char*)stiles, (const unsigned int*)ready, VD / kScanP) != cudaSuccess)
        return LR_ERR_CUDA;
    return check_launch();
}

template <int VD>
lr_status gla_bwd_t(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt, const lr_grads& gr,
                    char* ws, cudaStream_t st) {
    const GlaWs w = gla_plan(d, true);
    GlaGradArgs ga{};
    ga.a = gla_args(d, in, ws);
    const GlaArgs& a = ga.a;
    const int kseg = chunks_per_segment(d);
    ga.stiles = kseg == 1 ? (const char*)ckpt + (size_t)a.nchunk * a.B * a.H * kKD * VD * sizeof(float)
                          : (const char*)(ws + w.stiles);
    ga.sready = kseg > 1 ? (const unsigned int*)(ws + w.sready) : nullptr;
    ga.gtiles = ws + w.gtiles;
    ga.gready = (const unsigned int*)(ws + w.ready);
    ga.halves = VD / kScanP;
    ga.dq = (__nv_bfloat16*)gr.dq;
    ga.dk = (__nv_bfloat16*)gr.dk;
    ga.dv = (__nv_bfloat16*)gr.dv;
    ga.dg = (__nv_bfloat16*)gr.dg;
    CUtensorMap mQ, mK, mV, mO;
    if (!(map4(&mQ, in.q, kKD, d.H, d.L, d.B, true) && map4(&mK, in.k, kKD, d.H, d.L, d.B, true) &&
          map4(&mV, in.v, VD, d.H, d.L, d.B, true) && map4(&mO, dy, VD, d.H, d.L, d.B, true)))
        return LR_ERR_INVALID_ARG;
    lr_status s = gla_scan<VD>(d, a, mQ, mO, nullptr, ws + w.gtiles, -1, (unsigned int*)(ws + w.ready), kseg, false, st);
    if (s != LR_OK) return s;
    if (kseg > 1) {  // the states entering every chunk, rebuilt from the f32 segment states beside the scan
        s = gla_scan<VD>(d, a, mK, mV, const_cast<void*>(ckpt), ws + w.stiles, +1, (unsigned int*)(ws + w.sready),
                         kseg, true, st);
        if (s != LR_OK) return s;
    }
    cudaFuncSetAttribute(gla_grad_kernel<VD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GGradSmem<VD>::kAlloc);
    note_launch("gla_chunk_grad");
    if (launch_pdl(gla_grad_kernel<VD>, dim3(a.nchunk * a.B * a.H), dim3(256), GGradSmem<VD>::kAlloc, st, mQ, mK, mV,
                   mO, ga) != cudaSuccess)
        return LR_ERR_CUDA;
    return check_launch();
}

}  // namespace

size_t gla_ws_bytes(const lr_desc& d, bool bwd) { return gla_plan(d, bwd).end; }
size_t gla_flag_bytes(const lr_desc& d, bool bwd) { return gla_plan(d, bwd).flags_end; }

lr_status gla_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws, cudaStream_t st) {
    return d.P == 64 ? gla_fwd_t<64>(d, in, y, ckpt, ws, st) : gla_fwd_t<128>(d, in, y, ckpt, ws, st);
}
lr_status gla_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt, const lr_grads& gr,
                  char* ws, cudaStream_t st) {
    return d.P == 64 ? gla_bwd_t<64>(d, in, dy, ckpt, gr, ws, st) : gla_bwd_t<128>(d, in, dy, ckpt, gr, ws, st);
}

}  // namespace lrs
