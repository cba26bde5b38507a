// diag.cu -- diagonal chassis: rglru_scan and rotlru_scan, forward and backward (sm_100a).
//
// Recurrence h_t = c_t h_{t-1} + b_t with a real (rglru) or complex (rotlru) diagonal
// coefficient c_t, read out as y_t = h_t ("mlx-recurrence", Apple Developer Forums thread
// 840535, "Current kernels": rglru_scan, rotlru_scan).  The sequence is cut into checkpoint
// segments of S steps; chunks compose with the associative operator
// (c2, b2) o (c1, b1) = (c2 c1, c2 b1 + b2) of the K-Search / mlx-mamba post (techtrendfeed
// repost, paragraph after Table 1).
//
// Tiling.  One CTA owns one tile = (batch row b, channel block, segment): S steps x CB units
// (rglru: 32 real channels; rotlru: 16 complex pairs = 32 floats).  The CTA loads the whole tile
// into shared memory with TMA (one box per tensor, ragged tails zero-filled by the TMA unit),
// splits it into NG time groups of S/NG steps (one thread per unit per group), scans each group
// sequentially in fp32, combines the groups in shared memory and joins the tiles of a row: a row of
// at most 8 tiles runs as one thread-block cluster whose tiles exchange their aggregates through
// distributed shared memory; longer rows chain through a single-pass look-back over per-tile carry
// records in global memory (aggregate first, inclusive prefix once known; bounded waits).  Both
// fold the same aggregates in the same order.  Results are written back into the tile's
// shared-memory slots and stored with TMA.
//
// Forward: carries flow to later segments; the carry entering each segment is the segment
// checkpoint (written to ckpt).  Backward ("segment checkpointing with recomputation during the
// backward pass", same post): each tile starts from its checkpoint, recomputes its states into
// registers, runs the adjoint recurrence G_t = dy_t + conj(c_{t+1}) G_{t+1} with carries flowing
// to earlier segments, and writes the input gradients; rotlru's parameter gradients are summed
// per tile into partials that a second kernel reduces in a fixed order.
#include <stdio.h>

#include <algorithm>

#include "common.cuh"
#include "host_common.h"

namespace lrs {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxSeg = 256;  // TMA box rows; S <= 256 keeps the tile in one box per tensor

__device__ __forceinline__ float one_of(float) { return 1.0f; }
__device__ __forceinline__ cpx one_of(cpx) { return {1.0f, 0.0f}; }
__device__ __forceinline__ float zero_of(float) { return 0.0f; }
__device__ __forceinline__ cpx zero_of(cpx) { return {0.0f, 0.0f}; }
__device__ __forceinline__ float mulx(float a, float b) { return a * b; }
__device__ __forceinline__ cpx mulx(cpx a, cpx b) { return cmul(a, b); }
__device__ __forceinline__ float fmax_(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ cpx fmax_(cpx a, cpx b, cpx c) { return cfma(a, b, c); }
__device__ __forceinline__ float conjx(float a) { return a; }
__device__ __forceinline__ cpx conjx(cpx a) { return conjc(a); }
__device__ __forceinline__ float addx(float a, float b) { return a + b; }
__device__ __forceinline__ cpx addx(cpx a, cpx b) { return {a.r + b.r, a.i + b.i}; }

template <typename V> struct Agg {
    V m;  // product of coefficients over the span
    V v;  // local result with zero carry-in
};

struct DiagArgs {
    int B, L, D, S, nseg, ncb;  // D = real channels of b / y
    unsigned int dflags;        // lr_desc flags (LR_TEST_WITHHOLD_CARRY)
    int direct;                 // tiles numbered by block index (the grid fits on the SMs at once)
    int cl;                     // > 0: a row's tiles form one thread-block cluster of cl CTAs (cl = nseg)
    int ahead;                  // forward, ticket mode: a tile prefetches the tile `ahead` tickets later into L2
    const float* mag;           // rotlru
    const float* theta;         // rotlru
    const float* lam;           // rglru with gates: Lambda [D]
    float* ckpt;                // [nseg, B, D] f32
    WsHeader* hdr;
    unsigned int* flags;        // [B * ncb * nseg]
    void* agg;                  // Agg<V>[tiles][CB]
    void* pre;                  // V[tiles][CB]
    float2* partial;            // bwd: rotlru [B * nseg][D/2] (dmag, dtheta); gated rglru [B * nseg][D] (dLambda, 0)
};

// Per-kind description.  Unit = the element one thread carries through time.
template <int KIND, typename T> struct Kind;

template <typename T> struct Kind<LR_RGLRU, T> {
    using V = float;
    static constexpr int CB = 32;        // units (channels) per tile
    static constexpr int NG = 8;         // time groups
    static constexpr int CW = CB;        // coefficient-tensor columns per tile
    static constexpr int BW = CB;        // b / y columns per tile
    struct Unit {
        __device__ Unit(const DiagArgs&, int) {}
        __device__ __forceinline__ V coef(const T* C, int t, int u) const {
            return IO<T>::ld(C + t * CW + u);
        }
    };
    static __device__ __forceinline__ V ldb(const T* Bs, int t, int u) { return IO<T>::ld(Bs + t * BW + u); }
    static __device__ __forceinline__ void stb(T* Bs, int t, int u, V v) { IO<T>::st(Bs + t * BW + u, v); }
    static __device__ __forceinline__ void st_ckpt(float* p, int chan0, V v) { p[chan0] = v; }
    static __device__ __forceinline__ V ld_ckpt(const float* p, int chan0) { return p[chan0]; }
    static constexpr int chans_per_unit = 1;
};

// rglru with the RG-LRU gate front-end (LR_RGLRU_GATES, f32): the coefficient tensor holds the
// recurrence gate r, a = sigmoid(Lambda)^(c r) = e^{c r log sigmoid(Lambda)} is formed where it is
// read; b = sqrt(1 - a^2) (i x) is formed once per tile from the input gate i and x.
constexpr int kRgGated = 5;         // internal kind id
constexpr float kRgC = 8.0f;        // the exponent constant c
template <typename T> struct Kind<kRgGated, T> {
    using V = float;
    static constexpr int CB = 16;        // channels per tile (16 x 16 groups measured 10 % faster than
    static constexpr int NG = 16;        // 32 x 8 on the rglru workload's shapes; plain rglru: equal)
    static constexpr int CW = CB;
    static constexpr int BW = CB;
    struct Unit {
        float clog;      // c log sigmoid(Lambda) (<= 0)
        float oms;       // 1 - sigmoid(Lambda)
        __device__ Unit(const DiagArgs& a, int d) {
            const float lam = d < a.D ? a.lam[d] : 1.0f;
            clog = -kRgC * log1pf(expf(-lam));
            oms = 1.0f / (1.0f + expf(lam));
        }
        __device__ __forceinline__ float coef(const T* C, int t, int u) const {
            return expf(IO<T>::ld(C + t * CW + u) * clog);
        }
    };
    static __device__ __forceinline__ V ldb(const T* Bs, int t, int u) { return IO<T>::ld(Bs + t * BW + u); }
    static __device__ __forceinline__ void stb(T* Bs, int t, int u, V v) { IO<T>::st(Bs + t * BW + u, v); }
    static __device__ __forceinline__ void st_ckpt(float* p, int chan0, V v) { p[chan0] = v; }
    static __device__ __forceinline__ V ld_ckpt(const float* p, int chan0) { return p[chan0]; }
    static constexpr int chans_per_unit = 1;
};

template <typename T> struct Kind<LR_ROTLRU, T> {
    using V = cpx;
    static constexpr int CB = 16;        // complex pairs per tile (8 pairs measured 1.4x slower)
    static constexpr int NG = 16;
    static constexpr int CW = CB;        // g columns (one per pair)
    static constexpr int BW = 2 * CB;    // b / y columns (re, im interleaved)
    struct Unit {
        float mag, cs, sn;
        __device__ Unit(const DiagArgs& a, int pair) {
            bool ok = pair < a.D / 2;
            mag = ok ? a.mag[pair] : 0.0f;
            float th = ok ? a.theta[pair] : 0.0f;
            sincosf(th, &sn, &cs);
        }
        __device__ __forceinline__ V coef(const T* C, int t, int u) const {
            float m = mag * IO<T>::ld(C + t * CW + u);
            return {m * cs, m * sn};
        }
    };
    static __device__ __forceinline__ V ldb(const T* Bs, int t, int u) {  // (re, im) in one access
        const float2 v = IO<T>::ld2(Bs + t * BW + 2 * u);
        return {v.x, v.y};
    }
    static __device__ __forceinline__ void stb(T* Bs, int t, int u, V v) {
        IO<T>::st2(Bs + t * BW + 2 * u, make_float2(v.r, v.i));
    }
    static __device__ __forceinline__ void st_ckpt(float* p, int chan0, V v) {
        *reinterpret_cast<float2*>(p + chan0) = make_float2(v.r, v.i);
    }
    static __device__ __forceinline__ V ld_ckpt(const float* p, int chan0) {
        const float2 v = *reinterpret_cast<const float2*>(p + chan0);
        return {v.x, v.y};
    }
    static constexpr int chans_per_unit = 2;
};

// Shared-memory plan of one tile.
template <int KIND, typename T, bool BWD> struct Smem {
    using K = Kind<KIND, T>;
    using V = typename K::V;
    static constexpr bool G = KIND == kRgGated;  // x tile (and, backward, a tile of b values)
    // rotlru backward: dy lands in b's slot once the forward recompute is done with b (three tiles
    // per SM instead of two)
    static constexpr bool AL = BWD && KIND == LR_ROTLRU;
    static __host__ __device__ constexpr size_t coef_bytes() { return size_t(kMaxSeg) * K::CW * sizeof(T); }
    static __host__ __device__ constexpr size_t b_bytes() { return size_t(kMaxSeg) * K::BW * sizeof(T); }
    static __host__ __device__ constexpr size_t off_coef() { return 128; }
    static __host__ __device__ constexpr size_t off_b() { return off_coef() + coef_bytes(); }
    static __host__ __device__ constexpr size_t off_dy() { return off_b() + (AL ? 0 : b_bytes()); }
    static __host__ __device__ constexpr size_t off_x() { return off_dy() + (BWD ? b_bytes() : 0); }
    static __host__ __device__ constexpr size_t off_e() { return off_x() + (G ? b_bytes() : 0); }
    static __host__ __device__ constexpr size_t off_aggf() { return off_e() + (G && BWD ? b_bytes() : 0); }
    static __host__ __device__ constexpr size_t off_aggr() { return off_aggf() + sizeof(Agg<V>) * K::NG * K::CB; }
    static __host__ __device__ constexpr size_t off_carry() {
        return off_aggr() + (BWD ? sizeof(Agg<V>) * K::NG * K::CB : 0);
    }
    static __host__ __device__ constexpr size_t off_cl() { return off_carry() + 2 * sizeof(V) * K::CB; }
    static __host__ __device__ constexpr size_t off_red() { return off_cl() + sizeof(Agg<V>) * K::CB; }
    static __host__ __device__ constexpr size_t off_misc() {
        return off_red() + (BWD ? sizeof(float2) * K::NG * K::CB : 0);
    }
    static __host__ __device__ constexpr size_t total() { return off_misc() + 64 + 128; }
};

template <typename V>
__device__ __forceinline__ void st_cg(V* p, V v) {
    if constexpr (sizeof(V) == 4) {
        __stcg(reinterpret_cast<float*>(p), *reinterpret_cast<float*>(&v));
    } else {
        __stcg(reinterpret_cast<float2*>(p), *reinterpret_cast<float2*>(&v));
    }
}
template <typename V>
__device__ __forceinline__ V ld_cg(const V* p) {
    V v;
    if constexpr (sizeof(V) == 4) {
        *reinterpret_cast<float*>(&v) = __ldcg(reinterpret_cast<const float*>(p));
    } else {
        *reinterpret_cast<float2*>(&v) = __ldcg(reinterpret_cast<const float2*>(p));
    }
    return v;
}
template <typename V>
__device__ __forceinline__ void st_cg_agg(Agg<V>* p, Agg<V> a) {
    st_cg(&p->m, a.m);
    st_cg(&p->v, a.v);
}
template <typename V>
__device__ __forceinline__ Agg<V> ld_cg_agg(const Agg<V>* p) {
    return {ld_cg(&p->m), ld_cg(&p->v)};
}

// A tile's records in the look-back.  Complex values (rotlru) are stored, fenced, and then the
// tile's flag is set with release semantics, so a reader that sees the flag may read them.  Real
// values are published without a fence: each 32-bit value travels with its status in one 64-bit
// word (a single store makes both visible), the flag is set with a relaxed store and only tells a
// reader which records to read, and a reader that finds a record's status missing reads it again.
// The workspace holding the records is zeroed before every call, so a status is this call's.
__device__ __forceinline__ uint64_t pack_rec(unsigned int st, float v) {
    return ((uint64_t)st << 32) | __float_as_uint(v);
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u32(unsigned int* p, unsigned int v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename V> struct Rec;
template <> struct Rec<cpx> {  // fenced
    static constexpr bool kFence = true;
    using AggT = Agg<cpx>;
    using PreT = cpx;
    static __device__ __forceinline__ void put_agg(AggT* p, Agg<cpx> a) { st_cg_agg(p, a); }
    static __device__ __forceinline__ void put_pre(PreT* p, cpx v) { st_cg(p, v); }
    static __device__ __forceinline__ bool get_agg(const AggT* p, Agg<cpx>& a) {
        a = ld_cg_agg(p);
        return true;
    }
    static __device__ __forceinline__ bool get_pre(const PreT* p, cpx& v) {
        v = ld_cg(p);
        return true;
    }
};
template <> struct Rec<float> {  // packed: status in the high word
    static constexpr bool kFence = false;
    struct AggT {
        uint64_t m, v;
    };
    using PreT = uint64_t;
    static __device__ __forceinline__ void put_agg(AggT* p, Agg<float> a) {
        st_relaxed_u64(&p->m, pack_rec(kFlagAgg, a.m));
        st_relaxed_u64(&p->v, pack_rec(kFlagAgg, a.v));
    }
    static __device__ __forceinline__ void put_pre(PreT* p, float v) { st_relaxed_u64(p, pack_rec(kFlagPrefix, v)); }
    static __device__ __forceinline__ bool get_agg(const AggT* p, Agg<float>& a) {
        const uint64_t m = ld_relaxed_u64(&p->m), v = ld_relaxed_u64(&p->v);
        a = {__uint_as_float((unsigned int)m), __uint_as_float((unsigned int)v)};
        return (m >> 32) == kFlagAgg && (v >> 32) == kFlagAgg;
    }
    static __device__ __forceinline__ bool get_pre(const PreT* p, float& v) {
        const uint64_t w = ld_relaxed_u64(p);
        v = __uint_as_float((unsigned int)w);
        return (w >> 32) == kFlagPrefix;
    }
};

// Publish a tile's aggregate (st = kFlagAgg) or inclusive prefix (kFlagPrefix); warp 0, one lane
// per unit (act: the lane's unit exists).
template <typename V>
__device__ __forceinline__ void publish_agg(unsigned int* flag, typename Rec<V>::AggT* rec, Agg<V> a, bool act,
                                            int lane) {
    if (act) Rec<V>::put_agg(rec, a);
    if (Rec<V>::kFence) __threadfence();
    __syncwarp();
    if (lane == 0) {
        if (Rec<V>::kFence)
            st_release(flag, kFlagAgg);
        else
            st_relaxed_u32(flag, kFlagAgg);
    }
}
template <typename V>
__device__ __forceinline__ void publish_pre(unsigned int* flag, typename Rec<V>::PreT* rec, V v, bool act,
                                            int lane) {
    if (act) Rec<V>::put_pre(rec, v);
    if (Rec<V>::kFence) __threadfence();
    __syncwarp();
    if (lane == 0) {
        if (Rec<V>::kFence)
            st_release(flag, kFlagPrefix);
        else
            st_relaxed_u32(flag, kFlagPrefix);
    }
}

// Read a record whose status was missing again until it is there (bounded by the wait that began
// at t0; false after giving up, with the error recorded).
template <typename V, bool PRE, typename R, typename O>
__device__ __forceinline__ bool reread(const R* p, O& out, unsigned long long t0, WsHeader* hdr, int info) {
    for (int it = 0;; ++it) {
        bool got;
        if constexpr (PRE)
            got = Rec<V>::get_pre(p, out);
        else
            got = Rec<V>::get_agg(p, out);
        if (got) return true;
        if (global_ns() - t0 > kWaitLimitNs) {
            record_error(hdr, LR_ERR_TIMEOUT, info);
            return false;
        }
        if (it > 16) __nanosleep(64);
    }
}

// Carry entering tile k of a row, deterministic whatever the timing.  Towards the start of the
// chain (dir = -1: earlier segments, forward pass; dir = +1: later segments, backward pass) the
// nearest tile that has published its inclusive prefix (or the end of the row) is found with
// every tile between it and k holding its aggregate; the aggregates of those tiles are then
// folded onto the prefix in chain order, x <- m x + v.  That is the same sequence of operations as
// a purely chained scan, so the result does not depend on which records happened to be ready.
//
// The warp (all 32 lanes call this) reads the flags of 32 tiles per round trip, lane i the tile at
// distance i + 1 of the window, and issues the aggregate loads KB at a time before folding them:
// a tile far down a row pays a few L2 round trips, not two per tile in between.  The wait is
// bounded; giving up records the error and yields a zero carry.
template <int KB, typename V>
__device__ __forceinline__ V lookback_carry(const unsigned int* flags, const typename Rec<V>::AggT* aggRec,
                                            const typename Rec<V>::PreT* preRec, size_t row, int k, int dir,
                                            int nseg, int CB, int lane, bool act, WsHeader* hdr, int info) {
    using R = Rec<V>;
    int dist = 0;  // distance of the window's first tile minus one
    int jp;        // the tile whose prefix starts the fold (out of range: the row's end, zero)
    const unsigned long long t0 = global_ns();
    for (int it = 0;; ++it) {
        const int j = k + dir * (dist + 1 + lane);
        const bool in = j >= 0 && j < nseg;
        const unsigned int f = in ? ld_acquire(&flags[row + j]) : (unsigned int)kFlagPrefix;
        const unsigned int pre = __ballot_sync(0xffffffffu, f == kFlagPrefix);
        const unsigned int none = __ballot_sync(0xffffffffu, f == kFlagNone);
        const int p = pre ? __ffs(pre) - 1 : 32, q = none ? __ffs(none) - 1 : 32;
        if (p < q) {  // every tile before the prefix holds its aggregate
            jp = k + dir * (dist + 1 + p);
            break;
        }
        if (q == 32) {  // a whole window of aggregates: look further
            dist += 32;
            continue;
        }
        if (global_ns() - t0 > kWaitLimitNs) {
            record_error(hdr, LR_ERR_TIMEOUT, info);
            return zero_of(V{});
        }
        if (it > 16) __nanosleep(128);
    }
    V x = zero_of(V{});
    if (jp >= 0 && jp < nseg && act) {
        const typename R::PreT* pp = &preRec[(row + jp) * CB + lane];
        if (!R::get_pre(pp, x) && !reread<V, true>(pp, x, t0, hdr, info)) return zero_of(V{});
    }
    for (int i = jp - dir; i != k;) {
        Agg<V> ag[KB];
        bool got[KB];
        int cnt = 0;
#pragma unroll
        for (int b = 0; b < KB; ++b) {
            const int ii = i - dir * b;
            const bool use = dir < 0 ? ii < k : ii > k;
            got[b] = true;
            ag[b] = Agg<V>{one_of(V{}), zero_of(V{})};
            if (use && act) got[b] = R::get_agg(&aggRec[(row + ii) * CB + lane], ag[b]);
            cnt += use ? 1 : 0;
        }
#pragma unroll
        for (int b = 0; b < KB; ++b)
            if (b < cnt) {
                if (!got[b] &&
                    !reread<V, false>(&aggRec[(row + i - dir * b) * CB + lane], ag[b], t0, hdr, info))
                    return zero_of(V{});
                x = fmax_(ag[b].m, x, ag[b].v);
            }
        i -= dir * cnt;
    }
    return x;
}

// The carry entering tile k when its neighbour k + dir has already published its inclusive prefix
// (or does not exist): read while the tile's own loads are in flight.  Returns whether every lane
// found it (otherwise the caller takes the look-back above, which yields the same value once the
// neighbour's prefix is out).
template <typename V>
__device__ __forceinline__ bool early_carry(const unsigned int* flags, const typename Rec<V>::PreT* preRec,
                                            size_t row, int k, int dir, int nseg, int CB, int lane, bool act,
                                            V& x) {
    x = zero_of(V{});
    const int j = k + dir;
    if (j < 0 || j >= nseg) return true;
    bool ready = ld_acquire(&flags[row + j]) == kFlagPrefix;
    if (ready && act) ready = Rec<V>::get_pre(&preRec[(row + j) * CB + lane], x);
    return __all_sync(0xffffffffu, ready);
}

// Dynamic shared memory, re-aligned to 128 bytes.
__device__ __forceinline__ char* smem_base() {
    extern __shared__ char dyn_smem[];
    uintptr_t p = reinterpret_cast<uintptr_t>(dyn_smem);
    return reinterpret_cast<char*>((p + 127) & ~uintptr_t(127)) ;
}

// Named barrier 1 over the whole CTA: warp 0 arrives once it has written the tile's carry and goes
// on to publish the tile's prefix and checkpoint, the other warps wait only for the carry.
__device__ __forceinline__ void carry_arrive() { asm volatile("bar.arrive 1, %0;" ::"n"(kThreads) : "memory"); }
__device__ __forceinline__ void carry_wait() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }

// Thread-block clusters: a row of at most 8 tiles runs as one cluster, and the tiles exchange their
// aggregates through distributed shared memory instead of global-memory records.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
// Arrival that only marks a CTA's reads of the other slots as done (their values are already in
// registers), so it needs no release ordering.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ Agg<float> ld_dsmem_agg(uint32_t addr, float) {
    float m, v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(m), "=f"(v) : "r"(addr) : "memory");
    return {m, v};
}
__device__ __forceinline__ Agg<cpx> ld_dsmem_agg(uint32_t addr, cpx) {
    float a, b, c, d;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(a), "=f"(b), "=f"(c), "=f"(d) : "r"(addr)
                 : "memory");
    return {{a, b}, {c, d}};
}
constexpr int kMaxCluster = 8;  // portable cluster size

// Cluster mode: the carry entering tile `seg` from the aggregates the other tiles of the row left in
// their cluster slot (dir = -1: ranks 0 .. seg - 1, folded in that order; dir = +1: ranks nseg - 1
// down to seg + 1), x <- m x + v from zero -- the same operations as the chained look-back.
// Warp 0, one lane per unit, after the cluster barrier that follows the slots' writes.
template <typename V>
__device__ __forceinline__ V cluster_carry(const Agg<V>* clAgg, int seg, int nseg, int dir, int lane, int CB) {
    V x = zero_of(V{});
    if (lane >= CB) return x;
    const uint32_t local = smem_u32(clAgg + lane);
    Agg<V> ag[kMaxCluster];
#pragma unroll
    for (int i = 0; i < kMaxCluster; ++i) {
        const int j = dir < 0 ? i : nseg - 1 - i;
        const bool use = dir < 0 ? j < seg : j > seg;
        ag[i] = use ? ld_dsmem_agg(dsmem_addr(local, j), V{}) : Agg<V>{one_of(V{}), zero_of(V{})};
    }
#pragma unroll
    for (int i = 0; i < kMaxCluster; ++i) {
        const int j = dir < 0 ? i : nseg - 1 - i;
        if (dir < 0 ? j < seg : j > seg) x = fmax_(ag[i].m, x, ag[i].v);
    }
    return x;
}

// Aggregate loads in flight in the look-back (8 spill registers in the gated forward and rotlru's
// backward tile kernels)
template <int KIND> constexpr int lookback_batch() { return KIND == LR_RGLRU ? 8 : 4; }

// Zeroes the head of the workspace (header, flags and, with real values, the tile records) and lets
// the scan kernel that follows start at once (programmatic launch): that kernel waits for this one
// only before it touches the workspace.
__global__ void ws_zero_kernel(uint4* __restrict__ p, size_t n16) {
    pdl_launch_dependents();
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// --------------------------------------------------------------------------------- forward
template <int KIND, typename T, bool FULL>
__global__ void __launch_bounds__(kThreads, KIND == LR_ROTLRU ? 4 : 2)  // tiles per SM (registers)
diag_fwd_kernel(const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapB,
                const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapY, DiagArgs a) {
    using K = Kind<KIND, T>;
    using V = typename K::V;
    using SM = Smem<KIND, T, false>;
    constexpr int CB = K::CB, NG = K::NG;
    char* sm = smem_base();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
    T* Cs = reinterpret_cast<T*>(sm + SM::off_coef());
    T* Bs = reinterpret_cast<T*>(sm + SM::off_b());
    T* Xs = reinterpret_cast<T*>(sm + SM::off_x());  // gated: x
    constexpr bool gated = KIND == kRgGated;
    Agg<V>* aggF = reinterpret_cast<Agg<V>*>(sm + SM::off_aggf());
    V* carryS = reinterpret_cast<V*>(sm + SM::off_carry());
    int* misc = reinterpret_cast<int*>(sm + SM::off_misc());

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr bool full = FULL;  // LR_FULL_STATE: checkpoint every step
    const int grp = tid / CB, u = tid % CB;

    // The tile and its loads.  The kernel starts while the workspace is being zeroed (programmatic
    // launch after ws_zero_kernel): the inputs may be read at once, the workspace only after
    // pdl_wait (record_error waits by itself).  With tiles numbered by block index the loads are
    // issued before that wait; in cluster mode there is no wait.
    auto take_tile = [&](unsigned int tk) {
        const int per_seg = a.B * a.ncb;
        const int sg = tk / per_seg, rem = tk % per_seg, bb = rem / a.ncb, cc = rem % a.ncb;
        misc[0] = sg;
        misc[1] = bb;
        misc[2] = cc;
        mbar_arrive_expect_tx(bar, (uint32_t)(a.S * (K::CW + (gated ? 2 : 1) * K::BW) * sizeof(T)));
        tma_load_3d(Cs, &mapC, bar, cc * K::CW, sg * a.S, bb);
        tma_load_3d(Bs, &mapB, bar, cc * K::BW, sg * a.S, bb);
        if (gated) tma_load_3d(Xs, &mapX, bar, cc * K::BW, sg * a.S, bb);
    };
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        if (a.cl)  // the row's tiles are the cluster's CTAs, in segment order
            take_tile((blockIdx.x % a.cl) * (a.B * a.ncb) + blockIdx.x / a.cl);
        else if (a.direct)
            take_tile(blockIdx.x);
    }
    if (!a.cl) pdl_wait();  // cluster mode touches the workspace only to record an error
    if (tid == 0 && !a.cl && !a.direct) {
        // ticket mode: the tile `ahead` (one per SM) tickets later is brought into L2 now, so its
        // loads find it there (forward rotlru tile 2.00 -> 1.86 ms; in the backward, whose dy is
        // prefetched by its own tile, the same made the kernel slower, and further ahead -- a
        // whole residency wave -- both kernels)
        const unsigned int tk = take_ticket(a.hdr, 0);
        take_tile(tk);
        const unsigned int nx = tk + (unsigned int)a.ahead;
        const int per_seg = a.B * a.ncb;
        if (a.ahead > 0 && nx < (unsigned int)(a.nseg * per_seg)) {
            const int sg = nx / per_seg, rem = nx % per_seg, bb = rem / a.ncb, cc = rem % a.ncb;
            tma_prefetch_3d(&mapC, cc * K::CW, sg * a.S, bb);
            tma_prefetch_3d(&mapB, cc * K::BW, sg * a.S, bb);
            if (gated) tma_prefetch_3d(&mapX, cc * K::BW, sg * a.S, bb);
        }
    }
    __syncthreads();
    const int seg = misc[0], b = misc[1], cb = misc[2];
    const int t0g = seg * a.S;
    const int unit = cb * CB + u;  // global unit index (channel or pair)
    const int units = K::chans_per_unit == 1 ? a.D : a.D / 2;
    const size_t row = (size_t)(b * a.ncb + cb) * a.nseg;
    auto* aggRec = reinterpret_cast<typename Rec<V>::AggT*>(a.agg);
    auto* preRec = reinterpret_cast<typename Rec<V>::PreT*>(a.pre);
    const bool act = warp == 0 && lane < CB && unit < units;
    V carry = zero_of(V{});
    bool have = false;
    if (warp == 0 && !a.cl) have = early_carry<V>(a.flags, preRec, row, seg, -1, a.nseg, CB, lane, act, carry);
    typename K::Unit U(a, unit);
    const int nt = min(a.S, a.L - t0g);
    const int spg = (a.S + NG - 1) / NG;
    const int j0 = grp * spg, j1 = min(j0 + spg, nt);
    bool ok = mbar_wait(bar, 0, a.hdr, 100);
    if constexpr (gated) {  // b = sqrt(1 - a^2) (i x) over the thread's own steps, into i's slot
        if (ok)
            for (int j = j0; j < j1; ++j) {
                const float L = IO<T>::ld(Cs + j * K::CW + u) * U.clog;  // log a
                const float bj = sqrtf(-expm1f(2.0f * L)) * IO<T>::ld(Bs + j * K::BW + u) * IO<T>::ld(Xs + j * K::BW + u);
                IO<T>::st(Bs + j * K::BW + u, bj);
            }
    }

    // group aggregate with zero carry-in
    V P = one_of(V{}), h = zero_of(V{});
    if (ok) {
        for (int j = j0; j < j1; ++j) {
            V c = U.coef(Cs, j, u);
            P = mulx(c, P);
            h = fmax_(c, h, K::ldb(Bs, j, u));
        }
    }
    aggF[grp * CB + u] = {P, h};
    __syncthreads();

    // tile carry through the chained look-back (warp 0, one lane per unit; usually known already,
    // early_carry); warp 0 then releases the other warps and publishes the tile's inclusive prefix
    // at once, since the look-backs of later tiles wait for it (the first segment's in particular)
    const bool has_succ = seg + 1 < a.nseg;
    Agg<V>* clAgg = reinterpret_cast<Agg<V>*>(sm + SM::off_cl());
    if (a.cl) {  // cluster mode: slots, barrier, fold of the earlier tiles' slots
        if (warp == 0 && lane < CB) {
            Agg<V> tile{one_of(V{}), zero_of(V{})};
            for (int g = 0; g < NG; ++g) {
                Agg<V> ag = aggF[g * CB + lane];
                tile.v = fmax_(ag.m, tile.v, ag.v);
                tile.m = mulx(ag.m, tile.m);
            }
            clAgg[lane] = tile;
        }
        cluster_arrive();
        cluster_wait();
        if (warp == 0) {
            carry = cluster_carry(clAgg, seg, a.nseg, -1, lane, CB);
            if (lane < CB) carryS[lane] = carry;
            __syncwarp();
            carry_arrive();
            cluster_arrive_relaxed();  // done reading the other tiles' slots
            const size_t slot = full ? (size_t)t0g : (size_t)seg;
            if (act) K::st_ckpt(a.ckpt + (slot * a.B + b) * a.D, unit * K::chans_per_unit, carry);
        } else {
            cluster_arrive_relaxed();
            carry_wait();
        }
    } else if (warp == 0) {
        Agg<V> tile{one_of(V{}), zero_of(V{})};
        if (lane < CB) {
            for (int g = 0; g < NG; ++g) {
                Agg<V> ag = aggF[g * CB + lane];
                tile.v = fmax_(ag.m, tile.v, ag.v);
                tile.m = mulx(ag.m, tile.m);
            }
        }
        if (!have) {
            if (seg > 0 && has_succ) {
                publish_agg<V>(&a.flags[row + seg], &aggRec[(row + seg) * CB + lane], tile, act, lane);
            }
            carry = lookback_carry<lookback_batch<KIND>(), V>(a.flags, aggRec, preRec, row, seg, -1, a.nseg, CB, lane,
                                                           act, a.hdr, 101);
        }
        if (lane < CB) carryS[lane] = carry;
        __syncwarp();
        carry_arrive();
        const bool withhold = (a.dflags & LR_TEST_WITHHOLD_CARRY) && seg == 0;
        if (has_succ && !withhold) {
            publish_pre<V>(&a.flags[row + seg], &preRec[(row + seg) * CB + lane], fmax_(tile.m, carry, tile.v), act,
                           lane);
        }
        const size_t slot = full ? (size_t)t0g : (size_t)seg;  // state entering the segment
        if (act) K::st_ckpt(a.ckpt + (slot * a.B + b) * a.D, unit * K::chans_per_unit, carry);
    } else {
        carry_wait();
    }

    // apply: recompute the group with its true carry-in, write y into the b slot
    V hh = carryS[u];
    for (int g = 0; g < grp; ++g) {
        Agg<V> ag = aggF[g * CB + u];
        hh = fmax_(ag.m, hh, ag.v);
    }
    if (ok) {
        for (int j = j0; j < j1; ++j) {
            V c = U.coef(Cs, j, u);
            hh = fmax_(c, hh, K::ldb(Bs, j, u));
            K::stb(Bs, j, u, hh);
            // full state: slot t + 1 is the state entering step t + 1 (the slot after the segment
            // is the next segment's carry, written there)
            if (full && j + 1 < a.S && t0g + j + 1 < a.L && unit < units)
                K::st_ckpt(a.ckpt + ((size_t)(t0g + j + 1) * a.B + b) * a.D, unit * K::chans_per_unit, hh);
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && ok) {
        tma_store_3d(&mapY, Bs, cb * K::BW, t0g, b);
        bulk_commit();
        bulk_wait_read_all();
    }
    if (a.cl) cluster_wait();  // no tile's slot is read after its CTA has exited
}

// -------------------------------------------------------------------------------- backward
template <int KIND, typename T, bool FULL>
__global__ void __launch_bounds__(kThreads, KIND == LR_ROTLRU ? 3 : 2)  // tiles per SM (shared memory)
diag_bwd_kernel(const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapB,
                const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapDY,
                const __grid_constant__ CUtensorMap mapDC, const __grid_constant__ CUtensorMap mapDB,
                const __grid_constant__ CUtensorMap mapDX, DiagArgs a) {
    using K = Kind<KIND, T>;
    using V = typename K::V;
    using SM = Smem<KIND, T, true>;
    constexpr int CB = K::CB, NG = K::NG;
    constexpr int SPG = kMaxSeg / NG;
    char* sm = smem_base();
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
    T* Cs = reinterpret_cast<T*>(sm + SM::off_coef());
    T* Bs = reinterpret_cast<T*>(sm + SM::off_b());
    T* Ds = reinterpret_cast<T*>(sm + SM::off_dy());
    // gated: x, and b = sqrt(1 - a^2) (i x) (the recompute's input; i stays for its gradient)
    constexpr bool gated = KIND == kRgGated;
    T* Xs = reinterpret_cast<T*>(sm + SM::off_x());
    T* Es = reinterpret_cast<T*>(sm + SM::off_e());
    T* Brec = gated ? Es : Bs;
    Agg<V>* aggF = reinterpret_cast<Agg<V>*>(sm + SM::off_aggf());
    Agg<V>* aggR = reinterpret_cast<Agg<V>*>(sm + SM::off_aggr());
    V* carryS = reinterpret_cast<V*>(sm + SM::off_carry());
    float2* red = reinterpret_cast<float2*>(sm + SM::off_red());
    int* misc = reinterpret_cast<int*>(sm + SM::off_misc());

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = tid / CB, u = tid % CB;
    // full state: the forward checkpointed every step, so the states are read, not recomputed (b
    // is not needed)
    constexpr bool full = FULL;

    // The tile (later segments first) and its loads: coefficients and b (the forward recompute) on
    // bar[0], dy (the adjoint) on bar[1].  As in the forward kernel, the workspace is touched only
    // after pdl_wait, and with tiles numbered by block index the loads are issued before it.
    auto take_tile = [&](unsigned int tk) {
        const int per_seg = a.B * a.ncb;
        const int sg = a.nseg - 1 - (int)(tk / per_seg), rem = tk % per_seg, bb = rem / a.ncb, cc = rem % a.ncb;
        misc[0] = sg;
        misc[1] = bb;
        misc[2] = cc;
        const int t0 = sg * a.S;
        mbar_arrive_expect_tx(&bar[0],
                              (uint32_t)(a.S * (K::CW + (full ? 0 : K::BW) + (gated ? K::BW : 0)) * sizeof(T)));
        tma_load_3d(Cs, &mapC, &bar[0], cc * K::CW, t0, bb);
        if (!full) tma_load_3d(Bs, &mapB, &bar[0], cc * K::BW, t0, bb);
        if (gated) tma_load_3d(Xs, &mapX, &bar[0], cc * K::BW, t0, bb);
        if (!(SM::AL && !full)) {
            mbar_arrive_expect_tx(&bar[1], (uint32_t)(a.S * K::BW * sizeof(T)));
            tma_load_3d(Ds, &mapDY, &bar[1], cc * K::BW, t0, bb);
        } else {  // dy lands in b's slot after the recompute: bring it into L2 meanwhile
            tma_prefetch_3d(&mapDY, cc * K::BW, t0, bb);
        }
    };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        if (a.cl)  // the row's tiles are the cluster's CTAs; tile numbers count later segments first
            take_tile((a.nseg - 1 - (int)(blockIdx.x % a.cl)) * (a.B * a.ncb) + blockIdx.x / a.cl);
        else if (a.direct)
            take_tile(blockIdx.x);
    }
    if (!a.cl) pdl_wait();  // cluster mode touches the workspace only for its partials (a region
                            // the zeroing leaves alone) and to record an error
    if (tid == 0 && !a.cl && !a.direct) take_tile(take_ticket(a.hdr, 1));
    __syncthreads();
    const int seg = misc[0], b = misc[1], cb = misc[2];
    const int t0g = seg * a.S;
    const int unit = cb * CB + u;
    const int units = K::chans_per_unit == 1 ? a.D : a.D / 2;
    const size_t row = (size_t)(b * a.ncb + cb) * a.nseg;
    auto* aggRec = reinterpret_cast<typename Rec<V>::AggT*>(a.agg);
    auto* preRec = reinterpret_cast<typename Rec<V>::PreT*>(a.pre);
    const bool act = warp == 0 && lane < CB && unit < units;
    V carry = zero_of(V{});
    bool have = false;
    if (warp == 0 && !a.cl) have = early_carry<V>(a.flags, preRec, row, seg, +1, a.nseg, CB, lane, act, carry);
    typename K::Unit U(a, unit);
    if (tid < CB && !full) {
        V c0 = zero_of(V{});
        if (unit < units)
            c0 = K::ld_ckpt(a.ckpt + ((size_t)seg * a.B + b) * a.D, unit * K::chans_per_unit);
        carryS[tid] = c0;
    }
    const int nt = min(a.S, a.L - t0g);
    const int spg = (a.S + NG - 1) / NG;
    const int j0 = grp * spg, j1 = min(j0 + spg, nt);
    const int n = max(j1 - j0, 0);
    bool ok = mbar_wait(&bar[0], 0, a.hdr, 200);
    if constexpr (gated) {  // b of the thread's own steps, from r, i, x
        if (ok)
            for (int j = j0; j < j1; ++j) {
                const float L = IO<T>::ld(Cs + j * K::CW + u) * U.clog;  // log a
                IO<T>::st(Es + j * K::BW + u,
                          sqrtf(-expm1f(2.0f * L)) * IO<T>::ld(Bs + j * K::BW + u) * IO<T>::ld(Xs + j * K::BW + u));
            }
    }

    // state entering each step of the group, in registers: recomputed from the segment
    // checkpoint, or (full state) read from that step's checkpoint slot
    V hprev[SPG];
    if (!full) {
        // forward aggregate of the group
        {
            V P = one_of(V{}), h = zero_of(V{});
            if (ok)
                for (int j = j0; j < j1; ++j) {
                    V c = U.coef(Cs, j, u);
                    P = mulx(c, P);
                    h = fmax_(c, h, K::ldb(Brec, j, u));
                }
            aggF[grp * CB + u] = {P, h};
        }
        __syncthreads();
        V h = carryS[u];
        for (int g = 0; g < grp; ++g) {
            Agg<V> ag = aggF[g * CB + u];
            h = fmax_(ag.m, h, ag.v);
        }
#pragma unroll
        for (int j = 0; j < SPG; ++j) {
            hprev[j] = h;
            if (j < n) {
                V c = U.coef(Cs, j0 + j, u);
                h = fmax_(c, h, K::ldb(Brec, j0 + j, u));
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < SPG; ++j)
            hprev[j] = (j < n && unit < units)
                           ? K::ld_ckpt(a.ckpt + ((size_t)(t0g + j0 + j) * a.B + b) * a.D, unit * K::chans_per_unit)
                           : zero_of(V{});
    }
    if constexpr (SM::AL && !full) {  // dy into b's slot, now that every thread is done with b
        __syncthreads();
        if (tid == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar[1], (uint32_t)(a.S * K::BW * sizeof(T)));
            tma_load_3d(Ds, &mapDY, &bar[1], cb * K::BW, t0g, b);
        }
    }
    // reverse aggregate of the group: outgoing carry = v + m * incoming
    ok = mbar_wait(&bar[1], 0, a.hdr, 202) && ok;
    {
        V M = one_of(V{}), r = zero_of(V{});
        if (ok)
            for (int j = j1 - 1; j >= j0; --j) {
                V cc = conjx(U.coef(Cs, j, u));
                V G = addx(K::ldb(Ds, j, u), r);
                r = mulx(cc, G);
                M = mulx(cc, M);
            }
        aggR[grp * CB + u] = {M, r};
    }
    __syncthreads();

    // tile carry from later segments (warp 0; usually known already), then the other warps are
    // released and the tile's prefix published, as in the forward kernel
    const bool has_pred = seg > 0;  // earlier segment waits on this one
    Agg<V>* clAgg = reinterpret_cast<Agg<V>*>(sm + SM::off_cl());
    if (a.cl) {  // cluster mode, as in the forward kernel (the later tiles' slots)
        if (warp == 0 && lane < CB) {
            Agg<V> tile{one_of(V{}), zero_of(V{})};
            for (int g = NG - 1; g >= 0; --g) {
                Agg<V> ag = aggR[g * CB + lane];
                tile.v = fmax_(ag.m, tile.v, ag.v);
                tile.m = mulx(ag.m, tile.m);
            }
            clAgg[lane] = tile;
        }
        cluster_arrive();
        cluster_wait();
        if (warp == 0) {
            carry = cluster_carry(clAgg, seg, a.nseg, +1, lane, CB);
            if (lane < CB) carryS[CB + lane] = carry;
            __syncwarp();
            carry_arrive();
            cluster_arrive_relaxed();
        } else {
            cluster_arrive_relaxed();
            carry_wait();
        }
    } else if (warp == 0) {
        Agg<V> tile{one_of(V{}), zero_of(V{})};
        if (lane < CB)
            for (int g = NG - 1; g >= 0; --g) {
                Agg<V> ag = aggR[g * CB + lane];
                tile.v = fmax_(ag.m, tile.v, ag.v);
                tile.m = mulx(ag.m, tile.m);
            }
        if (!have) {
            if (has_pred && seg + 1 < a.nseg) {
                publish_agg<V>(&a.flags[row + seg], &aggRec[(row + seg) * CB + lane], tile, act, lane);
            }
            carry = lookback_carry<lookback_batch<KIND>(), V>(a.flags, aggRec, preRec, row, seg, +1, a.nseg, CB, lane,
                                                           act, a.hdr, 201);
        }
        if (lane < CB) carryS[CB + lane] = carry;
        __syncwarp();
        carry_arrive();
        const bool withhold = (a.dflags & LR_TEST_WITHHOLD_CARRY) && seg == a.nseg - 1;
        if (has_pred && !withhold) {
            publish_pre<V>(&a.flags[row + seg], &preRec[(row + seg) * CB + lane], fmax_(tile.m, carry, tile.v), act,
                           lane);
        }
    } else {
        carry_wait();
    }

    // adjoint sweep of the group with its true carry; gradients into the shared slots
    V r = carryS[CB + u];
    for (int g = NG - 1; g > grp; --g) {
        Agg<V> ag = aggR[g * CB + u];
        r = fmax_(ag.m, r, ag.v);
    }
    float acc_mag = 0.0f, acc_th = 0.0f;
#pragma unroll
    for (int jj = SPG - 1; jj >= 0; --jj) {
        if (jj < n && ok) {
            const int j = j0 + jj;
            V G = addx(K::ldb(Ds, j, u), r);
            const V hp = hprev[jj];
            if constexpr (KIND == LR_RGLRU) {
                float c = IO<T>::ld(Cs + j * K::CW + u);
                IO<T>::st(Ds + j * K::BW + u, G);       // db
                IO<T>::st(Cs + j * K::CW + u, G * hp);  // da
                r = c * G;
            } else if constexpr (gated) {
                // db = G, da = G h_{t-1}, carried through b = s (i x), s = sqrt(1 - a^2), and
                // a = e^{c r log sigmoid(Lambda)}: ds/da = -a / s
                const float rg = IO<T>::ld(Cs + j * K::CW + u);
                const float L = rg * U.clog;
                const float av = expf(L), sv = sqrtf(-expm1f(2.0f * L));
                const float iv = IO<T>::ld(Bs + j * K::BW + u), xv = IO<T>::ld(Xs + j * K::BW + u);
                const float da_tot = G * hp - G * iv * xv * av / sv;
                IO<T>::st(Bs + j * K::BW + u, G * sv * xv);           // di
                IO<T>::st(Xs + j * K::BW + u, G * sv * iv);           // dx
                IO<T>::st(Cs + j * K::CW + u, da_tot * av * U.clog);  // dr
                acc_mag = fmaf(da_tot * av * kRgC * rg, U.oms, acc_mag);  // dLambda
                r = av * G;
            } else {
                float gt = IO<T>::ld(Cs + j * K::CW + u);
                float m = U.mag * gt;
                cpx lam{m * U.cs, m * U.sn};
                K::stb(Ds, j, u, G);                               // db
                cpx dl = cmul(G, conjc(hp));                        // dlambda = G conj(h_{t-1})
                float dm = fmaf(dl.r, U.cs, dl.i * U.sn);           // Re(dlambda e^{-i theta})
                IO<T>::st(Cs + j * K::CW + u, U.mag * dm);          // dg
                acc_mag = fmaf(gt, dm, acc_mag);
                acc_th = fmaf(m, fmaf(dl.i, U.cs, -dl.r * U.sn), acc_th);
                r = cmul(conjc(lam), G);
            }
        }
    }
    if constexpr (KIND == LR_ROTLRU || gated) {
        red[grp * CB + u] = make_float2(acc_mag, acc_th);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if constexpr (KIND == LR_ROTLRU || gated) {  // rotlru: dmag, dtheta; gated rglru: dLambda
        if (tid < CB && unit < units) {
            float sm_ = 0.0f, st_ = 0.0f;
            for (int g = 0; g < NG; ++g) {
                float2 v = red[g * CB + tid];
                sm_ += v.x;
                st_ += v.y;
            }
            a.partial[((size_t)b * a.nseg + seg) * units + unit] = make_float2(sm_, st_);
        }
    }
    if (tid == 0 && ok) {
        tma_store_3d(&mapDC, Cs, cb * K::CW, t0g, b);
        if constexpr (gated) {
            tma_store_3d(&mapDB, Bs, cb * K::BW, t0g, b);  // di
            tma_store_3d(&mapDX, Xs, cb * K::BW, t0g, b);  // dx
        } else {
            tma_store_3d(&mapDB, Ds, cb * K::BW, t0g, b);
        }
        bulk_commit();
        bulk_wait_read_all();
    }
    if (a.cl) cluster_wait();  // no tile's slot is read after its CTA has exited
}

// Fixed-order reduction of rotlru's per-tile parameter partials over (batch row, segment).  A
// block owns kRedPairs pairs; its kRedSlices slices each sum every kRedSlices-th row (rows in
// increasing order), and the slices are then folded by a fixed pairwise tree, so the result does
// not depend on timing.
constexpr int kRedPairs = 16, kRedSlices = 64;
__global__ void __launch_bounds__(kRedPairs * kRedSlices)
rotlru_param_reduce(const float2* __restrict__ partial, int rows, int K, float* __restrict__ dmag,
                    float* __restrict__ dtheta) {
    __shared__ float2 red[kRedSlices][kRedPairs];
    const int x = threadIdx.x % kRedPairs, y = threadIdx.x / kRedPairs;
    const int k = blockIdx.x * kRedPairs + x;
    float2 acc = make_float2(0.0f, 0.0f);
    if (k < K) {
#pragma unroll 8
        for (int r = y; r < rows; r += kRedSlices) {
            const float2 v = __ldg(&partial[(size_t)r * K + k]);
            acc.x += v.x;
            acc.y += v.y;
        }
    }
    red[y][x] = acc;
    __syncthreads();
#pragma unroll
    for (int off = kRedSlices / 2; off > 0; off >>= 1) {
        if (y < off) {
            red[y][x].x += red[y + off][x].x;
            red[y][x].y += red[y + off][x].y;
        }
        __syncthreads();
    }
    if (y == 0 && k < K) {
        dmag[k] = red[0][x].x;
        if (dtheta) dtheta[k] = red[0][x].y;
    }
}

// ------------------------------------------------------------------------------ host side
struct Geo {
    int nseg, ncb, tiles, cb;
};

Geo geo(const lr_desc& d) {
    Geo g;
    g.nseg = (int)((d.L + d.segment - 1) / d.segment);
    int units = d.kind == LR_RGLRU ? (int)d.D : (int)(d.D / 2);
    // units per tile: the kernels' tile width (the same for both I/O types)
    g.cb = d.kind == LR_ROTLRU                  ? Kind<LR_ROTLRU, float>::CB
           : (d.flags & LR_RGLRU_GATES) != 0 ? Kind<kRgGated, float>::CB
                                             : Kind<LR_RGLRU, float>::CB;
    static_assert(Kind<LR_RGLRU, float>::CB == Kind<LR_RGLRU, __nv_bfloat16>::CB &&
                      Kind<LR_ROTLRU, float>::CB == Kind<LR_ROTLRU, __nv_bfloat16>::CB,
                  "tile width independent of the I/O type");
    g.ncb = (units + g.cb - 1) / g.cb;
    g.tiles = (int)d.B * g.ncb * g.nseg;
    return g;
}

// Tiles may be numbered by block index, instead of by a ticket taken as each CTA starts, when the
// grid has at most one CTA per SM: all of its CTAs can then be resident together, so a tile that
// waits for another never keeps it from starting, whatever order the CTAs start in.  The ticket
// costs a global atomic round trip before the tile's loads can be issued.
bool direct_tiles(const Geo& g) { return g.tiles <= device_sm_count(); }

// A row of 2 .. 8 tiles runs as one thread-block cluster (cluster mode): its tiles exchange
// aggregates through distributed shared memory, with no global records, flags or waits on other
// CTAs.  Longer rows take the look-back, and so do calls with the failure-path test flag (a
// withheld carry needs the look-back's bounded waits) or the look-back test flag.
int cluster_size(const lr_desc& d, const Geo& g) {
    if (d.flags & (LR_TEST_WITHHOLD_CARRY | LR_TEST_LOOKBACK)) return 0;
    return (g.nseg >= 2 && g.nseg <= kMaxCluster) ? g.nseg : 0;
}

struct DiagWs {
    size_t flags, agg, pre, zero_end, partial, end;
};

// Workspace: flags, then the tiles' aggregate and prefix records (8 bytes per unit and record
// value: a complex value, or a real value with its status word), then partials.  Zeroed before each
// call: the flags, and with real values the records too (their status words).
DiagWs ws_plan(const lr_desc& d, bool bwd) {
    Geo g = geo(d);
    const size_t vs = 8;
    WsCursor c;
    DiagWs w;
    w.flags = c.take(sizeof(unsigned int) * g.tiles);
    w.agg = c.take(2 * vs * g.cb * (size_t)g.tiles);
    w.pre = c.take(vs * g.cb * (size_t)g.tiles);
    w.zero_end = d.kind == LR_RGLRU ? c.off : w.agg;
    const bool gates = d.kind == LR_RGLRU && (d.flags & LR_RGLRU_GATES);
    w.partial = (bwd && (d.kind == LR_ROTLRU || gates))
                    ? c.take(sizeof(float2) * d.B * g.nseg * (d.kind == LR_ROTLRU ? d.D / 2 : d.D))
                    : 0;
    w.end = c.off;
    return w;
}

// Zero the workspace head the scan kernel relies on (ws_zero_kernel; the scan kernel is launched
// after it as a programmatic dependent).
lr_status zero_ws(const lr_desc& d, bool bwd, char* ws, cudaStream_t st) {
    const size_t n16 = (cluster_size(d, geo(d)) ? 256 : ws_plan(d, bwd).zero_end) / 16;  // cluster mode: header
    const int blocks = (int)std::min<size_t>((n16 + 255) / 256, (size_t)4 * device_sm_count());
    note_launch("diag_ws_zero");
    ws_zero_kernel<<<std::max(blocks, 1), 256, 0, st>>>(reinterpret_cast<uint4*>(ws), n16);
    return check_launch();
}

// The dynamic shared-memory limit is a per-device attribute of the function, so it is set on every
// call (a host-side call of about a microsecond): a process may drive several devices.
template <int KIND, typename T, bool BWD, bool FULL>
void set_smem_attr(const void* fn) {
    cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem<KIND, T, BWD>::total());
}

template <int KIND, typename T>
lr_status launch_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                     cudaStream_t st) {
    using K = Kind<KIND, T>;
    Geo g = geo(d);
    DiagWs w = ws_plan(d, false);
    const int es = sizeof(T);
    constexpr bool rg = KIND != LR_ROTLRU;
    CUtensorMap mC, mB, mX, mY;
    const void* coef = rg ? in.a : in.g;
    uint64_t coefC = rg ? d.D : d.D / 2;
    bool ok = make_tmap_3d(&mC, coef, es, coefC, d.L, d.B, K::CW, d.segment) &&
              make_tmap_3d(&mB, in.b, es, d.D, d.L, d.B, K::BW, d.segment) &&
              make_tmap_3d(&mY, y, es, d.D, d.L, d.B, K::BW, d.segment);
    if (KIND == kRgGated)
        ok = ok && make_tmap_3d(&mX, in.x, es, d.D, d.L, d.B, K::BW, d.segment);
    else
        mX = mB;  // not read
    if (!ok) return LR_ERR_INVALID_ARG;
    const int cl = cluster_size(d, g);
    DiagArgs a{(int)d.B, (int)d.L, (int)d.D, d.segment, g.nseg, g.ncb, d.flags, direct_tiles(g), cl,
               device_sm_count(), in.mag, in.theta, in.A, (float*)ckpt, (WsHeader*)ws,
               (unsigned int*)(ws + w.flags), ws + w.agg, ws + w.pre, nullptr};
    const bool full = (d.flags & LR_FULL_STATE) != 0;
    auto fn = full ? diag_fwd_kernel<KIND, T, true> : diag_fwd_kernel<KIND, T, false>;
    if (full)
        set_smem_attr<KIND, T, false, true>((const void*)fn);
    else
        set_smem_attr<KIND, T, false, false>((const void*)fn);
    lr_status s = zero_ws(d, false, ws, st);
    if (s != LR_OK) return s;
    note_launch(KIND == LR_RGLRU ? "rglru_fwd_tile" : KIND == kRgGated ? "rglru_gated_fwd_tile" : "rotlru_fwd_tile");
    if (launch_cluster_ex(fn, dim3(g.tiles), dim3(kThreads), Smem<KIND, T, false>::total(), st, true, cl, mC, mB, mX,
                          mY, a) != cudaSuccess)
        return LR_ERR_CUDA;
    return check_launch();
}

template <int KIND, typename T>
lr_status launch_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                     const lr_grads& gr, char* ws, cudaStream_t st) {
    using K = Kind<KIND, T>;
    Geo g = geo(d);
    DiagWs w = ws_plan(d, true);
    const int es = sizeof(T);
    constexpr bool rg = KIND != LR_ROTLRU;
    CUtensorMap mC, mB, mX, mDY, mDC, mDB, mDX;
    const void* coef = rg ? in.a : in.g;
    void* dcoef = rg ? gr.da : gr.dg;
    uint64_t coefC = rg ? d.D : d.D / 2;
    bool ok = make_tmap_3d(&mC, coef, es, coefC, d.L, d.B, K::CW, d.segment) &&
              make_tmap_3d(&mB, in.b, es, d.D, d.L, d.B, K::BW, d.segment) &&
              make_tmap_3d(&mDY, dy, es, d.D, d.L, d.B, K::BW, d.segment) &&
              make_tmap_3d(&mDC, dcoef, es, coefC, d.L, d.B, K::CW, d.segment) &&
              make_tmap_3d(&mDB, gr.db, es, d.D, d.L, d.B, K::BW, d.segment);
    if (KIND == kRgGated) {
        ok = ok && make_tmap_3d(&mX, in.x, es, d.D, d.L, d.B, K::BW, d.segment) &&
             make_tmap_3d(&mDX, gr.dx, es, d.D, d.L, d.B, K::BW, d.segment);
    } else {
        mX = mB;  // not read
        mDX = mDB;  // not written
    }
    if (!ok) return LR_ERR_INVALID_ARG;
    const int cl = cluster_size(d, g);
    DiagArgs a{(int)d.B, (int)d.L, (int)d.D, d.segment, g.nseg, g.ncb, d.flags, direct_tiles(g), cl, 0, in.mag,
               in.theta, in.A, (float*)ckpt, (WsHeader*)ws, (unsigned int*)(ws + w.flags), ws + w.agg, ws + w.pre,
               w.partial ? (float2*)(ws + w.partial) : nullptr};
    const bool full = (d.flags & LR_FULL_STATE) != 0;
    auto fn = full ? diag_bwd_kernel<KIND, T, true> : diag_bwd_kernel<KIND, T, false>;
    if (full)
        set_smem_attr<KIND, T, true, true>((const void*)fn);
    else
        set_smem_attr<KIND, T, true, false>((const void*)fn);
    lr_status s = zero_ws(d, true, ws, st);
    if (s != LR_OK) return s;
    note_launch(KIND == LR_RGLRU ? "rglru_bwd_tile" : KIND == kRgGated ? "rglru_gated_bwd_tile" : "rotlru_bwd_tile");
    if (launch_cluster_ex(fn, dim3(g.tiles), dim3(kThreads), Smem<KIND, T, true>::total(), st, true, cl, mC, mB, mX,
                          mDY, mDC, mDB, mDX, a) != cudaSuccess)
        return LR_ERR_CUDA;
    s = check_launch();
    if (s != LR_OK) return s;
    if (KIND == LR_ROTLRU) {
        int K2 = (int)(d.D / 2);
        note_launch("rotlru_param_reduce");
        rotlru_param_reduce<<<(K2 + kRedPairs - 1) / kRedPairs, kRedPairs * kRedSlices, 0, st>>>(
            a.partial, (int)d.B * g.nseg, K2, gr.dmag, gr.dtheta);
        s = check_launch();
    } else if (KIND == kRgGated && gr.dA) {  // dLambda: the same fixed-order reduction, one value
        int K1 = (int)d.D;
        note_launch("rglru_param_reduce");
        rotlru_param_reduce<<<(K1 + kRedPairs - 1) / kRedPairs, kRedPairs * kRedSlices, 0, st>>>(
            a.partial, (int)d.B * g.nseg, K1, gr.dA, nullptr);
        s = check_launch();
    }
    return s;
}

}  // namespace

size_t diag_ws_bytes(const lr_desc& d, bool bwd) { return ws_plan(d, bwd).end; }
size_t diag_flag_bytes(const lr_desc& d, bool bwd) { return ws_plan(d, bwd).zero_end; }

lr_status diag_fwd(const lr_desc& d, const lr_inputs& in, void* y, void* ckpt, char* ws,
                   cudaStream_t st) {
    if (d.kind == LR_RGLRU && (d.flags & LR_RGLRU_GATES)) return launch_fwd<kRgGated, float>(d, in, y, ckpt, ws, st);
    if (d.kind == LR_RGLRU)
        return d.io == LR_F32 ? launch_fwd<LR_RGLRU, float>(d, in, y, ckpt, ws, st)
                              : launch_fwd<LR_RGLRU, __nv_bfloat16>(d, in, y, ckpt, ws, st);
    return d.io == LR_F32 ? launch_fwd<LR_ROTLRU, float>(d, in, y, ckpt, ws, st)
                          : launch_fwd<LR_ROTLRU, __nv_bfloat16>(d, in, y, ckpt, ws, st);
}

lr_status diag_bwd(const lr_desc& d, const lr_inputs& in, const void* dy, const void* ckpt,
                   const lr_grads& gr, char* ws, cudaStream_t st) {
    if (d.kind == LR_RGLRU && (d.flags & LR_RGLRU_GATES))
        return launch_bwd<kRgGated, float>(d, in, dy, ckpt, gr, ws, st);
    if (d.kind == LR_RGLRU)
        return d.io == LR_F32 ? launch_bwd<LR_RGLRU, float>(d, in, dy, ckpt, gr, ws, st)
                              : launch_bwd<LR_RGLRU, __nv_bfloat16>(d, in, dy, ckpt, gr, ws, st);
    return d.io == LR_F32 ? launch_bwd<LR_ROTLRU, float>(d, in, dy, ckpt, gr, ws, st)
                          : launch_bwd<LR_ROTLRU, __nv_bfloat16>(d, in, dy, ckpt, gr, ws, st);
}

}  // namespace lrs
