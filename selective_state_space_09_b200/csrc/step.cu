// step.cu -- decode and continuation: the recurrence advanced by L steps from a given state,
// forward only, no checkpoints (h_t = a_t (.) h_{t-1} + b_t, y_t = readout(h_t) of the
// "mlx-recurrence" post, Apple Developer Forums thread 840535, opening paragraphs and "Current
// kernels"; one token at a time is the decode mode of the mlx-mamba post, K-Search / mlx-mamba
// blog post, techtrendfeed repost, the decode paragraph after Table 1).
//
// The state is f32 in the kind's state layout and stays in registers across the call's steps:
//   rglru   [B, D]        one thread per channel
//   rotlru  [B, D]        one thread per complex pair (re, im interleaved)
//   S6      [B, D, N]     one thread per (b, d, n), N <= 32, the readout reduced by shuffles
//   SSD     [B, H, N, P]  matrix state S[n][p] (the layout of the checkpoint slots), and
//   GLA     [B, H, K, V]  S[k][v]: one kernel for both, since an SSD step is a GLA step with
//                         q = C_t, k = beta_t B_t, v = x_t and forget gate abar_t; one CTA per
//                         (b, h, 32 columns), 8 slices of the K (N) rows, K <= 128.
// Everything is fp32 (ZOH beta through expm1f); a step-by-step run matches the scan within the
// rounding of the scan's own blocking.
#include "common.cuh"
#include "host_common.h"

namespace lrs {
namespace {

constexpr float kLog2eS = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {  // 2^x, the MUFU approximation
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------------ diagonal kinds
// GATES: the RG-LRU gate front-end -- a holds the recurrence gate r, b the input gate i, and the
// step is h = a h + sqrt(1 - a^2) (i x) with a = sigmoid(Lambda)^(8 r), formed in the log domain
template <typename T, bool GATES>
__global__ void __launch_bounds__(256)
rglru_step_kernel(const T* __restrict__ a, const T* __restrict__ b, const T* __restrict__ x,
                  const float* __restrict__ lam, T* __restrict__ y, const float* s_in, float* s_out, int B, int L,
                  int D) {
    const size_t u = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (size_t)B * D) return;
    const int bi = (int)(u / D), d = (int)(u % D);
    float clog = 0.0f;  // 8 log sigmoid(Lambda)
    if (GATES) clog = -8.0f * log1pf(expf(-lam[d]));
    float h = s_in ? s_in[u] : 0.0f;
    for (int t = 0; t < L; ++t) {
        const size_t i = ((size_t)bi * L + t) * D + d;
        if (GATES) {
            const float Lg = IO<T>::ld(a + i) * clog;
            h = fmaf(expf(Lg), h, sqrtf(-expm1f(2.0f * Lg)) * IO<T>::ld(b + i) * IO<T>::ld(x + i));
        } else {
            h = fmaf(IO<T>::ld(a + i), h, IO<T>::ld(b + i));
        }
        IO<T>::st(y + i, h);
    }
    s_out[u] = h;
}

template <typename T>
__global__ void __launch_bounds__(256)
rotlru_step_kernel(const T* __restrict__ b, const T* __restrict__ g, const float* __restrict__ mag,
                   const float* __restrict__ theta, T* __restrict__ y, const float* s_in, float* s_out, int B,
                   int L, int D) {
    const int K = D / 2;
    const size_t u = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (size_t)B * K) return;
    const int bi = (int)(u / K), k = (int)(u % K);
    float sn, cs;
    sincosf(theta[k], &sn, &cs);
    const float mg = mag[k];
    cpx h = s_in ? cpx{s_in[2 * u], s_in[2 * u + 1]} : cpx{0.0f, 0.0f};
    for (int t = 0; t < L; ++t) {
        const float m = mg * IO<T>::ld(g + ((size_t)bi * L + t) * K + k);
        const size_t i = ((size_t)bi * L + t) * D + 2 * k;
        const float2 bv = IO<T>::ld2(b + i);
        h = cfma(cpx{m * cs, m * sn}, h, cpx{bv.x, bv.y});
        IO<T>::st2(y + i, make_float2(h.r, h.i));
    }
    s_out[2 * u] = h.r;
    s_out[2 * u + 1] = h.i;
}

// --------------------------------------------------------------------------------- S6
// abar, beta of one (dt, A): ZOH (exact zero-order hold), dirac (beta = 1), ZOH-Euler (beta = dt)
// or bilinear (Tustin).
__device__ __forceinline__ void disc_coef(int disc, float dt, float A, float& ab, float& be) {
    if (disc != LR_DISC_BILINEAR) {
        const float u = dt * A;
        ab = ex2(u * kLog2eS);
        be = disc == LR_DISC_ZOH ? (A != 0.0f ? expm1f(u) / A : dt) : (disc == LR_DISC_DIRAC ? 1.0f : dt);
    } else {
        const float u = 0.5f * dt * A, r = 1.0f / (1.0f - u);
        ab = (1.0f + u) * r;
        be = dt * r;
    }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + ex2(-z * kLog2eS)); }

// dt from the raw delta: itself, or softplus(delta + bias) (LR_DELTA_SOFTPLUS; bias may be null)
__device__ __forceinline__ float step_dt(float raw, int softplus, const float* bias, int i) {
    if (!softplus) return raw;
    const float v = raw + (bias ? bias[i] : 0.0f);
    return v > 20.0f ? v : log1pf(expf(v));
}

constexpr int kS6MaxN = 32;

// One thread per (b, d, n): NL lanes (a power of two >= N, at most 32) per channel, the readout
// sum over n by butterfly shuffles within those lanes (lanes n >= N hold zero).
template <typename T>
__global__ void __launch_bounds__(256)
s6_step_kernel(const T* __restrict__ x, const T* __restrict__ delta, const float* __restrict__ A,
               const T* __restrict__ Bm, const T* __restrict__ Cm, const float* __restrict__ Dskip,
               const T* __restrict__ z, T* __restrict__ y, const float* s_in, float* s_out, int B, int L, int D,
               int N, int NL, int disc, int softplus, const float* __restrict__ dbias) {
    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t u = gtid / NL;  // channel (b, d)
    const int n = (int)(gtid % NL);
    const bool live = u < (size_t)B * D;  // whole groups of NL lanes share this
    const bool act = live && n < N;
    const int bi = live ? (int)(u / D) : 0, d = live ? (int)(u % D) : 0;
    float h = (act && s_in) ? s_in[u * N + n] : 0.0f;
    const float An = act ? A[(size_t)d * N + n] : 0.0f;
    const float Dd = (live && Dskip) ? Dskip[d] : 0.0f;
    for (int t = 0; t < L; ++t) {
        const size_t i = ((size_t)bi * L + t) * D + d;
        float xv = 0.0f, s = 0.0f;
        if (act) {
            const size_t bt = ((size_t)bi * L + t) * N + n;
            xv = IO<T>::ld(x + i);
            float ab, be;
            disc_coef(disc, step_dt(IO<T>::ld(delta + i), softplus, dbias, d), An, ab, be);
            h = fmaf(ab, h, be * IO<T>::ld(Bm + bt) * xv);
            s = IO<T>::ld(Cm + bt) * h;
        }
        for (int o = NL / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o, NL);
        if (live && n == 0) {
            s = fmaf(Dd, xv, s);
            if (z) s *= silu_f(IO<T>::ld(z + i));
            IO<T>::st(y + i, s);
        }
    }
    if (act) s_out[u * N + n] = h;
}

// ------------------------------------------------------------------- SSD / GLA matrix state
constexpr int kMatCols = 32, kMatSlices = 8, kMatMaxK = 128, kMatRows = kMatMaxK / kMatSlices;

struct MatStepArgs {
    int B, L, H, K, V, G, HpG;  // K: state rows (GLA K, SSD N); V: columns (GLA V, SSD P)
    int ssd, disc, softplus;
    const void *q, *k, *v, *g;  // GLA: q, k [B,L,H,K]; v [B,L,H,V]; g [B,L,H]
    const void *x, *dt, *Bm, *Cm, *z;  // SSD: x, z [B,L,H,P]; dt [B,L,H]; Bm, Cm [B,L,G,N]
    const float *A, *Dskip, *dbias;
    void* y;                    // [B, L, H, V]
    const float* s_in;          // [B, H, K, V] or null
    float* s_out;
};

// One CTA per (b, h, block of kMatCols columns); thread (c, r): column c of the block, rows
// r, r + kMatSlices, ... of the state.  Per step: the step's row vectors (q, k) and the gate in
// shared memory, S <- g S + k v^T, partial readouts summed over the row slices in a fixed order.
template <typename T>
__global__ void __launch_bounds__(kMatCols * kMatSlices)
mat_step_kernel(MatStepArgs a) {
    __shared__ float qs[kMatMaxK], ks[kMatMaxK], part[kMatSlices][kMatCols];
    __shared__ float gsh;
    const int tid = threadIdx.x, c = tid % kMatCols, r0 = tid / kMatCols;
    const int ncb = (a.V + kMatCols - 1) / kMatCols;
    const int cb = blockIdx.x % ncb, bh = blockIdx.x / ncb, bi = bh / a.H, h = bh % a.H;
    const int col = cb * kMatCols + c;
    const bool cok = col < a.V;
    const size_t sbase = (size_t)bh * a.K * a.V;
    float S[kMatRows];
#pragma unroll
    for (int j = 0; j < kMatRows; ++j) {
        const int row = r0 + kMatSlices * j;
        S[j] = (a.s_in && cok && row < a.K) ? a.s_in[sbase + (size_t)row * a.V + col] : 0.0f;
    }
    const float Ah = a.ssd ? a.A[h] : 0.0f, Dh = (a.ssd && a.Dskip) ? a.Dskip[h] : 0.0f;
    for (int t = 0; t < a.L; ++t) {
        const size_t bt = (size_t)bi * a.L + t;
        if (a.ssd) {
            float ab, be;
            disc_coef(a.disc, step_dt(IO<T>::ld((const T*)a.dt + bt * a.H + h), a.softplus, a.dbias, h), Ah, ab, be);
            const int gi = h / a.HpG;
            const T* Bt = (const T*)a.Bm + (bt * a.G + gi) * a.K;
            const T* Ct = (const T*)a.Cm + (bt * a.G + gi) * a.K;
            for (int i = tid; i < a.K; i += blockDim.x) {
                ks[i] = be * IO<T>::ld(Bt + i);
                qs[i] = IO<T>::ld(Ct + i);
            }
            if (tid == 0) gsh = ab;
        } else {
            const T* qt = (const T*)a.q + (bt * a.H + h) * a.K;
            const T* kt = (const T*)a.k + (bt * a.H + h) * a.K;
            for (int i = tid; i < a.K; i += blockDim.x) {
                ks[i] = IO<T>::ld(kt + i);
                qs[i] = IO<T>::ld(qt + i);
            }
            if (tid == 0) gsh = IO<T>::ld((const T*)a.g + bt * a.H + h);
        }
        const T* vrow = (const T*)(a.ssd ? a.x : a.v) + (bt * a.H + h) * a.V;
        const float vv = cok ? IO<T>::ld(vrow + col) : 0.0f;
        __syncthreads();
        const float gt = gsh;
        float o = 0.0f;
#pragma unroll
        for (int j = 0; j < kMatRows; ++j) {
            const int row = r0 + kMatSlices * j;
            if (row < a.K) {
                S[j] = fmaf(gt, S[j], ks[row] * vv);
                o = fmaf(S[j], qs[row], o);
            }
        }
        part[r0][c] = o;
        __syncthreads();
        if (r0 == 0 && cok) {
            float s = 0.0f;
#pragma unroll
            for (int j = 0; j < kMatSlices; ++j) s += part[j][c];
            T* yp = (T*)a.y + (bt * a.H + h) * a.V + col;
            if (a.ssd) {
                s = fmaf(Dh, vv, s);
                if (a.z) s *= silu_f(IO<T>::ld((const T*)a.z + (bt * a.H + h) * a.V + col));
            }
            IO<T>::st(yp, s);
        }
        __syncthreads();  // the step's vectors and partials are free again
    }
#pragma unroll
    for (int j = 0; j < kMatRows; ++j) {
        const int row = r0 + kMatSlices * j;
        if (cok && row < a.K) a.s_out[sbase + (size_t)row * a.V + col] = S[j];
    }
}

template <typename T>
lr_status step_impl(const lr_desc& d, const lr_inputs& in, const float* s_in, float* s_out, void* y,
                    cudaStream_t st) {
    const int B = (int)d.B, L = (int)d.L;
    switch (d.kind) {
        case LR_RGLRU: {
            const size_t n = (size_t)d.B * d.D;
            const unsigned grid = (unsigned)((n + 255) / 256);
            if (d.flags & LR_RGLRU_GATES) {
                note_launch("rglru_gated_step");
                rglru_step_kernel<T, true><<<grid, 256, 0, st>>>((const T*)in.a, (const T*)in.b, (const T*)in.x,
                                                                 in.A, (T*)y, s_in, s_out, B, L, (int)d.D);
            } else {
                note_launch("rglru_step");
                rglru_step_kernel<T, false><<<grid, 256, 0, st>>>((const T*)in.a, (const T*)in.b, nullptr,
                                                                  nullptr, (T*)y, s_in, s_out, B, L, (int)d.D);
            }
            return check_launch();
        }
        case LR_ROTLRU: {
            const size_t n = (size_t)d.B * (d.D / 2);
            note_launch("rotlru_step");
            rotlru_step_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
                (const T*)in.b, (const T*)in.g, in.mag, in.theta, (T*)y, s_in, s_out, B, L, (int)d.D);
            return check_launch();
        }
        case LR_S6: {
            int NL = 1;
            while (NL < d.N) NL *= 2;
            const size_t n = (size_t)d.B * d.D * NL;
            note_launch("s6_step");
            s6_step_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(
                (const T*)in.x, (const T*)in.delta, in.A, (const T*)in.Bm, (const T*)in.Cm,
                (d.flags & LR_HAS_DSKIP) ? in.Dskip : nullptr, (d.flags & LR_HAS_Z) ? (const T*)in.z : nullptr,
                (T*)y, s_in, s_out, B, L, (int)d.D, (int)d.N, NL, (int)d.disc, (d.flags & LR_DELTA_SOFTPLUS) ? 1 : 0,
                in.delta_bias);
            return check_launch();
        }
        default: {
            MatStepArgs a{};
            a.B = B;
            a.L = L;
            a.H = (int)d.H;
            a.K = (int)d.N;
            a.V = (int)d.P;
            a.ssd = d.kind == LR_SSD;
            a.disc = (int)d.disc;
            a.G = a.ssd ? (int)d.G : 1;
            a.HpG = (int)(d.H / a.G);
            a.q = in.q;
            a.k = in.k;
            a.v = in.v;
            a.g = in.g;
            a.x = in.x;
            a.dt = in.delta;
            a.Bm = in.Bm;
            a.Cm = in.Cm;
            a.z = (a.ssd && (d.flags & LR_HAS_Z)) ? in.z : nullptr;
            a.A = in.A;
            a.Dskip = (a.ssd && (d.flags & LR_HAS_DSKIP)) ? in.Dskip : nullptr;
            a.softplus = (a.ssd && (d.flags & LR_DELTA_SOFTPLUS)) ? 1 : 0;
            a.dbias = a.softplus ? in.delta_bias : nullptr;
            a.y = y;
            a.s_in = s_in;
            a.s_out = s_out;
            const int ncb = (a.V + kMatCols - 1) / kMatCols;
            note_launch(a.ssd ? "ssd_step" : "gla_step");
            mat_step_kernel<T><<<(unsigned)((size_t)B * a.H * ncb), kMatCols * kMatSlices, 0, st>>>(a);
            return check_launch();
        }
    }
}

}  // namespace

bool step_supported(const lr_desc& d) {
    switch (d.kind) {
        case LR_S6: return d.N <= kS6MaxN;
        case LR_SSD:
        case LR_GLA: return d.N <= kMatMaxK;
        default: return true;
    }
}

lr_status step_run(const lr_desc& d, const lr_inputs& in, const float* s_in, float* s_out, void* y,
                   cudaStream_t st) {
    return d.io == LR_BF16 ? step_impl<__nv_bfloat16>(d, in, s_in, s_out, y, st)
                           : step_impl<float>(d, in, s_in, s_out, y, st);
}

}  // namespace lrs
