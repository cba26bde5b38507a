/*
 * lrscan.h -- C ABI of the B200 (sm_100a) fused linear-recurrence scan library.
 *
 * The operation.  A linear recurrence h_t = a_t (.) h_{t-1} + b_t with readout y_t = f(h_t),
 * run over the whole sequence in one pass on the GPU instead of one dispatch per step, with a
 * backward pass that stores only the states at segment boundaries and recomputes the rest
 * ("mlx-recurrence", Apple Developer Forums thread 840535: opening paragraphs, and the list of
 * kernels under "Current kernels").  The associative operator (a2,b2) o (a1,b1) =
 * (a2 a1, a2 b1 + b2) that lets the sequence be split into chunks is the one stated in the
 * K-Search / mlx-mamba blog post (techtrendfeed repost, paragraph after Table 1).  The
 * time-varying selective scan with ZOH or bilinear discretisation follows "lrnnx: A library for
 * Linear RNNs" (ai.info summary, Key Contributions 2 and 3).
 *
 * Kinds (per-kind definitions, t = 0..L-1, h_{-1} = 0):
 *   LR_RGLRU   h_t = a_t h_{t-1} + b_t, y_t = h_t.                                  state [B, D]
 *   LR_ROTLRU  pair k = channels (2k, 2k+1) = (re, im); lambda_t = mag_k g_t[k] e^{i theta_k};
 *              h_t = lambda_t h_{t-1} + b_t (complex), y_t = h_t.                   state [B, D]
 *   LR_S6      per (d, n): abar, beta = disc(dt_t[d], A[d,n]);
 *              h_t[d,n] = abar h_{t-1}[d,n] + beta B_t[n] x_t[d];
 *              y_t[d] = (sum_n C_t[n] h_t[d,n] + D_d x_t[d]) * silu(z_t[d]).     state [B, D, N]
 *   LR_SSD     per head h, group g = h / (H / G): abar_t, beta_t = disc(dt_t[h], A_h);
 *              h_t[p,n] = abar_t h_{t-1}[p,n] + beta_t x_t[p] B_t[g,n];
 *              y_t[p] = sum_n C_t[g,n] h_t[p,n] + D_h x_t[p]  (times silu(z_t[p]) if z).
 *                                                                                state [B, H, P, N]
 *   LR_GLA     S_t = g_t S_{t-1} + k_t v_t^T (K x V), o_t = S_t^T q_t.          state [B, H, K, V]
 *   disc ZOH:       abar = exp(dt A), beta = (exp(dt A) - 1) / A.
 *   disc BILINEAR:  abar = (1 + dt A/2) / (1 - dt A/2), beta = dt / (1 - dt A/2).
 *   disc DIRAC:     abar = exp(dt A), beta = 1 (the input an impulse at the sample time).
 *   disc ZOH_EULER: abar = exp(dt A), beta = dt (zero-order hold for A, Euler for B).
 *   (The lrnnx summary names ZOH, bilinear and dirac discretisation without defining them; the
 *   readings above are this library's.)
 *
 * Layouts.  Row-major, last index contiguous, token-major:
 *   rglru   a, b, y, dy, da, db            [B, L, D]              io dtype
 *           (LR_RGLRU_GATES: r, i, x, dr, di, dx [B, L, D]; Lambda, dLambda [D] f32)
 *   rotlru  b, y, dy, db                   [B, L, D] (re, im interleaved)   io dtype
 *           g, dg                          [B, L, D/2]            io dtype
 *           mag, theta, dmag, dtheta       [D/2]                  f32
 *   s6      x, delta, z, y, dy, dx, ddelta, dz   [B, L, D]        io dtype
 *           A, dA [D, N] f32;  Bm, Cm [B, L, N] io;  dBm, dCm [B, L, N] f32;  Dskip, dDskip [D] f32
 *   ssd     x, z, y, dy, dx, dz [B, L, H, P] io;  delta, ddelta [B, L, H] io;
 *           A, dA, Dskip, dDskip [H] f32;  Bm, Cm [B, L, G, N] io;  dBm, dCm [B, L, G, N] f32
 *   gla     q, k, dq, dk [B, L, H, K] io;  v, o, dy, dv [B, L, H, V] io;  g, dg [B, L, H] io
 *   (for GLA the descriptor's N field carries K and P carries V).
 *
 * Ownership.  The caller allocates and frees every buffer: inputs, outputs, gradients, the
 * checkpoint buffer (lr_ckpt_bytes) and the workspace (lr_workspace_bytes).  The library
 * allocates nothing and frees nothing, and keeps no pointer after a call returns.  All pointers
 * passed to lr_scan_fwd / lr_scan_bwd are device pointers.
 *
 * Asynchrony and errors.  lr_scan_fwd / lr_scan_bwd validate on the host and enqueue work on the
 * given CUDA stream (a cudaStream_t passed as void*; NULL = legacy default stream); the returned
 * status covers validation and launch errors only.  Faults the kernels detect themselves (a
 * bounded wait that gave up, a failed bounds check in a checking build) are recorded in the
 * workspace and reported by lr_get_error.  Kernels never trap, assert or spin without a bound.
 *
 * Alignment.  Every pointer must be 16-byte aligned and the innermost dimension of every
 * per-token tensor must span a multiple of 16 bytes (LR_ERR_ALIGNMENT otherwise) -- except the
 * per-head dt of SSD and g of GLA ([B, L, H]), which may have any H.
 *
 * Gradients are written, not accumulated.
 */
#ifndef LRSCAN_H
#define LRSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LRSCAN_VERSION 1

typedef enum {
    LR_OK = 0,
    LR_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, non-positive or inconsistent shape   */
    LR_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement (see lr_validate) */
    LR_ERR_ALIGNMENT = 3,     /* pointer or innermost extent not 16-byte aligned                */
    LR_ERR_WORKSPACE = 4,     /* workspace smaller than lr_workspace_bytes                      */
    LR_ERR_CUDA = 5,          /* a CUDA runtime call failed (launch, memset, copy)              */
    LR_ERR_TIMEOUT = 6,       /* device: a bounded wait gave up (reported by lr_get_error)      */
    LR_ERR_DEVICE_CHECK = 7   /* device: a bounds/consistency check failed (lr_get_error)       */
} lr_status;

typedef enum { LR_RGLRU = 0, LR_ROTLRU = 1, LR_S6 = 2, LR_SSD = 3, LR_GLA = 4 } lr_kind;
typedef enum {
    LR_DISC_NONE = 0,
    LR_DISC_ZOH = 1,
    LR_DISC_BILINEAR = 2,
    LR_DISC_DIRAC = 3,
    LR_DISC_ZOH_EULER = 4
} lr_disc;
typedef enum { LR_F32 = 0, LR_BF16 = 1 } lr_dtype;

/* flags */
#define LR_HAS_Z 1u       /* S6 / SSD: multiply the readout by silu(z)   */
#define LR_HAS_DSKIP 2u   /* S6 / SSD: add the D-skip term D * x         */
/* Full-state mode (rglru, rotlru, S6): the forward pass checkpoints the state entering every step
 * (the checkpoint buffer holds L states, slot t = state entering step t, as with segment 1) and
 * the backward pass reads those states instead of recomputing them from segment checkpoints --
 * the "original full-state" design that the mlx-recurrence post (Apple Developer Forums thread
 * 840535, opening paragraphs) compares segment checkpoint-and-recompute against.  Outputs and
 * gradients are those of the default mode; the memory is L / S times the checkpoint memory.  The
 * segment length still sets the tiling.  SSD and GLA: LR_ERR_UNSUPPORTED. */
#define LR_FULL_STATE 4u
/* S6 / SSD: the step length is dt = softplus(delta + delta_bias) computed in the kernels (the
 * layer's raw delta and an f32 bias per channel (S6, [D]) or head (SSD, [H]), NULL = no bias);
 * the backward writes ddelta for the raw delta, dd * sigma(delta + bias), and, if ddelta_bias is
 * non-NULL, ddelta_bias = its sum over batch and time. */
#define LR_DELTA_SOFTPLUS 8u
/* rglru, f32 I/O: the RG-LRU gate front-end computed in the kernels.  The pages name the rglru
 * kernel for "Griffin and RecurrentGemma-style architectures" (mlx-recurrence post, Apple
 * Developer Forums thread 840535, "Current kernels") without stating its gates; this library
 * reads them as Griffin's: a_t = sigmoid(Lambda)^(8 r_t), b_t = sqrt(1 - a_t^2) (i_t x_t), then
 * h_t = a_t h_{t-1} + b_t, y_t = h_t.  With this flag the rglru members take other meanings:
 *   in->a   recurrence gate r [B, L, D] (values in (0, 1), typically a sigmoid output)
 *   in->b   input gate i      [B, L, D]
 *   in->x   the layer input x [B, L, D]
 *   in->A   Lambda [D] f32
 *   gr->da, gr->db, gr->dx   dr, di, dx [B, L, D];  gr->dA  dLambda [D] f32 (NULL = not wanted)
 * a is formed as e^{8 r log sigmoid(Lambda)} and 1 - a^2 as -expm1(2 log a), so b keeps its
 * relative precision as a approaches 1.  dr is undefined where r = 0 exactly (b's derivative
 * contains 1 / sqrt(1 - a^2)).  Not combined with LR_FULL_STATE (LR_ERR_UNSUPPORTED); other
 * kinds: LR_ERR_INVALID_ARG.  lr_step accepts it (forward only). */
#define LR_RGLRU_GATES 16u
/* Test hook for the failure path: the tiles of the first segment never publish their carry
 * (rglru, rotlru), or the state scan never counts checkpoint slot 0 (SSD, GLA), so the tiles or
 * chunk kernels that depend on it wait out their bound (about 1 s), record LR_ERR_TIMEOUT and
 * finish with incomplete inputs.  Results of such a call are meaningless; lr_get_error reports
 * the timeout. */
#define LR_TEST_WITHHOLD_CARRY 0x80000000u
/* Test hook for the work distribution: SSD kernels that loop over the heads of a group inside one
 * CTA take the largest head blocks they support (16 heads) instead of sizing the blocks to fill
 * the GPU.  Results are bitwise identical with and without it; small test problems use it to
 * cover the multi-head pipelines. */
#define LR_TEST_MAX_HEAD_BLOCK 0x40000000u
/* Test hook for the carry exchange of rglru / rotlru: rows of at most 8 segment tiles normally run
 * as one thread-block cluster whose tiles exchange their aggregates through distributed shared
 * memory; with this flag they take the look-back over global-memory records that longer rows use.
 * Results are bitwise identical either way. */
#define LR_TEST_LOOKBACK 0x20000000u

/* Problem descriptor.  Unused dimensions are 0.  S6: D, N.  SSD: H, P, N, G, chunk.
 * GLA: H, P (= V), N (= K), chunk.  rglru / rotlru: D.  segment = checkpoint segment length S
 * (the backward pass stores the state every S steps and recomputes inside a segment). */
typedef struct {
    int32_t kind;      /* lr_kind  */
    int32_t disc;      /* lr_disc  (S6 / SSD: ZOH, BILINEAR, DIRAC or ZOH_EULER; others: NONE) */
    int32_t io;        /* lr_dtype of per-token tensors                         */
    uint32_t flags;    /* LR_HAS_Z | LR_HAS_DSKIP                               */
    int64_t B, L, D, H, P, N, G;
    int32_t chunk;     /* SSD / GLA chunk length Q (0 = default 64)             */
    int32_t segment;   /* checkpoint segment length S                           */
} lr_desc;

/* Inputs, per kind (unused members NULL).  Device pointers. */
typedef struct {
    const void *a, *b;            /* rglru a, b; rotlru b                    */
    const void *g;                /* rotlru magnitude gate; gla forget gate  */
    const float *mag, *theta;     /* rotlru                                  */
    const void *x, *delta;        /* s6 / ssd                                */
    const float *A;               /* s6 [D,N] / ssd [H]                      */
    const void *Bm, *Cm;          /* s6 / ssd                                */
    const float *Dskip;           /* s6 [D] / ssd [H] (LR_HAS_DSKIP)         */
    const void *z;                /* s6 / ssd (LR_HAS_Z)                     */
    const void *q, *k, *v;        /* gla                                     */
    const float *delta_bias;      /* s6 [D] / ssd [H] (LR_DELTA_SOFTPLUS)     */
} lr_inputs;

/* Gradients, per kind (unused members NULL).  Device pointers. */
typedef struct {
    void *da, *db, *dg;           /* rglru da, db; rotlru db, dg; gla dg     */
    float *dmag, *dtheta;         /* rotlru                                  */
    void *dx, *ddelta;            /* s6 / ssd                                */
    float *dA, *dBm, *dCm, *dDskip;
    void *dz;
    void *dq, *dk, *dv;           /* gla                                     */
    float *ddelta_bias;           /* s6 [D] / ssd [H] (LR_DELTA_SOFTPLUS)     */
} lr_grads;

/* Host-side check of a descriptor: LR_OK, or the status lr_scan_fwd would return for it
 * (INVALID_ARG for inconsistent shapes, UNSUPPORTED for a valid request outside the library's
 * limits, ALIGNMENT for innermost extents that are not multiples of 16 bytes). */
lr_status lr_validate(const lr_desc *desc);

/* Bytes of the checkpoint buffer: ceil(L/S) states, f32 (slot k = state after k*S steps); L
 * states with LR_FULL_STATE.
 * The forward pass writes it and the backward pass reads it.  0 on an invalid descriptor.
 * Layout per slot: rglru / rotlru [B, D]; s6 [B, D, N]; ssd [B, H, N, P]; gla [B, H, K, V].
 * SSD and GLA with segment == chunk (128): the f32 slots are followed by a bf16 copy of every
 * slot's per-head state blocks in the library's internal tensor-core tile order (read back by the
 * kernels only).  With longer segments (a whole number of chunks) the buffer holds the f32 segment
 * states only; the backward pass rebuilds the state entering every chunk from them. */
size_t lr_ckpt_bytes(const lr_desc *desc);

/* Bytes of scratch the forward (backward = 0) or backward (backward = 1) pass needs: per-tile
 * carry records and flags, parameter-gradient partial sums and the error word.  The content need
 * not be initialised; each call resets what it uses.  0 on an invalid descriptor. */
size_t lr_workspace_bytes(const lr_desc *desc, int backward);

/* Forward pass over the whole sequence: writes y and the segment checkpoints.
 *   desc, in   problem and input pointers (see the layout table above)
 *   y          output, same layout and dtype as the kind's per-token output
 *   ckpt       checkpoint buffer of lr_ckpt_bytes(desc) bytes (written)
 *   ws         workspace of ws_bytes >= lr_workspace_bytes(desc, 0) bytes
 *   stream     cudaStream_t as void*
 * Returns LR_OK once the work is enqueued. */
lr_status lr_scan_fwd(const lr_desc *desc, const lr_inputs *in, void *y, void *ckpt, void *ws,
                      size_t ws_bytes, void *stream);

/* Backward pass: recomputes the states inside each segment from ckpt and runs the adjoint
 * recurrence in reverse; writes every non-NULL gradient required by the kind
 * (rglru: da, db, and with LR_RGLRU_GATES dx and (optional) dA; rotlru: db, dg, dmag, dtheta; s6: dx, ddelta, dA, dBm, dCm, dDskip if
 * LR_HAS_DSKIP, dz if LR_HAS_Z; ssd: the same with per-head dA, dDskip; gla: dq, dk, dv, dg).
 *   dy         upstream gradient of y (io dtype, y's layout)
 *   ckpt       the buffer the matching lr_scan_fwd call wrote
 *   ws         workspace of ws_bytes >= lr_workspace_bytes(desc, 1) bytes */
lr_status lr_scan_bwd(const lr_desc *desc, const lr_inputs *in, const void *dy, const void *ckpt,
                      lr_grads *grads, void *ws, size_t ws_bytes, void *stream);

/* Decode and continuation (forward only): advances the recurrence by desc->L steps from the
 * state `state_in` and writes the outputs of those steps and the state after the last one.  One
 * token per call (L = 1) is the decode step; a longer call continues a sequence.  Running L1
 * steps and then L2 steps from the returned state is the same recurrence as L1 + L2 steps (the
 * recurrence h_t = a_t h_{t-1} + b_t of the mlx-recurrence post, Apple Developer Forums thread
 * 840535, "Current kernels"; one-token decode as in the mlx-mamba post, techtrendfeed repost,
 * paragraph after Table 1).
 *   desc        as for lr_scan_fwd; `segment` and `chunk` are ignored.  Limits of this path:
 *               S6 N <= 32; SSD N <= 128; GLA K (desc->N) <= 128 (LR_ERR_UNSUPPORTED beyond).
 *               SSD takes ZOH or BILINEAR and may have a z gate here.
 *   in          per-token inputs of the L steps, [B, L, ...] as for lr_scan_fwd (contiguous)
 *   state_in    f32 state entering the call, NULL for the zero state; layouts:
 *                 rglru, rotlru [B, D] (rotlru re, im interleaved per pair);  S6 [B, D, N];
 *                 SSD [B, H, N, P] (row n, column p: the layout of the checkpoint slots);
 *                 GLA [B, H, K, V]
 *   state_out   f32 state after the last step (written); may be the same buffer as state_in
 *   y           outputs of the L steps (io dtype, the kind's output layout)
 * Pointers need the alignment of their element type only (rotlru b, y: two elements).  No
 * workspace, no checkpoint; nothing is allocated and nothing synchronises, so the call can be
 * captured in a CUDA graph.  Returns LR_OK once the work is enqueued. */
lr_status lr_step(const lr_desc *desc, const lr_inputs *in, const void *state_in, void *state_out,
                  void *y, void *stream);

/* Synchronises `stream`, then reads and clears the device-side error record in `ws`.  Every
 * lr_scan_fwd / lr_scan_bwd call resets that record when it starts, so this reports the most
 * recent call that used `ws`.  LR_OK, LR_ERR_TIMEOUT or LR_ERR_DEVICE_CHECK; LR_ERR_CUDA
 * if the synchronisation itself failed.  `info`, if non-NULL, receives a kernel-specific code. */
lr_status lr_get_error(void *ws, void *stream, int32_t *info);

/* Static, human-readable name of a status. */
const char *lr_status_string(lr_status s);

/* Timing hook (benchmarks).  While set, on this host thread, every kernel launch of an
 * lr_scan_fwd / lr_scan_bwd call first records events[k] on the call's stream, k = 0, 1, ...
 * counting the launches of that call (launches past n record nothing).  Kernel k then runs between
 * events[k] and events[k + 1] (the last one until whatever the caller records after the call).
 * events: n cudaEvent_t handles passed as void*, owned by the caller; NULL or n = 0 turns the
 * hook off.  Records only; never synchronises. */
void lr_set_launch_events(void *const *events, int n);

/* Names of the kernels the last lr_scan_fwd / lr_scan_bwd / lr_step call on this host thread launched,
 * separated by '+' (a fingerprint that lets tests check which code path ran). */
const char *lr_last_dispatch(void);

/* Number of kernel launches the last lr_scan_fwd / lr_scan_bwd / lr_step call on this thread enqueued. */
int lr_last_launch_count(void);

int lr_version(void);

/* Calibration probe (benchmarks).  The pages give no rates for the arithmetic pipes a scan may be
 * bound by; the S6 scan is bound by exponentials and fp32 FMAs rather than by memory, so its
 * roofline needs the rate of each pipe on the part it runs on.  Enqueues one kernel on `stream`
 * that keeps one pipe busy: which = 0 the special-function unit (ex2.approx.ftz.f32), which = 1
 * the fp32 FMA pipe (fma.rn.f32); `blocks` x `threads` threads each run `iters` iterations of 8
 * independent dependency chains and write one float to out[blocks * threads] (device, caller
 * owned).  Returns the number of results the launch produces (time it with CUDA events recorded
 * around the call; results / seconds is the pipe's rate), or -1 for invalid arguments (threads
 * a multiple of 32 in [32, 1024], blocks and iters >= 1) or a failed launch. */
int64_t lr_probe_pipe(int which, float *out, int blocks, int threads, int iters, void *stream);

/* lr_rglru_fwd_noalloc -- the rglru forward pass for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists for deployment, not for the method.
 *
 * Who needs it: code that runs inside a framework owning every device byte through its own pool
 * (and offering no scratch buffer to plug-ins), hosts that only let a plug-in run a fixed
 * callback on the tensors they hand over, and latency-critical loops where cudaMalloc / cudaFree
 * would synchronise the device.  Such callers cannot provide the workspace lr_scan_fwd needs.
 *
 * It computes exactly what lr_scan_fwd computes for LR_RGLRU (same kernel): y [B, L, D] and the
 * segment checkpoints `ckpt` (lr_ckpt_bytes(desc) bytes), from device inputs a, b.  Its scratch
 * is a 1 MiB array inside the library (held by every GPU that loads the library until the
 * process exits); the call allocates nothing.  Limit: problems whose forward workspace
 * (lr_workspace_bytes(desc, 0), about 770 bytes per tile of 32 channels x S steps per batch row)
 * exceeds 1 MiB are rejected with LR_ERR_WORKSPACE.
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  All calls on a device
 * share the array and each call clears the part that must start at zero, so calls that overlap
 * on the GPU (unordered streams) race and must be avoided.  With `check` non-zero the call
 * synchronises `stream` and returns the kernel's device-side status (LR_ERR_TIMEOUT if a bounded
 * wait gave up); otherwise it returns once the work is enqueued.  Other statuses as
 * lr_scan_fwd (LR_ERR_INVALID_ARG also for a kind other than LR_RGLRU; LR_ERR_UNSUPPORTED with
 * LR_RGLRU_GATES, whose inputs this signature does not carry). */
lr_status lr_rglru_fwd_noalloc(const lr_desc *desc, const void *a, const void *b, void *y,
                               void *ckpt, void *stream, int check);

/* The device-side status of the last lr_rglru_fwd_noalloc call on the current device, for callers
 * that enqueue it with check = 0 (it has no workspace to hand to lr_get_error).  Synchronises
 * `stream`, then reads and clears the error record at the start of the library's array: LR_OK,
 * LR_ERR_TIMEOUT or LR_ERR_DEVICE_CHECK (`info`, if non-NULL, receives the kernel's detail code);
 * LR_ERR_CUDA if the synchronisation or the read failed.  Every lr_rglru_fwd_noalloc call clears
 * the record when it starts, so a status must be read before the next call on that device is
 * enqueued. */
lr_status lr_rglru_noalloc_error(void *stream, int32_t *info);

#ifdef __cplusplus
}
#endif
#endif /* LRSCAN_H */
