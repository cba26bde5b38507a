"""fp64 CPU oracle for the fused linear-recurrence scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package.  The product path (the C-ABI library and its Python binding) never does, and shares no
code with it.  The arithmetic lives in ``lr_oracle.c`` (plain sequential loops in double
precision); this module only marshals numpy arrays to it.

Every function takes numpy arrays (any float dtype; bf16 inputs must already be widened exactly,
e.g. ``tensor.double().numpy()``) in the token-major layouts documented in ``lr_oracle.c`` and
returns float64 arrays.  ``S`` (segment length) > 0 additionally returns the checkpointed states
after k*S steps, k = 0..ceil(L/S)-1.  Every forward takes an optional initial state ``h0`` (zero
when omitted) and, with ``final=True``, also returns the state after the last step, both in the
kind's state layout: rglru / rotlru [B, D], S6 [B, D, N], SSD [B, H, P, N], GLA [B, H, K, V].
Results are returned as ``y``, ``(y, ck)``, ``(y, hL)`` or ``(y, ck, hL)``.

S6 and SSD take ``delta_softplus=True`` with an optional ``delta_bias`` (per channel / head): the
step length is then ``dt = softplus(delta + delta_bias)`` (an elementwise front-end, written out
here in numpy), and the backward returns the gradient for the raw ``delta``,
``d dt * sigmoid(delta + bias)``, and ``delta_bias``, its sum over batch and time.

Sources: the mlx-recurrence post (Apple Developer Forums thread 840535, "Current kernels" and the
segment-checkpointing paragraph), "lrnnx: A library for Linear RNNs" (ai.info summary, Key
Contributions 2-3), and the K-Search / mlx-mamba blog post (techtrendfeed repost, the paragraph
after Table 1, for the recurrence and its associative operator).
"""
import ctypes
import os

import numpy as np

from . import build as _build

DISC = {"none": 0, "zoh": 1, "bilinear": 2, "dirac": 3, "zoh_euler": 4}

_lib = None


def load(path):
    """Open a compiled oracle library and declare its signatures."""
    L = ctypes.CDLL(path)
    i64, dp, ci = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.c_int
    L.orc_set_threads.argtypes = [ci]
    L.orc_get_threads.restype = ci
    L.orc_rglru_fwd.argtypes = [i64, i64, i64, dp, dp, dp, i64, dp, dp, dp]
    L.orc_rglru_bwd.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp]
    L.orc_rotlru_fwd.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp, i64, dp, dp, dp]
    L.orc_rotlru_bwd.argtypes = [i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, dp, dp]
    L.orc_s6_fwd.argtypes = [i64, i64, i64, i64, ci] + [dp] * 8 + [i64, dp, dp, dp]
    L.orc_s6_bwd.argtypes = [i64, i64, i64, i64, ci] + [dp] * 15
    L.orc_ssd_fwd.argtypes = [i64, i64, i64, i64, i64, i64, ci] + [dp] * 8 + [i64, dp, dp, dp]
    L.orc_ssd_bwd.argtypes = [i64, i64, i64, i64, i64, i64, ci] + [dp] * 15
    L.orc_gla_fwd.argtypes = [i64, i64, i64, i64, i64] + [dp] * 5 + [i64, dp, dp, dp]
    L.orc_gla_bwd.argtypes = [i64, i64, i64, i64, i64] + [dp] * 9
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor (CPU); widen exactly
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x):
    if x is None:
        return ctypes.POINTER(ctypes.c_double)()
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _softplus_front(delta, bias, axis_shape):
    """dt = softplus(delta + bias) and sigmoid(delta + bias) (bias broadcast along the last axis)."""
    v = delta + (0.0 if bias is None else _f64(bias).reshape(axis_shape))
    return np.logaddexp(0.0, v), 0.5 * (1.0 + np.tanh(0.5 * v))


def _nseg(L, S):
    return (L + S - 1) // S if S and S > 0 else 0


def _state(h0, shape):
    """Initial state as a contiguous float64 array of `shape` (None stays None)."""
    if h0 is None:
        return None
    h0 = _f64(h0)
    if h0.shape != tuple(shape):
        raise ValueError("initial state has shape %s, expected %s" % (h0.shape, tuple(shape)))
    return h0


def _ret(y, ck, hL, S, final):
    out = (y,) + ((ck,) if S else ()) + ((hL,) if final else ())
    return out[0] if len(out) == 1 else out


# ---------------------------------------------------------------------------------------- rglru
def rglru_fwd(a, b, S=0, h0=None, final=False):
    a, b = _f64(a), _f64(b)
    B, L, D = a.shape
    y = np.empty_like(a)
    ck = np.empty((_nseg(L, S), B, D)) if S else None
    h0 = _state(h0, (B, D))
    hL = np.empty((B, D)) if final else None
    lib().orc_rglru_fwd(B, L, D, _p(a), _p(b), _p(y), int(S or 0), _p(ck), _p(h0), _p(hL))
    return _ret(y, ck, hL, S, final)


def rglru_bwd(a, b, dy):
    a, b, dy = _f64(a), _f64(b), _f64(dy)
    B, L, D = a.shape
    da, db = np.empty_like(a), np.empty_like(a)
    lib().orc_rglru_bwd(B, L, D, _p(a), _p(b), _p(dy), _p(da), _p(db))
    return {"a": da, "b": db}


# --------------------------------------------------------------------- rglru with gate front-end
RG_LRU_C = 8.0  # the exponent constant of a = sigmoid(Lambda)^(c r)


def _rg_gates(r, i, x, lam):
    """a = sigmoid(Lambda)^(c r), s = sqrt(1 - a^2), b = s (i x): the RG-LRU gate front-end."""
    logsig = -np.logaddexp(0.0, -lam)          # log sigmoid(Lambda), per channel
    a = np.exp(RG_LRU_C * r * logsig)
    s = np.sqrt(1.0 - a * a)
    return a, s, s * i * x, logsig


def rglru_gated_fwd(r, i, x, lam, S=0, h0=None, final=False):
    """rglru on the gates: a = sigmoid(Lambda)^(c r), b = sqrt(1 - a^2) (i x) (r, i, x: [B, L, D],
    Lambda: [D]); the recurrence itself is the rglru oracle above."""
    r, i, x, lam = map(_f64, (r, i, x, lam))
    a, _, b, _ = _rg_gates(r, i, x, lam)
    return rglru_fwd(a, b, S=S, h0=h0, final=final)


def rglru_gated_bwd(r, i, x, lam, dy):
    """Gradients of the gated rglru by the chain rule through the rglru oracle's (da, db):
    di = db s x, dx = db s i, da_tot = da - db (i x) a / s, dr = da_tot a c log sigmoid(Lambda),
    dLambda = sum_{b,t} da_tot a c r (1 - sigmoid(Lambda))."""
    r, i, x, lam, dy = map(_f64, (r, i, x, lam, dy))
    a, s, b, logsig = _rg_gates(r, i, x, lam)
    g = rglru_bwd(a, b, dy)
    da_tot = g["a"] - g["b"] * i * x * a / s
    sig = 0.5 * (1.0 + np.tanh(0.5 * lam))
    return {"r": da_tot * a * RG_LRU_C * logsig, "i": g["b"] * s * x, "x": g["b"] * s * i,
            "lam": (da_tot * a * RG_LRU_C * r * (1.0 - sig)).sum(axis=(0, 1))}


# --------------------------------------------------------------------------------------- rotlru
def rotlru_fwd(b, g, mag, theta, S=0, h0=None, final=False):
    b, g, mag, theta = _f64(b), _f64(g), _f64(mag), _f64(theta)
    B, L, D = b.shape
    y = np.empty_like(b)
    ck = np.empty((_nseg(L, S), B, D)) if S else None
    h0 = _state(h0, (B, D))
    hL = np.empty((B, D)) if final else None
    lib().orc_rotlru_fwd(B, L, D, _p(b), _p(g), _p(mag), _p(theta), _p(y), int(S or 0), _p(ck),
                         _p(h0), _p(hL))
    return _ret(y, ck, hL, S, final)


def rotlru_bwd(b, g, mag, theta, dy):
    b, g, mag, theta, dy = _f64(b), _f64(g), _f64(mag), _f64(theta), _f64(dy)
    B, L, D = b.shape
    db, dg = np.empty_like(b), np.empty_like(g)
    dmag, dth = np.empty_like(mag), np.empty_like(theta)
    lib().orc_rotlru_bwd(B, L, D, _p(b), _p(g), _p(mag), _p(theta), _p(dy), _p(db), _p(dg),
                         _p(dmag), _p(dth))
    return {"b": db, "g": dg, "mag": dmag, "theta": dth}


# ------------------------------------------------------------------------------------------- S6
def s6_fwd(x, delta, A, Bm, Cm, Dskip=None, z=None, disc="zoh", S=0, h0=None, final=False,
           delta_softplus=False, delta_bias=None):
    x, delta, A, Bm, Cm = map(_f64, (x, delta, A, Bm, Cm))
    if delta_softplus:
        delta, _ = _softplus_front(delta, delta_bias, (1, 1, -1))
    Dskip, z = _f64(Dskip), _f64(z)
    B, L, D = x.shape
    N = A.shape[1]
    y = np.empty_like(x)
    ck = np.empty((_nseg(L, S), B, D, N)) if S else None
    h0 = _state(h0, (B, D, N))
    hL = np.empty((B, D, N)) if final else None
    lib().orc_s6_fwd(B, L, D, N, DISC[disc], _p(x), _p(delta), _p(A), _p(Bm), _p(Cm),
                     _p(Dskip), _p(z), _p(y), int(S or 0), _p(ck), _p(h0), _p(hL))
    return _ret(y, ck, hL, S, final)


def s6_bwd(x, delta, A, Bm, Cm, Dskip, z, dy, disc="zoh", delta_softplus=False, delta_bias=None):
    x, delta, A, Bm, Cm, dy = map(_f64, (x, delta, A, Bm, Cm, dy))
    sg = None
    if delta_softplus:
        delta, sg = _softplus_front(delta, delta_bias, (1, 1, -1))
    Dskip, z = _f64(Dskip), _f64(z)
    B, L, D = x.shape
    N = A.shape[1]
    dx, ddt = np.empty_like(x), np.empty_like(x)
    dA, dB, dC = np.empty_like(A), np.empty_like(Bm), np.empty_like(Cm)
    dD = np.empty(D) if Dskip is not None else None
    dz = np.empty_like(x) if z is not None else None
    lib().orc_s6_bwd(B, L, D, N, DISC[disc], _p(x), _p(delta), _p(A), _p(Bm), _p(Cm),
                     _p(Dskip), _p(z), _p(dy), _p(dx), _p(ddt), _p(dA), _p(dB), _p(dC),
                     _p(dD), _p(dz))
    out = {"x": dx, "delta": ddt, "A": dA, "B": dB, "C": dC, "D": dD, "z": dz}
    if sg is not None:
        out["delta"] = ddt * sg
        out["delta_bias"] = out["delta"].sum(axis=(0, 1))
    return out


# ------------------------------------------------------------------------------------------ SSD
def ssd_fwd(x, delta, A, Bm, Cm, Dskip=None, z=None, disc="zoh", S=0, h0=None, final=False,
            delta_softplus=False, delta_bias=None):
    x, delta, A, Bm, Cm = map(_f64, (x, delta, A, Bm, Cm))
    if delta_softplus:
        delta, _ = _softplus_front(delta, delta_bias, (1, 1, -1))
    Dskip, z = _f64(Dskip), _f64(z)
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.empty_like(x)
    ck = np.empty((_nseg(L, S), B, H, P, N)) if S else None
    h0 = _state(h0, (B, H, P, N))
    hL = np.empty((B, H, P, N)) if final else None
    lib().orc_ssd_fwd(B, L, H, P, N, G, DISC[disc], _p(x), _p(delta), _p(A), _p(Bm), _p(Cm),
                      _p(Dskip), _p(z), _p(y), int(S or 0), _p(ck), _p(h0), _p(hL))
    return _ret(y, ck, hL, S, final)


def ssd_bwd(x, delta, A, Bm, Cm, Dskip, z, dy, disc="zoh", delta_softplus=False, delta_bias=None):
    x, delta, A, Bm, Cm, dy = map(_f64, (x, delta, A, Bm, Cm, dy))
    sg = None
    if delta_softplus:
        delta, sg = _softplus_front(delta, delta_bias, (1, 1, -1))
    Dskip, z = _f64(Dskip), _f64(z)
    B, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    dx, ddt = np.empty_like(x), np.empty_like(delta)
    dA, dB, dC = np.empty_like(A), np.empty_like(Bm), np.empty_like(Cm)
    dD = np.empty(H) if Dskip is not None else None
    dz = np.empty_like(x) if z is not None else None
    lib().orc_ssd_bwd(B, L, H, P, N, G, DISC[disc], _p(x), _p(delta), _p(A), _p(Bm), _p(Cm),
                      _p(Dskip), _p(z), _p(dy), _p(dx), _p(ddt), _p(dA), _p(dB), _p(dC),
                      _p(dD), _p(dz))
    out = {"x": dx, "delta": ddt, "A": dA, "B": dB, "C": dC, "D": dD, "z": dz}
    if sg is not None:
        out["delta"] = ddt * sg
        out["delta_bias"] = out["delta"].sum(axis=(0, 1))
    return out


# ------------------------------------------------------------------------------------------ GLA
def gla_fwd(q, k, v, g, S=0, h0=None, final=False):
    q, k, v, g = map(_f64, (q, k, v, g))
    B, L, H, K = q.shape
    V = v.shape[3]
    o = np.empty_like(v)
    ck = np.empty((_nseg(L, S), B, H, K, V)) if S else None
    h0 = _state(h0, (B, H, K, V))
    hL = np.empty((B, H, K, V)) if final else None
    lib().orc_gla_fwd(B, L, H, K, V, _p(q), _p(k), _p(v), _p(g), _p(o), int(S or 0), _p(ck),
                      _p(h0), _p(hL))
    return _ret(o, ck, hL, S, final)


def gla_bwd(q, k, v, g, do):
    q, k, v, g, do = map(_f64, (q, k, v, g, do))
    B, L, H, K = q.shape
    V = v.shape[3]
    dq, dk, dv, dg = np.empty_like(q), np.empty_like(k), np.empty_like(v), np.empty_like(g)
    lib().orc_gla_bwd(B, L, H, K, V, _p(q), _p(k), _p(v), _p(g), _p(do), _p(dq), _p(dk), _p(dv),
                      _p(dg))
    return {"q": dq, "k": dk, "v": dv, "g": dg}
