"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics (CPU only).

The oracle is a sequential loop.  Each test below checks it against something that is NOT that
loop: a closed form evaluated by brute force, a library routine (scipy's discretisation of a
continuous-time system), a geometric series, a tree-ordered evaluation of the associative
operator, an invariant, another kind it must reduce to, or finite differences of its own
forward pass.  A dropped term, a wrong sign, an index shifted by one or a transposed operand in
``oracle/lr_oracle.c`` fails at least one of them (``test_planted_mistakes`` checks this claim
for a few such mistakes).

Sources: the recurrence and its four kinds -- mlx-recurrence post (Apple Developer Forums thread
840535, opening paragraphs and "Current kernels"); the associative operator and its prefix-scan
evaluation -- K-Search / mlx-mamba blog post (techtrendfeed repost, paragraph after Table 1);
ZOH / bilinear discretisation and the parallel / recurrent / step-wise equivalence test matrix --
"lrnnx: A library for Linear RNNs" (ai.info summary, Key Contributions 2-3, Main Findings).
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.signal import cont2discrete

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
REL = 1e-12


def rel_err(x, ref):
    x, ref = np.asarray(x), np.asarray(ref)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


# ------------------------------------------------------------------------ independent helpers
def scipy_disc(dt, A, method):
    """(abar, beta) of dh/dt = A h + u sampled at step dt, from scipy (matrix exponential for
    ZOH, generalised bilinear transform with alpha = 1/2 for Tustin).  The two mixed schemes take
    abar from scipy's ZOH and beta from their definition: dirac (an impulse input enters the state
    undamped, beta = 1) and ZOH-Euler (beta from scipy's forward Euler, dt)."""
    def c2d(m):
        Ad, Bd, _, _, _ = cont2discrete((np.array([[A]]), np.array([[1.0]]), np.array([[1.0]]),
                                         np.array([[0.0]])), float(dt), method=m)
        return Ad[0, 0], Bd[0, 0]
    if method == "dirac":
        return c2d("zoh")[0], 1.0
    if method == "zoh_euler":
        return c2d("zoh")[0], c2d("euler")[1]
    return c2d(method)


def closed_form(a, b):
    """h_t = sum_{s<=t} (prod_{r=s+1..t} a_r) b_s, by brute force (real or complex, 1-D)."""
    L = len(a)
    out = np.zeros(L, dtype=np.result_type(a, b))
    for t in range(L):
        out[t] = sum(np.prod(a[s + 1:t + 1]) * b[s] for s in range(t + 1))
    return out


def tree_scan(a, b, rng):
    """Inclusive prefix of (a_t, b_t) under (a2,b2) o (a1,b1) = (a2 a1, a2 b1 + b2), evaluated
    with random chunking: each chunk by Hillis-Steele doubling, then chunk carries combined
    by the same operator.  Returns the b-component, i.e. h_t."""
    L = len(a)
    cuts = sorted(set([0, L] + list(rng.integers(1, L, size=max(1, L // 5)))))
    A, Bv = np.array(a, dtype=np.result_type(a, b)), np.array(b, dtype=np.result_type(a, b))
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        ca, cb = A[lo:hi].copy(), Bv[lo:hi].copy()
        k = 1
        while k < hi - lo:
            na, nb = ca.copy(), cb.copy()
            na[k:] = ca[k:] * ca[:-k]
            nb[k:] = ca[k:] * cb[:-k] + cb[k:]
            ca, cb = na, nb
            k *= 2
        A[lo:hi], Bv[lo:hi] = ca, cb
    carry_a, carry_b = None, None
    out = np.empty_like(Bv)
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        if carry_a is None:
            out[lo:hi] = Bv[lo:hi]
        else:
            out[lo:hi] = A[lo:hi] * carry_b + Bv[lo:hi]
        carry_b = out[hi - 1]
        carry_a = 1.0
    return out


def silu(z):
    return z / (1.0 + np.exp(-z))


# ------------------------------------------------------------------------------- P1: closed form
def test_rglru_closed_form(orc):
    rng = np.random.default_rng(1)
    B, L, D = 2, 13, 3
    a = rng.uniform(-1.1, 1.1, (B, L, D))
    b = rng.normal(size=(B, L, D))
    y, ck = orc.rglru_fwd(a, b, S=4)
    for bi in range(B):
        for d in range(D):
            ref = closed_form(a[bi, :, d], b[bi, :, d])
            assert rel_err(y[bi, :, d], ref) < REL
            for kk in range(ck.shape[0]):
                want = 0.0 if kk == 0 else ref[kk * 4 - 1]
                assert abs(ck[kk, bi, d] - want) <= REL * max(1.0, abs(want))


def test_rotlru_closed_form(orc):
    rng = np.random.default_rng(2)
    B, L, D = 2, 11, 6
    K = D // 2
    b = rng.normal(size=(B, L, D))
    g = rng.uniform(0.2, 1.0, (B, L, K))
    mag = rng.uniform(0.5, 1.0, K)
    th = rng.uniform(-math.pi, math.pi, K)
    y, ck = orc.rotlru_fwd(b, g, mag, th, S=3)
    for bi in range(B):
        for k in range(K):
            lam = mag[k] * g[bi, :, k] * np.exp(1j * th[k])
            bc = b[bi, :, 2 * k] + 1j * b[bi, :, 2 * k + 1]
            ref = closed_form(lam, bc)
            assert rel_err(y[bi, :, 2 * k] + 1j * y[bi, :, 2 * k + 1], ref) < REL
            for kk in range(1, ck.shape[0]):
                got = ck[kk, bi, 2 * k] + 1j * ck[kk, bi, 2 * k + 1]
                assert abs(got - ref[kk * 3 - 1]) < REL * max(1.0, abs(ref).max())


@pytest.mark.parametrize("disc", ["zoh", "bilinear", "dirac", "zoh_euler"])
def test_s6_closed_form_with_scipy_discretisation(orc, disc):
    """S6 output as the quadratic form y_t = (sum_{s<=t} sum_n C_t[n] (prod abar) beta_s B_s[n]
    x_s + D x_t) silu(z_t), with abar and beta from scipy's discretisation."""
    rng = np.random.default_rng(3)
    B, L, D, N = 2, 7, 3, 2
    x = rng.normal(size=(B, L, D))
    dt = rng.uniform(0.01, 0.9, (B, L, D))
    A = -rng.uniform(0.3, 3.0, (D, N))
    Bm, Cm = rng.normal(size=(B, L, N)), rng.normal(size=(B, L, N))
    Dk, z = rng.normal(size=D), rng.normal(size=(B, L, D))
    y, ck = orc.s6_fwd(x, dt, A, Bm, Cm, Dk, z, disc=disc, S=3)
    for bi in range(B):
        for d in range(D):
            for n in range(N):
                ab = np.empty(L)
                be = np.empty(L)
                for t in range(L):
                    ab[t], be[t] = scipy_disc(dt[bi, t, d], A[d, n], disc)
                hn = closed_form(ab, be * Bm[bi, :, n] * x[bi, :, d])
                for kk in range(1, ck.shape[0]):
                    assert abs(ck[kk, bi, d, n] - hn[kk * 3 - 1]) < 1e-12
            ref = np.zeros(L)
            for t in range(L):
                s = D * 0.0
                for n in range(N):
                    for s_ in range(t + 1):
                        prod = 1.0
                        for r in range(s_ + 1, t + 1):
                            prod *= scipy_disc(dt[bi, r, d], A[d, n], disc)[0]
                        beta_s = scipy_disc(dt[bi, s_, d], A[d, n], disc)[1]
                        s += Cm[bi, t, n] * prod * beta_s * Bm[bi, s_, n] * x[bi, s_, d]
                ref[t] = (s + Dk[d] * x[bi, t, d]) * silu(z[bi, t, d])
            assert rel_err(y[bi, :, d], ref) < 1e-11


def test_ssd_quadratic_form(orc):
    """SSD per (b, h): Y = (M o C B^T) X + D X with M[t,s] = prod_{r=s+1..t} abar_r * beta_s."""
    rng = np.random.default_rng(4)
    B, L, H, P, N, G = 2, 9, 4, 3, 5, 2
    x = rng.normal(size=(B, L, H, P))
    dt = rng.uniform(0.02, 0.8, (B, L, H))
    A = -rng.uniform(0.5, 8.0, H)
    Bm, Cm = rng.normal(size=(B, L, G, N)), rng.normal(size=(B, L, G, N))
    Dk = rng.normal(size=H)
    y, ck = orc.ssd_fwd(x, dt, A, Bm, Cm, Dk, None, disc="zoh", S=4)
    for bi in range(B):
        for h in range(H):
            gi = h // (H // G)
            ab = np.array([scipy_disc(dt[bi, t, h], A[h], "zoh")[0] for t in range(L)])
            be = np.array([scipy_disc(dt[bi, t, h], A[h], "zoh")[1] for t in range(L)])
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    M[t, s] = np.prod(ab[s + 1:t + 1]) * be[s]
            CB = Cm[bi, :, gi, :] @ Bm[bi, :, gi, :].T
            ref = (M * CB) @ x[bi, :, h, :] + Dk[h] * x[bi, :, h, :]
            assert rel_err(y[bi, :, h, :], ref) < REL
            # checkpoint k = state after 4k steps: sum_s M[4k-1, s] x_s B_s^T  (P x N)
            for kk in range(1, ck.shape[0]):
                t = kk * 4 - 1
                st = sum(M[t, s] * np.outer(x[bi, s, h, :], Bm[bi, s, gi, :]) for s in range(t + 1))
                assert rel_err(ck[kk, bi, h], st) < REL


def test_gla_closed_form(orc):
    """GLA: o_t = sum_{s<=t} (prod_{r=s+1..t} g_r) (q_t . k_s) v_s."""
    rng = np.random.default_rng(5)
    B, L, H, K, V = 2, 8, 2, 3, 4
    q, k = rng.normal(size=(B, L, H, K)), rng.normal(size=(B, L, H, K))
    v, g = rng.normal(size=(B, L, H, V)), rng.uniform(0.3, 1.0, (B, L, H))
    o, ck = orc.gla_fwd(q, k, v, g, S=3)
    for bi in range(B):
        for h in range(H):
            ref = np.zeros((L, V))
            for t in range(L):
                for s in range(t + 1):
                    ref[t] += np.prod(g[bi, s + 1:t + 1, h]) * (q[bi, t, h] @ k[bi, s, h]) * v[bi, s, h]
            assert rel_err(o[bi, :, h], ref) < REL
            for kk in range(1, ck.shape[0]):
                t = kk * 3 - 1
                st = sum(np.prod(g[bi, s + 1:t + 1, h]) * np.outer(k[bi, s, h], v[bi, s, h])
                         for s in range(t + 1))
                assert rel_err(ck[kk, bi, h], st) < REL


# -------------------------------------------------------------------------- P2: geometric series
def test_geometric_series(orc):
    L = 200
    for a0, b0 in [(0.5, 1.0), (0.99, -2.0), (-0.7, 0.3), (1.0, 0.25)]:
        a = np.full((1, L, 1), a0)
        b = np.full((1, L, 1), b0)
        y = orc.rglru_fwd(a, b)[0, :, 0]
        t = np.arange(1, L + 1)
        ref = b0 * t if a0 == 1.0 else b0 * (1 - a0 ** t) / (1 - a0)
        assert rel_err(y, ref) < REL


# ------------------------------------------------------------------ P3: associative tree scan
def test_associative_tree_scan(orc):
    rng = np.random.default_rng(6)
    for trial in range(5):
        L = int(rng.integers(2, 300))
        a = rng.uniform(-1.05, 1.05, (1, L, 1))
        b = rng.normal(size=(1, L, 1))
        y = orc.rglru_fwd(a, b)[0, :, 0]
        assert rel_err(y, tree_scan(a[0, :, 0], b[0, :, 0], rng)) < 1e-11
        # complex (rotlru) through the same operator
        K = 1
        g = rng.uniform(0.3, 1.0, (1, L, K))
        mag, th = np.array([0.99]), np.array([rng.uniform(0, 3)])
        bb = rng.normal(size=(1, L, 2))
        yc = orc.rotlru_fwd(bb, g, mag, th)[0]
        lam = mag[0] * g[0, :, 0] * np.exp(1j * th[0])
        ref = tree_scan(lam, bb[0, :, 0] + 1j * bb[0, :, 1], rng)
        assert rel_err(yc[:, 0] + 1j * yc[:, 1], ref) < 1e-11


# ------------------------------------------------------------------- P4: rotation invariant
def test_rotation_norm_invariant(orc):
    L = 400
    th = np.array([0.3, math.pi / 2, 2.9])
    K = len(th)
    b = np.zeros((1, L, 2 * K))
    b0 = np.array([[0.6, -0.8], [1.0, 0.0], [-2.0, 1.5]])
    b[0, 0, :] = b0.reshape(-1)
    y = orc.rotlru_fwd(b, np.ones((1, L, K)), np.ones(K), th)[0]
    for k in range(K):
        h = y[:, 2 * k] + 1j * y[:, 2 * k + 1]
        r0 = abs(b0[k, 0] + 1j * b0[k, 1])
        assert np.max(np.abs(np.abs(h) - r0)) < 1e-12
        ang0 = math.atan2(b0[k, 1], b0[k, 0])
        want = np.exp(1j * (ang0 + th[k] * np.arange(L)))
        assert np.max(np.abs(h / r0 - want)) < 1e-11


# -------------------------------------------------------------- P5: cross-kind reductions
def test_rotlru_zero_angle_is_rglru(orc):
    rng = np.random.default_rng(7)
    B, L, K = 2, 30, 3
    b = rng.normal(size=(B, L, 2 * K))
    g = rng.uniform(0.2, 1, (B, L, K))
    mag = rng.uniform(0.5, 1, K)
    y = orc.rotlru_fwd(b, g, mag, np.zeros(K))
    a = mag[None, None, :] * g
    yr = orc.rglru_fwd(a, b[:, :, 0::2])
    yi = orc.rglru_fwd(a, b[:, :, 1::2])
    assert rel_err(y[:, :, 0::2], yr) < REL and rel_err(y[:, :, 1::2], yi) < REL
    dy = rng.normal(size=b.shape)
    gr = orc.rotlru_bwd(b, g, mag, np.zeros(K), dy)
    r_re = orc.rglru_bwd(a, b[:, :, 0::2], dy[:, :, 0::2])
    r_im = orc.rglru_bwd(a, b[:, :, 1::2], dy[:, :, 1::2])
    assert rel_err(gr["b"][:, :, 0::2], r_re["b"]) < REL
    # dl/dm_t = da_re + da_im (theta = 0), dg = mag * dl/dm
    assert rel_err(gr["g"], mag * (r_re["a"] + r_im["a"])) < 1e-11


@pytest.mark.parametrize("disc", ["zoh", "bilinear", "dirac", "zoh_euler"])
def test_s6_with_headwise_parameters_is_ssd(orc, disc):
    rng = np.random.default_rng(8)
    B, L, H, P, N = 2, 10, 3, 2, 4
    D = H * P
    x = rng.normal(size=(B, L, H, P))
    dt = rng.uniform(0.05, 0.6, (B, L, H))
    Ah = -rng.uniform(0.5, 4, H)
    Bm, Cm = rng.normal(size=(B, L, 1, N)), rng.normal(size=(B, L, 1, N))
    Dh = rng.normal(size=H)
    z = rng.normal(size=(B, L, H, P))
    y_ssd = orc.ssd_fwd(x, dt, Ah, Bm, Cm, Dh, z, disc=disc)
    x6 = x.reshape(B, L, D)
    dt6 = np.repeat(dt, P, axis=2)
    A6 = np.repeat(Ah, P)[:, None] * np.ones((1, N))
    D6 = np.repeat(Dh, P)
    z6 = z.reshape(B, L, D)
    y6 = orc.s6_fwd(x6, dt6, A6, Bm[:, :, 0], Cm[:, :, 0], D6, z6, disc=disc)
    assert rel_err(y6, y_ssd.reshape(B, L, D)) < REL
    dy = rng.normal(size=(B, L, H, P))
    gs = orc.ssd_bwd(x, dt, Ah, Bm, Cm, Dh, z, dy, disc=disc)
    g6 = orc.s6_bwd(x6, dt6, A6, Bm[:, :, 0], Cm[:, :, 0], D6, z6, dy.reshape(B, L, D), disc=disc)
    assert rel_err(g6["x"], gs["x"].reshape(B, L, D)) < 1e-11
    assert rel_err(g6["z"], gs["z"].reshape(B, L, D)) < 1e-11
    assert rel_err(g6["delta"].reshape(B, L, H, P).sum(-1), gs["delta"]) < 1e-11
    assert rel_err(g6["A"].reshape(H, P, N).sum((1, 2)), gs["A"]) < 1e-11
    assert rel_err(g6["D"].reshape(H, P).sum(1), gs["D"]) < 1e-11
    assert rel_err(g6["B"], gs["B"][:, :, 0]) < 1e-11
    assert rel_err(g6["C"], gs["C"][:, :, 0]) < 1e-11


def test_gla_reduces_to_ssd(orc):
    """GLA with q = C, k = beta B, v = x, g = abar is SSD without the D skip (one head per group)."""
    rng = np.random.default_rng(9)
    B, L, H, P, N = 1, 12, 2, 3, 4
    x = rng.normal(size=(B, L, H, P))
    dt = rng.uniform(0.05, 0.6, (B, L, H))
    Ah = -rng.uniform(0.5, 4, H)
    Bm, Cm = rng.normal(size=(B, L, H, N)), rng.normal(size=(B, L, H, N))
    y = orc.ssd_fwd(x, dt, Ah, Bm, Cm, None, None, disc="zoh")
    ab = np.exp(dt * Ah)
    be = np.expm1(dt * Ah) / Ah
    o = orc.gla_fwd(Cm, be[..., None] * Bm, x, ab)
    assert rel_err(o, y) < REL


def test_small_step_zoh_minus_bilinear_is_third_order(orc):
    """exp(u) and (1+u/2)/(1-u/2) agree to O(u^3): the two-step S6 output difference scales
    as dt^3 (log-log slope ~3)."""
    errs, dts = [], [1e-2, 5e-3, 2.5e-3, 1.25e-3]
    for dtv in dts:
        x = np.ones((1, 2, 1))
        dt = np.full((1, 2, 1), dtv)
        A = np.array([[-2.0]])
        Bm = np.ones((1, 2, 1))
        Cm = np.ones((1, 2, 1))
        yz = orc.s6_fwd(x, dt, A, Bm, Cm, None, None, disc="zoh")
        yb = orc.s6_fwd(x, dt, A, Bm, Cm, None, None, disc="bilinear")
        errs.append(abs(yz[0, 1, 0] - yb[0, 1, 0]))
    slope = np.polyfit(np.log(dts), np.log(errs), 1)[0]
    assert 2.8 < slope < 3.2


def test_zoh_beta_tends_to_dt_as_A_vanishes(orc):
    x = np.full((1, 1, 1), 1.7)
    dt = np.full((1, 1, 1), 0.3)
    Bm = np.ones((1, 1, 1)) * 2.0
    Cm = np.ones((1, 1, 1))
    for Av in [-1e-3, -1e-6, -1e-9, 0.0]:
        y = orc.s6_fwd(x, dt, np.array([[Av]]), Bm, Cm, None, None, disc="zoh")
        # beta = dt (1 + dt A / 2 + O(A^2)): the gap closes linearly in A
        bound = 0.5 * 0.3 ** 2 * abs(Av) * 2.0 * 1.7 * 1.01 + 1e-14
        assert abs(y[0, 0, 0] - 0.3 * 2.0 * 1.7) <= bound


# --------------------------------------------------------------- P6: finite differences
def _fd_check(fwd, bwd, inputs, names, dy, eps=1e-6, tol=1e-7):
    """Central differences of l = <fwd(inputs), dy> against bwd(...)[name] for each name."""
    grads = bwd(inputs, dy)
    for name in names:
        arr = inputs[name]
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = arr[idx]
            arr[idx] = old + eps
            lp = np.sum(fwd(inputs) * dy)
            arr[idx] = old - eps
            lm = np.sum(fwd(inputs) * dy)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        err = rel_err(grads[name], num)
        assert err < tol, (name, err)


def test_fd_rglru(orc):
    rng = np.random.default_rng(10)
    inp = {"a": rng.uniform(-1, 1, (2, 7, 3)), "b": rng.normal(size=(2, 7, 3))}
    dy = rng.normal(size=(2, 7, 3))
    _fd_check(lambda i: orc.rglru_fwd(i["a"], i["b"]),
              lambda i, d: orc.rglru_bwd(i["a"], i["b"], d), inp, ["a", "b"], dy)


def test_fd_rotlru(orc):
    rng = np.random.default_rng(11)
    K = 2
    inp = {"b": rng.normal(size=(2, 6, 2 * K)), "g": rng.uniform(0.3, 1, (2, 6, K)),
           "mag": rng.uniform(0.5, 1, K), "theta": rng.uniform(-2, 2, K)}
    dy = rng.normal(size=(2, 6, 2 * K))
    _fd_check(lambda i: orc.rotlru_fwd(i["b"], i["g"], i["mag"], i["theta"]),
              lambda i, d: orc.rotlru_bwd(i["b"], i["g"], i["mag"], i["theta"], d),
              inp, ["b", "g", "mag", "theta"], dy)


@pytest.mark.parametrize("disc", ["zoh", "bilinear", "dirac", "zoh_euler"])
def test_fd_s6(orc, disc):
    rng = np.random.default_rng(12)
    B, L, D, N = 2, 5, 3, 2
    inp = {"x": rng.normal(size=(B, L, D)), "delta": rng.uniform(0.05, 0.8, (B, L, D)),
           "A": -rng.uniform(0.3, 3, (D, N)), "B": rng.normal(size=(B, L, N)),
           "C": rng.normal(size=(B, L, N)), "D": rng.normal(size=D),
           "z": rng.normal(size=(B, L, D))}
    dy = rng.normal(size=(B, L, D))
    f = lambda i: orc.s6_fwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], disc=disc)
    b = lambda i, d: orc.s6_bwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], d,
                                disc=disc)
    _fd_check(f, b, inp, ["x", "delta", "A", "B", "C", "D", "z"], dy)


@pytest.mark.parametrize("disc", ["zoh", "bilinear", "dirac", "zoh_euler"])
def test_fd_ssd(orc, disc):
    rng = np.random.default_rng(13)
    B, L, H, P, N, G = 1, 5, 4, 2, 3, 2
    inp = {"x": rng.normal(size=(B, L, H, P)), "delta": rng.uniform(0.05, 0.8, (B, L, H)),
           "A": -rng.uniform(0.3, 3, H), "B": rng.normal(size=(B, L, G, N)),
           "C": rng.normal(size=(B, L, G, N)), "D": rng.normal(size=H),
           "z": rng.normal(size=(B, L, H, P))}
    dy = rng.normal(size=(B, L, H, P))
    f = lambda i: orc.ssd_fwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], disc=disc)
    b = lambda i, d: orc.ssd_bwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], d,
                                 disc=disc)
    _fd_check(f, b, inp, ["x", "delta", "A", "B", "C", "D", "z"], dy)


def test_fd_gla(orc):
    rng = np.random.default_rng(14)
    B, L, H, K, V = 1, 5, 2, 3, 2
    inp = {"q": rng.normal(size=(B, L, H, K)), "k": rng.normal(size=(B, L, H, K)),
           "v": rng.normal(size=(B, L, H, V)), "g": rng.uniform(0.3, 1, (B, L, H))}
    dy = rng.normal(size=(B, L, H, V))
    _fd_check(lambda i: orc.gla_fwd(i["q"], i["k"], i["v"], i["g"]),
              lambda i, d: orc.gla_bwd(i["q"], i["k"], i["v"], i["g"], d),
              inp, ["q", "k", "v", "g"], dy)


def test_softplus_front_end(orc):
    """delta_softplus: the same scan on dt = softplus(delta + bias) computed outside the oracle by
    torch's softplus; the raw-delta and bias gradients by finite differences (S6 and SSD)."""
    import torch
    rng = np.random.default_rng(19)
    B, L, D, N = 2, 5, 3, 2
    inp = {"x": rng.normal(size=(B, L, D)), "delta": rng.normal(-1.0, 1.0, (B, L, D)),
           "A": -rng.uniform(0.3, 3, (D, N)), "B": rng.normal(size=(B, L, N)),
           "C": rng.normal(size=(B, L, N)), "D": rng.normal(size=D), "z": rng.normal(size=(B, L, D)),
           "bias": rng.normal(size=D)}
    dt = torch.nn.functional.softplus(torch.from_numpy(inp["delta"] + inp["bias"])).numpy()
    ref = orc.s6_fwd(inp["x"], dt, inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], disc="zoh")
    got = orc.s6_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"], disc="zoh",
                     delta_softplus=True, delta_bias=inp["bias"])
    assert rel_err(got, ref) < 1e-14
    f = lambda i: orc.s6_fwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], disc="zoh",
                             delta_softplus=True, delta_bias=i["bias"])
    b2 = lambda i, d: {**(g := orc.s6_bwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], i["z"], d,
                                          disc="zoh", delta_softplus=True, delta_bias=i["bias"])),
                       "bias": g["delta_bias"]}
    _fd_check(f, b2, inp, ["delta", "bias", "A", "x"], rng.normal(size=(B, L, D)))
    H, P, Ns, G = 4, 2, 3, 2
    si = {"x": rng.normal(size=(1, L, H, P)), "delta": rng.normal(-1.0, 1.0, (1, L, H)),
          "A": -rng.uniform(0.3, 3, H), "B": rng.normal(size=(1, L, G, Ns)), "C": rng.normal(size=(1, L, G, Ns)),
          "D": rng.normal(size=H), "bias": rng.normal(size=H)}
    fs = lambda i: orc.ssd_fwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], None, disc="zoh_euler",
                               delta_softplus=True, delta_bias=i["bias"])
    bs = lambda i, d: {**(g := orc.ssd_bwd(i["x"], i["delta"], i["A"], i["B"], i["C"], i["D"], None, d,
                                           disc="zoh_euler", delta_softplus=True, delta_bias=i["bias"])),
                       "bias": g["delta_bias"]}
    _fd_check(fs, bs, si, ["delta", "bias", "A"], rng.normal(size=(1, L, H, P)))


def test_rglru_gate_front_end(orc):
    """RG-LRU gates: the output is rglru on a = sigmoid(Lambda)^(8 r), b = sqrt(1 - a^2) i x
    evaluated here with torch (a separate evaluation of the gate formulas); all four gradients by
    finite differences."""
    import torch
    rng = np.random.default_rng(29)
    B, L, D = 2, 6, 3
    inp = {"r": rng.uniform(0.05, 0.95, (B, L, D)), "i": rng.uniform(0.05, 0.95, (B, L, D)),
           "x": rng.normal(size=(B, L, D)), "lam": rng.uniform(2.0, 6.0, D)}
    t = {k: torch.from_numpy(v) for k, v in inp.items()}
    a = torch.sigmoid(t["lam"]) ** (8.0 * t["r"])
    b = torch.sqrt(1.0 - a * a) * t["i"] * t["x"]
    assert rel_err(orc.rglru_gated_fwd(inp["r"], inp["i"], inp["x"], inp["lam"]), orc.rglru_fwd(a.numpy(), b.numpy())) < 1e-14
    _fd_check(lambda q: orc.rglru_gated_fwd(q["r"], q["i"], q["x"], q["lam"]),
              lambda q, d: orc.rglru_gated_bwd(q["r"], q["i"], q["x"], q["lam"], d),
              inp, ["r", "i", "x", "lam"], rng.normal(size=(B, L, D)))


# ------------------------------------------------------ P7: execution-mode equivalence
def test_prefix_and_stepwise_equivalence(orc):
    """Running on a prefix reproduces the full run's first steps (causality), and restarting
    from a checkpointed state reproduces the rest (recurrent vs parallel vs step-wise)."""
    rng = np.random.default_rng(15)
    B, L, D, N, S = 2, 24, 3, 2, 8
    x = rng.normal(size=(B, L, D))
    dt = rng.uniform(0.05, 0.5, (B, L, D))
    A = -rng.uniform(0.3, 3, (D, N))
    Bm, Cm = rng.normal(size=(B, L, N)), rng.normal(size=(B, L, N))
    y, ck = orc.s6_fwd(x, dt, A, Bm, Cm, None, None, disc="zoh", S=S)
    for Lp in (1, 5, 17):
        yp = orc.s6_fwd(x[:, :Lp], dt[:, :Lp], A, Bm[:, :Lp], Cm[:, :Lp], None, None, disc="zoh")
        assert rel_err(yp, y[:, :Lp]) < REL
    # one step at a time from checkpoint k: h_{t} = abar h_{t-1} + beta B x, y = C.h
    k = 2
    h = ck[k].copy()
    for t in range(k * S, L):
        ab = np.exp(dt[:, t, :, None] * A[None])
        be = np.expm1(dt[:, t, :, None] * A[None]) / A[None]
        h = ab * h + be * Bm[:, t, None, :] * x[:, t, :, None]
        assert rel_err((h * Cm[:, t, None, :]).sum(-1), y[:, t]) < 1e-11


# ----------------------------------------- initial / final state (decode and continuation)
def _split_runs(orc):
    """(name, full-run callable, state shape) for every kind on small random inputs; the callable
    takes (slice of steps, h0) and returns (y, h_final)."""
    rng = np.random.default_rng(41)
    B, L = 2, 11
    cases = []
    a = rng.uniform(-1.1, 1.1, (B, L, 3))
    b = rng.normal(size=(B, L, 3))
    cases.append(("rglru", L, lambda sl, h0: orc.rglru_fwd(a[:, sl], b[:, sl], h0=h0, final=True), (B, 3)))
    br = rng.normal(size=(B, L, 4))
    g = rng.uniform(0.5, 1.0, (B, L, 2))
    mag, th = rng.uniform(0.8, 1.0, 2), rng.uniform(0, 1, 2)
    cases.append(("rotlru", L, lambda sl, h0: orc.rotlru_fwd(br[:, sl], g[:, sl], mag, th, h0=h0, final=True),
                  (B, 4)))
    D, N = 3, 2
    x, z = rng.normal(size=(B, L, D)), rng.normal(size=(B, L, D))
    dt = rng.uniform(0.05, 0.5, (B, L, D))
    A6 = -rng.uniform(0.3, 3, (D, N))
    B6, C6, D6 = rng.normal(size=(B, L, N)), rng.normal(size=(B, L, N)), rng.normal(size=D)
    cases.append(("s6", L, lambda sl, h0: orc.s6_fwd(x[:, sl], dt[:, sl], A6, B6[:, sl], C6[:, sl], D6, z[:, sl],
                                                     disc="bilinear", h0=h0, final=True), (B, D, N)))
    H, P, Ns, G = 4, 3, 5, 2
    xs = rng.normal(size=(B, L, H, P))
    dts = rng.uniform(0.05, 0.5, (B, L, H))
    As = -rng.uniform(0.3, 3, H)
    Bs, Cs = rng.normal(size=(B, L, G, Ns)), rng.normal(size=(B, L, G, Ns))
    Ds = rng.normal(size=H)
    cases.append(("ssd", L, lambda sl, h0: orc.ssd_fwd(xs[:, sl], dts[:, sl], As, Bs[:, sl], Cs[:, sl], Ds, None,
                                                      disc="zoh", h0=h0, final=True), (B, H, P, Ns)))
    K, V = 3, 5
    q, k = rng.normal(size=(B, L, 2, K)), rng.normal(size=(B, L, 2, K))
    v, gg = rng.normal(size=(B, L, 2, V)), rng.uniform(0.5, 1.0, (B, L, 2))
    cases.append(("gla", L, lambda sl, h0: orc.gla_fwd(q[:, sl], k[:, sl], v[:, sl], gg[:, sl], h0=h0, final=True),
                  (B, 2, K, V)))
    return cases


def test_split_runs_compose(orc):
    """P7 for the state interface: L1 steps, then L - L1 steps from the returned state, equals the
    whole run (outputs and final state), for every split point and for one step at a time."""
    for name, L, run, shape in _split_runs(orc):
        y, hL = run(slice(0, L), None)
        y0, hz = run(slice(0, L), np.zeros(shape))
        assert rel_err(y0, y) == 0.0 and rel_err(hz, hL) == 0.0, name
        for L1 in (1, 4, L - 1):
            y1, h1 = run(slice(0, L1), None)
            y2, h2 = run(slice(L1, L), h1)
            assert rel_err(np.concatenate([y1, y2], axis=1), y) < REL, (name, L1)
            assert rel_err(h2, hL) < REL, (name, L1)
        h, ys = None, []
        for t in range(L):
            yt, h = run(slice(t, t + 1), h)
            ys.append(yt)
        assert rel_err(np.concatenate(ys, axis=1), y) < REL and rel_err(h, hL) < REL, name


def test_initial_state_closed_forms(orc):
    """With zero inputs the state only decays from h0: brute-force products of the per-step
    coefficients applied to h0, read out per kind.  Non-square P x N and K x V make a transposed
    state layout fail."""
    rng = np.random.default_rng(43)
    B, L = 2, 7
    # rglru: y_t = (prod_{r<=t} a_r) h0
    a = rng.uniform(-1.1, 1.1, (B, L, 3))
    h0 = rng.normal(size=(B, 3))
    y = orc.rglru_fwd(a, np.zeros((B, L, 3)), h0=h0)
    assert rel_err(y, np.cumprod(a, axis=1) * h0[:, None]) < REL
    # rotlru: h_t = (prod m_r) e^{i (t+1) theta} h0
    g = rng.uniform(0.5, 1.0, (B, L, 2))
    mag, th = rng.uniform(0.8, 1.0, 2), rng.uniform(0, 1, 2)
    h0 = rng.normal(size=(B, 4))
    y = orc.rotlru_fwd(np.zeros((B, L, 4)), g, mag, th, h0=h0)
    hc = h0[:, 0::2] + 1j * h0[:, 1::2]
    ref = np.cumprod(mag * g, axis=1) * np.exp(1j * th * np.arange(1, L + 1)[:, None]) * hc[:, None]
    assert rel_err(y[..., 0::2], ref.real) < REL and rel_err(y[..., 1::2], ref.imag) < REL
    # SSD: y_t[p] = sum_n C_t[n] (prod_{r<=t} e^{dt_r A}) h0[p, n]
    H, P, N = 2, 3, 5
    dt = rng.uniform(0.05, 0.5, (B, L, H))
    A = -rng.uniform(0.3, 3, H)
    Cm = rng.normal(size=(B, L, 1, N))
    h0 = rng.normal(size=(B, H, P, N))
    y = orc.ssd_fwd(np.zeros((B, L, H, P)), dt, A, rng.normal(size=(B, L, 1, N)), Cm, None, None, h0=h0)
    dec = np.exp(np.cumsum(dt * A, axis=1))                       # [B, L, H]
    ref = np.einsum("bln,bhpn,blh->blhp", Cm[:, :, 0], h0, dec)
    assert rel_err(y, ref) < REL
    # S6: y_t = (sum_n C_t[n] prod_r abar_r[n] h0[n]) silu(z_t)
    D6, N6 = 2, 3
    dt6 = rng.uniform(0.05, 0.5, (B, L, D6))
    A6 = -rng.uniform(0.3, 3, (D6, N6))
    C6, z6 = rng.normal(size=(B, L, N6)), rng.normal(size=(B, L, D6))
    h0 = rng.normal(size=(B, D6, N6))
    y = orc.s6_fwd(np.zeros((B, L, D6)), dt6, A6, rng.normal(size=(B, L, N6)), C6, None, z6, disc="zoh", h0=h0)
    dec6 = np.exp(np.cumsum(dt6[..., None] * A6[None, None], axis=1))   # [B, L, D, N]
    ref = np.einsum("bln,bldn,bdn->bld", C6, dec6, h0) * silu(z6)
    assert rel_err(y, ref) < REL
    # GLA: o_t = (prod_{r<=t} g_r) S0^T q_t
    K, V = 3, 5
    gg = rng.uniform(0.5, 1.0, (B, L, 2))
    q = rng.normal(size=(B, L, 2, K))
    S0 = rng.normal(size=(B, 2, K, V))
    o = orc.gla_fwd(q, np.zeros((B, L, 2, K)), np.zeros((B, L, 2, V)), gg, h0=S0)
    ref = np.einsum("blh,bhkv,blhk->blhv", np.cumprod(gg, axis=1), S0, q)
    assert rel_err(o, ref) < REL


# ------------------------------------------------------------------- golden fixtures
def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_rglru_halving(orc):
    g = _golden("rglru_halving.json")
    y = orc.rglru_fwd(np.array(g["a"])[None, :, None], np.array(g["b"])[None, :, None])
    assert np.array_equal(y[0, :, 0], np.array(g["y"]))


def test_golden_rotlru_quarter_turn(orc):
    g = _golden("rotlru_quarter_turn.json")
    L = len(g["y_re"])
    b = np.zeros((1, L, 2))
    b[0, 0] = g["b0"]
    y = orc.rotlru_fwd(b, np.ones((1, L, 1)), np.ones(1), np.array([g["theta"]]))
    assert np.max(np.abs(y[0, :, 0] - np.array(g["y_re"]))) < 1e-15
    assert np.max(np.abs(y[0, :, 1] - np.array(g["y_im"]))) < 1e-15


def test_golden_gla_two_steps(orc):
    g = _golden("gla_two_steps.json")
    q, k, v, gg = (np.array(g[n], dtype=float) for n in ("q", "k", "v", "g"))
    o = orc.gla_fwd(q, k, v, gg)
    assert np.allclose(o, np.array(g["o"]), rtol=0, atol=1e-15)


# ------------------------------------------------------ the pins catch planted mistakes
def test_planted_mistakes_are_caught(tmp_path):
    """Build copies of the oracle with one plausible mistake each and check that the pins above
    reject every copy (run on the CPU only; the real oracle is untouched)."""
    import subprocess
    src = open(os.path.join(os.path.dirname(__file__), "..", "oracle", "lr_oracle.c")).read()
    mutants = {
        # forward uses the previous step's gate (index shifted by one)
        "shifted_gate": ("h = a[i] * h + b[i];", "h = (t > 0 ? a[i - D] : a[i]) * h + b[i];"),
        # rotation applied clockwise (sign of the imaginary part of lambda)
        "wrong_rotation": ("double lr = m * c, li = m * s;", "double lr = m * c, li = -m * s;"),
        # GLA state update without the forget gate (the decay g_t dropped)
        "gla_dropped_decay": ("St[i * V + j] = gt * St[i * V + j] + kt[i] * vt[j];",
                              "St[i * V + j] = St[i * V + j] + kt[i] * vt[j];"),
        # ZOH beta = dt instead of expm1(u)/A
        "euler_beta": ("*beta = (A != 0.0) ? expm1(u) / A : dt;", "*beta = dt;"),
        # SSD ignores its initial state
        "ssd_h0_ignored": ("                if (h0)\n                    memcpy(h, h0 + (bi * H + hh) * P * N",
                           "                if (0)\n                    memcpy(h, h0 + (bi * H + hh) * P * N"),
        # rglru returns the first step's state as the final one
        "rglru_stale_final": ("if (hL) hL[bi * D + d] = h;", "if (hL) hL[bi * D + d] = y[(bi * L) * D + d];"),
        # ZOH-Euler: the dt-dependence of beta dropped from the gradient
        "euler_dbeta_dropped": ("*db_ddt = disc == ORC_DISC_ZOH_EULER ? 1.0 : 0.0;", "*db_ddt = 0.0;"),
        # dirac read as an Euler input (beta = dt)
        "dirac_as_euler": ("        *beta = 1.0;", "        *beta = dt;"),
    }
    import oracle as real
    for name, (old, new) in mutants.items():
        assert old in src, name
        csrc = tmp_path / (name + ".c")
        csrc.write_text(src.replace(old, new, 1))
        so = tmp_path / (name + ".so")
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                               str(csrc), "-lm"])
        saved = real._lib
        real._lib = real.load(str(so))
        try:
            failed = 0
            for test, args in ((test_rglru_closed_form, ()), (test_rotlru_closed_form, ()),
                               (test_gla_closed_form, ()),
                               (test_s6_closed_form_with_scipy_discretisation, ("zoh",)),
                               (test_split_runs_compose, ()), (test_initial_state_closed_forms, ()),
                               (test_s6_closed_form_with_scipy_discretisation, ("dirac",)),
                               (test_fd_s6, ("zoh_euler",))):
                try:
                    test(real, *args)
                except AssertionError:
                    failed += 1
            assert failed >= 1, name
        finally:
            real._lib = saved
