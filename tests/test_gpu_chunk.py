"""GPU parity of the chunked-matmul kinds (SSD, GLA; tcgen05 tensor cores) against the fp64
oracle.  bf16 I/O, tolerance max|err| <= 2e-2 max|ref| per tensor (y, checkpoints, every
gradient).  Cases cover several chunks chained through the forward and reverse look-backs, a
ragged last chunk (L not a multiple of 128), a single chunk, several heads per group (SSD), both
value widths (64, 128), and the workloads at full size on sampled heads."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, run_gpu, to64
from selective_state_space_09_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2

# (B, L, H, P, G).  Also covers: dt boxes by TMA (H a multiple of 8) and by per-lane loads (other
# H); several head blocks adding into dB, dC rows zeroed by the scan kernel, with more chunks than
# heads per group (1, 1000, 2: each head zeroes four chunks' rows).
SSD_CASES = [(1, 512, 4, 64, 1), (2, 300, 8, 64, 2), (1, 128, 2, 64, 1), (1, 77, 8, 64, 1),
             (1, 384, 12, 64, 1), (2, 260, 10, 64, 2), (1, 520, 40, 64, 2), (1, 1000, 2, 64, 1)]
SSD_FWD = ("ssd_state_scan+ssd_chunk_out",)
SSD_BWD = ("ssd_state_scan+ssd_chunk_grad+ssd_param_reduce",)


def _ssd_ref(inp, disc="zoh"):
    a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], None)
    ry, rck = oracle.ssd_fwd(*a, disc=disc, S=128)
    rg = oracle.ssd_bwd(*a, inp["dy"], disc=disc)
    return ry, rck, rg


@pytest.mark.parametrize("wide", [False, True])
@pytest.mark.parametrize("B,L,H,P,G", SSD_CASES)
def test_ssd_parity(B, L, H, P, G, wide):
    """wide: the largest head blocks per CTA (several heads pipelined through one CTA)."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(B, L, H, P, 128, G=G, seed=B * 31 + L)
    flags = lrscan.TEST_MAX_HEAD_BLOCK if wide else 0
    y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc="zoh", chunk=128, flags=flags)
    ry, rck, rg = _ssd_ref(inp)
    assert_close("y", y, ry, TOL)
    assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)   # kernel state [N, P], oracle [P, N]
    assert_close("dx", gr["dx"], rg["x"], TOL)
    assert_close("ddelta", gr["ddelta"], rg["delta"], TOL)
    assert_close("dA", gr["dA"], rg["A"], TOL)
    assert_close("dB", gr["dBm"], rg["B"], TOL)
    assert_close("dC", gr["dCm"], rg["C"], TOL)
    assert_close("dD", gr["dDskip"], rg["D"], TOL)
    assert disp[0] in SSD_FWD and disp[1] in SSD_BWD
    assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("disc", ["dirac", "zoh_euler"])
@pytest.mark.parametrize("B,L,H,P,G", [(1, 512, 4, 64, 1), (2, 260, 10, 64, 2)])
def test_ssd_parity_other_discretisations(B, L, H, P, G, disc):
    """dirac (beta = 1) and ZOH-Euler (beta = dt): the same kernels with another beta and its
    derivatives."""
    inp = inputs.ssd(B, L, H, P, 128, G=G, seed=B * 37 + L)
    y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc=disc, chunk=128)
    ry, rck, rg = _ssd_ref(inp, disc)
    assert_close("y", y, ry, TOL)
    assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)
    for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D")):
        assert_close(name, gr[name], rg[ref], TOL)
    assert disp[0] in SSD_FWD and disp[1] in SSD_BWD
    assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("B,L,H,P,G,dt_shift", [(1, 512, 4, 64, 1, 0.0), (2, 260, 10, 64, 2, 0.0),
                                                 (1, 77, 8, 64, 1, 0.0), (1, 384, 12, 64, 1, 1.5)])
def test_ssd_parity_bilinear(B, L, H, P, G, dt_shift):
    """Bilinear (Tustin) SSD on the chunked path: abar = (1 + u) / (1 - u), u = dt A / 2, is negative
    wherever dt |A| > 2 and passes through 0 at dt |A| = 2.  The decays are carried as a log
    magnitude and a sign parity; the decay gradient is formed from sums whose every term holds
    abar_t, so dividing by abar_t stays accurate near 0.  dt_shift raises the step lengths so that
    most steps have abar < 0."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(B, L, H, P, 128, G=G, seed=B * 41 + L)
    if dt_shift:
        inp["delta"] = (inp["delta"].float() + dt_shift).to(torch.bfloat16)
    u = 0.5 * inp["delta"].double() * inp["A"].double()
    neg = float((1.0 + u < 0).double().mean())
    assert neg > 0.05, neg  # the case exercises negative decays
    for flags in (0, lrscan.TEST_MAX_HEAD_BLOCK):
        y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc="bilinear", chunk=128, flags=flags)
        ry, rck, rg = _ssd_ref(inp, "bilinear")
        assert_close("y", y, ry, TOL)
        assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)
        for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D")):
            assert_close(name, gr[name], rg[ref], TOL)
        assert disp[0] in SSD_FWD and disp[1] in SSD_BWD
        assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("disc", ["zoh", "bilinear", "zoh_euler"])
@pytest.mark.parametrize("B,L,H,P,G", [(1, 512, 4, 64, 1), (2, 260, 10, 64, 2), (1, 77, 8, 64, 1)])
def test_ssd_parity_z_gate(B, L, H, P, G, disc):
    """The silu(z) gate on the chunked SSD path: y = (C h + D x) silu(z); the backward forms
    ds = dy silu(z) once, and dz from the readout before the gate (one more product, P x)."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(B, L, H, P, 128, G=G, seed=B * 43 + L, with_z=True)
    for flags in (0, lrscan.TEST_MAX_HEAD_BLOCK):
        y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc=disc, chunk=128, flags=flags)
        a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
        ry, rck = oracle.ssd_fwd(*a, disc=disc, S=128)
        rg = oracle.ssd_bwd(*a, inp["dy"], disc=disc)
        assert_close("y", y, ry, TOL)
        assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)
        for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D"),
                          ("dz", "z")):
            assert_close(name, gr[name], rg[ref], TOL)
        assert disp[0] in SSD_FWD
        assert disp[1] == "ssd_gate_prep+ssd_state_scan+ssd_chunk_grad+ssd_param_reduce"
        assert plan.device_error() == (0, 0)


def test_ssd_bilinear_softplus_front_end():
    """Bilinear with dt = softplus(delta + bias) formed in the kernels."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(1, 300, 8, 64, 128, G=1, seed=29)
    gen = torch.Generator().manual_seed(8)
    inp["delta"] = (torch.randn(inp["delta"].shape, generator=gen) - 1.0).to(torch.bfloat16)
    inp["delta_bias"] = 0.5 * torch.randn(8, generator=gen)
    y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc="bilinear", chunk=128, flags=lrscan.DELTA_SOFTPLUS)
    a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], None)
    ry = oracle.ssd_fwd(*a, disc="bilinear", delta_softplus=True, delta_bias=inp["delta_bias"])
    rg = oracle.ssd_bwd(*a, inp["dy"], disc="bilinear", delta_softplus=True, delta_bias=inp["delta_bias"])
    assert_close("y", y, ry, TOL)
    for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D"),
                      ("ddelta_bias", "delta_bias")):
        assert_close(name, gr[name], rg[ref], TOL)
    assert plan.device_error() == (0, 0)


def test_ssd_softplus_front_end():
    """LR_DELTA_SOFTPLUS on the chunked SSD path: gradients for the raw delta and the bias."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(2, 260, 10, 64, 128, G=2, seed=23)
    gen = torch.Generator().manual_seed(6)
    inp["delta"] = (torch.randn(inp["delta"].shape, generator=gen) - 2.0).to(torch.bfloat16)
    inp["delta_bias"] = 0.5 * torch.randn(10, generator=gen)
    y, ck, gr, plan, disp = run_gpu("ssd", inp, 128, disc="zoh", chunk=128, flags=lrscan.DELTA_SOFTPLUS)
    a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], None)
    ry = oracle.ssd_fwd(*a, disc="zoh", delta_softplus=True, delta_bias=inp["delta_bias"])
    rg = oracle.ssd_bwd(*a, inp["dy"], disc="zoh", delta_softplus=True, delta_bias=inp["delta_bias"])
    assert_close("y", y, ry, TOL)
    for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D"),
                      ("ddelta_bias", "delta_bias")):
        assert_close(name, gr[name], rg[ref], TOL)
    assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("kind", ["ssd", "gla"])
def test_withheld_slot_times_out_and_context_survives(kind):
    """Failure path of the scan / chunk-kernel protocol: the state scan never counts slot 0, so the
    chunk kernels of the first chunk wait out their bound, record LR_ERR_TIMEOUT (status 6) with
    the waiting site and finish.  A normal call afterwards on the same context is correct."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(1, 300, 8, 64, 128, seed=41) if kind == "ssd" else inputs.gla(1, 300, 8, 128, 128, seed=41)
    disc = "zoh" if kind == "ssd" else "none"
    y, ck, gr, plan, _ = run_gpu(kind, inp, 128, disc=disc, chunk=128, flags=lrscan.TEST_WITHHOLD_CARRY)
    status, info = plan.device_error()
    assert status == 6 and info in ((716, 728) if kind == "ssd" else (813, 828)), (status, info)
    y, ck, gr, plan, _ = run_gpu(kind, inp, 128, disc=disc, chunk=128)
    assert plan.device_error() == (0, 0)
    if kind == "ssd":
        ref = oracle.ssd_fwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], None, disc="zoh")
    else:
        ref = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"])
    assert_close("y", y, ref, TOL)


def test_ssd_head_blocking_bitwise():
    """The head blocking of the output kernel changes only which CTA computes a head."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(1, 640, 24, 64, 128, G=1, seed=5)
    a = run_gpu("ssd", inp, 128, disc="zoh", chunk=128)
    b = run_gpu("ssd", inp, 128, disc="zoh", chunk=128, flags=lrscan.TEST_MAX_HEAD_BLOCK)
    assert torch.equal(a[0], b[0])
    assert torch.equal(a[1], b[1])


def test_ssd_deterministic():
    """With at most two head blocks per group (the widest blocks, 24 heads -> 16 + 8) every output,
    dB and dC included, is bitwise reproducible: each dB / dC element is the sum of at most two
    reduction-adds onto zero."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.ssd(2, 700, 24, 64, 128, G=1, seed=8)
    a = run_gpu("ssd", inp, 128, disc="zoh", chunk=128, flags=lrscan.TEST_MAX_HEAD_BLOCK)
    b = run_gpu("ssd", inp, 128, disc="zoh", chunk=128, flags=lrscan.TEST_MAX_HEAD_BLOCK)
    assert torch.equal(a[0], b[0])
    for k in a[2]:
        assert torch.equal(a[2][k], b[2][k]), k


# (B, L, H, V): the gate fetched by TMA boxes (H a multiple of 8) and by per-lane loads (other H);
# V = 128 is scanned as two 64-column halves
GLA_CASES = [(1, 512, 2, 128), (2, 300, 3, 128), (1, 128, 1, 128), (2, 200, 2, 64), (1, 300, 8, 128),
             (2, 260, 16, 64)]


@pytest.mark.parametrize("B,L,H,V", GLA_CASES)
def test_gla_parity(B, L, H, V):
    inp = inputs.gla(B, L, H, 128, V, seed=B * 17 + L)
    y, ck, gr, plan, disp = run_gpu("gla", inp, 128, chunk=128)
    ry, rck = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], S=128)
    rg = oracle.gla_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["dy"])
    assert_close("o", y, ry, TOL)
    assert_close("ckpt", ck, rck, TOL)
    for gk, rk in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g")):
        assert_close(gk, gr[gk], rg[rk], TOL)
    assert disp == ("gla_state_scan+gla_chunk_out", "gla_state_scan+gla_chunk_grad")
    assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("S", [256, 512])
@pytest.mark.parametrize("case", ["ssd", "ssd_bilinear_z", "gla128", "gla64"])
def test_segments_longer_than_a_chunk(case, S):
    """Checkpoint segments of several chunks: the checkpoint holds the f32 state entering each
    segment only (no bf16 copies), the forward keeps the tiles of every chunk in its workspace, and
    the backward rebuilds them from the segment states before the gradient kernels read them.  The
    checkpoints match the oracle's at segment S; outputs and gradients match the oracle, and equal
    the one-chunk-segment run bitwise (the rebuilt tiles are the forward's)."""
    from selective_state_space_09_b200 import lrscan
    L = 700  # 6 chunks, the last one ragged: segments of 2 + 2 + 2 (S = 256) or 4 + 2 (S = 512)
    if case.startswith("ssd"):
        kind, disc = "ssd", ("bilinear" if case == "ssd_bilinear_z" else "zoh")
        inp = inputs.ssd(2, L, 8, 64, 128, G=2, seed=S + 3, with_z=case == "ssd_bilinear_z")
    else:
        kind, disc = "gla", "none"
        inp = inputs.gla(1, L, 4, 128, 128 if case == "gla128" else 64, seed=S + 5)
    y, ck, gr, plan, disp = run_gpu(kind, inp, S, disc=disc, chunk=128)
    y1, ck1, gr1, plan1, _ = run_gpu(kind, inp, 128, disc=disc, chunk=128)
    assert plan.device_error() == (0, 0) and plan1.device_error() == (0, 0)
    nseg = -(-L // S)
    state = 2 * 8 * 128 * 64 if kind == "ssd" else 1 * 4 * 128 * inp["v"].shape[-1]
    assert lrscan.ckpt_bytes(plan.desc) == nseg * state * 4
    assert kind + "_state_recompute" in disp[1].split("+")
    if kind == "ssd":
        a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
        ry, rck = oracle.ssd_fwd(*a, disc=disc, S=S)
        rg = oracle.ssd_bwd(*a, inp["dy"], disc=disc)
        assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)
        names = (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"), ("dDskip", "D"))
        if inp["z"] is not None:
            names += (("dz", "z"),)
    else:
        ry, rck = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], S=S)
        rg = oracle.gla_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["dy"])
        assert_close("ckpt", ck, rck, TOL)
        names = (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"))
    assert_close("y", y, ry, TOL)
    for gk, rk in names:
        assert_close(gk, gr[gk], rg[rk], TOL)
    # the same numbers as with one chunk per segment (dB, dC: sums of reduction-adds over head
    # blocks in arbitrary order, bitwise only up to two blocks per group)
    assert torch.equal(y, y1)
    assert torch.equal(ck, ck1[::S // 128])
    for gk, _ in names:
        if gk in ("dBm", "dCm"):
            assert_close(gk, gr[gk], to64(gr1[gk]), 1e-5)
        else:
            assert torch.equal(gr[gk], gr1[gk]), gk


def test_gla_deterministic():
    inp = inputs.gla(2, 384, 2, 128, 128, seed=3)
    a = run_gpu("gla", inp, 128, chunk=128)
    b = run_gpu("gla", inp, 128, chunk=128)
    assert torch.equal(a[0], b[0])
    for k in a[2]:
        assert torch.equal(a[2][k], b[2][k]), k


@pytest.mark.slow
def test_ssd_full_size():
    """The SSD workload (B=2, H=32, P=64, N=128, L=4096) against the oracle run on the whole
    workload (64 independent (batch row, head) units on the host cores): every tensor compared
    whole, relative to its own max."""
    import os
    w = inputs.WORKLOADS["ssd"]
    inp = inputs.ssd(w["B"], w["L"], w["H"], w["P"], w["N"], seed=0, device="cuda")
    y, ck, gr, plan, _ = run_gpu("ssd", inp, w["segment"], disc="zoh", chunk=w["chunk"])
    assert plan.device_error() == (0, 0)
    oracle.set_threads(max(8, min(32, os.cpu_count() or 8)))
    ref = {k: (to64(v) if v is not None else None) for k, v in inp.items()}
    ry, rck, rg = _ssd_ref(ref)
    assert_close("y", y, ry, TOL)
    assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)
    for gk, rk in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"),
                   ("dDskip", "D")):
        assert_close(gk, gr[gk], rg[rk], TOL)


@pytest.mark.slow
def test_gla_full_size_sampled():
    """The GLA workload (B=4, H=16, K=V=128, L=2048) on sampled (batch row, head) units."""
    w = inputs.WORKLOADS["gla"]
    inp = inputs.gla(w["B"], w["L"], w["H"], w["K"], w["V"], seed=0, device="cuda")
    y, ck, gr, plan, _ = run_gpu("gla", inp, w["segment"], chunk=w["chunk"])
    assert plan.device_error() == (0, 0)
    oracle.set_threads(4)
    for b, h in ((0, 0), (3, 15), (1, 7)):
        sub = {k: to64(v[b:b + 1, :, h:h + 1]) for k, v in inp.items()}
        ry, rck = oracle.gla_fwd(sub["q"], sub["k"], sub["v"], sub["g"], S=128)
        rg = oracle.gla_bwd(sub["q"], sub["k"], sub["v"], sub["g"], sub["dy"])
        assert_close("o[%d,%d]" % (b, h), y[b:b + 1, :, h:h + 1], ry, TOL)
        assert_close("ckpt[%d,%d]" % (b, h), ck[:, b:b + 1, h:h + 1], rck, TOL)
        for gk, rk in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g")):
            assert_close("%s[%d,%d]" % (gk, b, h), gr[gk][b:b + 1, :, h:h + 1], rg[rk], TOL)
