"""GPU parity of the S6 selective scan (ZOH and bilinear, fused D skip and silu(z)) against the
fp64 oracle: bf16 I/O, tolerance max|err| <= 2e-2 max|ref| per tensor (y, checkpoints, dx,
d(dt), dz, dA, dB, dC, dD).  Cases cover several 64-channel blocks, ragged channel blocks and
ragged last segments, L = 1, the optional z gate and D skip, and the S6 workload at full size on
sampled channels (dB, dC, which sum over all channels, checked on sampled time steps)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, gpu_inputs, run_gpu, to64
from selective_state_space_09_b200 import inputs, lrscan

pytestmark = pytest.mark.gpu
TOL = 2e-2

CASES = [
    # B, L, D, S, disc, with_z, with_D
    (2, 200, 128, 64, "zoh", True, True),      # ragged last segment, 2 channel blocks
    (2, 200, 128, 64, "bilinear", True, True),
    (1, 77, 96, 16, "zoh", True, True),        # ragged channel block (96 = 64 + 32)
    (3, 64, 64, 8, "bilinear", False, True),   # no gate
    (1, 40, 64, 32, "zoh", True, False),       # no D skip
    (1, 1, 64, 8, "zoh", True, True),          # single step
    (2, 129, 136, 64, "bilinear", True, True),
    (2, 200, 128, 64, "dirac", True, True),    # beta = 1
    (1, 77, 96, 16, "zoh_euler", True, True),  # beta = dt
    (2, 129, 136, 64, "zoh_euler", False, True),
    (1, 1, 64, 8, "dirac", True, False),
]


def _oracle(inp, disc, S):
    args = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
    y, ck = oracle.s6_fwd(*args, disc=disc, S=S)
    g = oracle.s6_bwd(*args, inp["dy"], disc=disc)
    return y, ck, g


@pytest.mark.parametrize("B,L,D,S,disc,with_z,with_D", CASES)
def test_s6_parity(B, L, D, S, disc, with_z, with_D):
    inp = inputs.s6(B, L, D, 16, seed=B * 7 + L, with_z=with_z, with_D=with_D)
    y, ck, gr, plan, disp = run_gpu("s6", inp, S, disc=disc)
    ry, rck, rg = _oracle(inp, disc, S)
    assert_close("y", y, ry, TOL)
    assert_close("ckpt", ck, rck, 1e-3)
    assert_close("dx", gr["dx"], rg["x"], TOL)
    assert_close("ddelta", gr["ddelta"], rg["delta"], TOL)
    assert_close("dA", gr["dA"], rg["A"], TOL)
    assert_close("dB", gr["dBm"], rg["B"], TOL)
    assert_close("dC", gr["dCm"], rg["C"], TOL)
    if with_D:
        assert_close("dD", gr["dDskip"], rg["D"], TOL)
    if with_z:
        assert_close("dz", gr["dz"], rg["z"], TOL)
    assert disp == ("s6_fwd_" + disc, "s6_bwd_%s+s6_param_reduce" % disc)
    assert plan.device_error() == (0, 0)


def test_s6_deterministic():
    inp = inputs.s6(2, 150, 128, 16, seed=9)
    a = run_gpu("s6", inp, 64, disc="zoh")
    b = run_gpu("s6", inp, 64, disc="zoh")
    assert torch.equal(a[0], b[0])
    for k in a[2]:
        assert torch.equal(a[2][k], b[2][k]), k


@pytest.mark.slow
@pytest.mark.parametrize("disc", ["zoh", "bilinear"])
def test_s6_full_size_sampled(disc):
    """The S6 workload (B=8, D=2048, N=16, L=2048, S=64).  The oracle recomputes sampled
    channels over every batch row (so dA and dD, sums over batch and time, are exact), and dB, dC
    on batch row 0 (sums over all 2048 channels)."""
    name = "s6_" + disc
    w = inputs.WORKLOADS[name]
    inp = inputs.s6(w["B"], w["L"], w["D"], w["N"], seed=0, device="cuda")
    y, ck, gr, plan, _ = run_gpu("s6", inp, w["segment"], disc=disc)
    assert plan.device_error() == (0, 0)
    oracle.set_threads(8)
    rng = np.random.default_rng(1)
    chans = sorted(set([0, w["D"] - 1] + list(rng.integers(0, w["D"], size=4))))
    for dch in chans:
        sl = slice(dch, dch + 1)
        sub = {"x": inp["x"][:, :, sl], "delta": inp["delta"][:, :, sl], "A": inp["A"][sl],
               "Bm": inp["Bm"], "Cm": inp["Cm"], "Dskip": inp["Dskip"][sl], "z": inp["z"][:, :, sl],
               "dy": inp["dy"][:, :, sl]}
        sub = {k: to64(v) for k, v in sub.items()}
        ry, rck, rg = _oracle(sub, disc, w["segment"])
        assert_close("y[%d]" % dch, y[:, :, sl], ry, TOL)
        assert_close("ckpt[%d]" % dch, ck[:, :, sl], rck, 1e-3)
        for gk, rk in (("dx", "x"), ("ddelta", "delta"), ("dz", "z")):
            assert_close("%s[%d]" % (gk, dch), gr[gk][:, :, sl], rg[rk], TOL)
        assert_close("dA[%d]" % dch, gr["dA"][sl], rg["A"], TOL)
        assert_close("dD[%d]" % dch, gr["dDskip"][sl], rg["D"], TOL)
    # dB, dC of batch row 0: need every channel of that row
    sub = {k: (to64(v[0:1]) if k not in ("A", "Dskip") else to64(v)) for k, v in inp.items()}
    _, _, rg = _oracle(sub, disc, w["segment"])
    assert_close("dB[b=0]", gr["dBm"][0:1], rg["B"], TOL)
    assert_close("dC[b=0]", gr["dCm"][0:1], rg["C"], TOL)


@pytest.mark.parametrize("disc", ["zoh", "bilinear"])
def test_s6_full_state_mode(disc):
    """LR_FULL_STATE: every step's state checkpointed (the oracle's segment-1 checkpoints) and read
    by the backward; outputs and gradients equal the default mode's bitwise."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.s6(2, 200, 128, 16, seed=9)
    y0, _, g0, _, _ = run_gpu("s6", inp, 64, disc=disc)
    y1, ck, g1, plan, _ = run_gpu("s6", inp, 64, disc=disc, flags=lrscan.FULL_STATE)
    assert ck.shape[0] == 200
    _, rck = oracle.s6_fwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"],
                           disc=disc, S=1)
    assert_close("full-state ckpt", ck, rck, TOL)
    assert torch.equal(y0, y1)
    for k in g0:
        assert torch.equal(g0[k], g1[k]), k
    assert plan.device_error() == (0, 0)


@pytest.mark.parametrize("disc", ["zoh", "zoh_euler"])
def test_s6_softplus_front_end(disc):
    """LR_DELTA_SOFTPLUS: dt = softplus(delta + bias) in the kernels; gradients for the raw delta
    and the bias against the oracle; the autograd wrapper gives the same values."""
    inp = inputs.s6(2, 200, 128, 16, seed=21)
    gen = torch.Generator().manual_seed(5)
    inp["delta"] = (torch.randn(inp["delta"].shape, generator=gen) - 2.0).to(torch.bfloat16)
    inp["delta_bias"] = 0.5 * torch.randn(128, generator=gen)
    y, ck, gr, plan, disp = run_gpu("s6", inp, 64, disc=disc, flags=lrscan.DELTA_SOFTPLUS)
    a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
    ry = oracle.s6_fwd(*a, disc=disc, delta_softplus=True, delta_bias=inp["delta_bias"])
    rg = oracle.s6_bwd(*a, inp["dy"], disc=disc, delta_softplus=True, delta_bias=inp["delta_bias"])
    assert_close("y", y, ry, TOL)
    for name, ref in (("dx", "x"), ("ddelta", "delta"), ("dA", "A"), ("dBm", "B"), ("dCm", "C"),
                      ("dDskip", "D"), ("dz", "z"), ("ddelta_bias", "delta_bias")):
        assert_close(name, gr[name], rg[ref], TOL)
    assert plan.device_error() == (0, 0)
    # the autograd wrapper (lrscan.s6) runs the same kernels
    g = gpu_inputs(inp)
    leaves = {k: g[k].clone().requires_grad_(True) for k in ("delta", "delta_bias")}
    out = lrscan.s6(g["x"], leaves["delta"], g["A"], g["Bm"], g["Cm"], g["Dskip"], g["z"], disc=disc, segment=64,
                    delta_softplus=True, delta_bias=leaves["delta_bias"])
    out.backward(g["dy"])
    assert torch.equal(out, y)
    assert torch.equal(leaves["delta"].grad, gr["ddelta"]) and torch.equal(leaves["delta_bias"].grad, gr["ddelta_bias"])
