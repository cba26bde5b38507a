"""GPU parity of the decode / continuation path (lr_step) against the fp64 oracle, and the
equivalence of execution modes (pin P7 at full scale).

* Parity: from a random initial state, one call of L steps gives the oracle's outputs and final
  state (the oracle's initial / final state interface, pinned in test_oracle_pins.py).
* Modes: one call of L steps, L calls of one step with the state updated in place, and the same L
  steps replayed from a CUDA graph are bitwise identical (the same kernel runs each step).
* Full scale: on the SSD workload (B=2, H=32, P=64, N=128, L=4096, bf16) decoding every token
  from a CUDA graph reproduces the chunked scan's outputs and, on a slice of heads, the oracle's
  outputs and final state.
Tolerances as for the scan: max|err| <= 1e-5 max|ref| with fp32 I/O, 2e-2 max|ref| with bf16 I/O,
per tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, assert_close, gpu_inputs, to64
from selective_state_space_09_b200 import inputs, lrscan

pytestmark = pytest.mark.gpu

CASES = [
    # kind, shape, io, disc
    ("rglru", dict(B=2, L=7, D=40), "f32", "none"),
    ("rglru", dict(B=3, L=1, D=96), "bf16", "none"),
    ("rotlru", dict(B=2, L=9, D=24), "f32", "none"),
    ("rotlru", dict(B=1, L=1, D=64), "bf16", "none"),
    ("s6", dict(B=2, L=6, D=48, N=16), "bf16", "zoh"),
    ("s6", dict(B=1, L=3, D=20, N=5), "f32", "bilinear"),
    ("ssd", dict(B=2, L=5, H=4, P=40, N=32, G=2), "bf16", "zoh"),
    ("ssd", dict(B=1, L=2, H=3, P=64, N=128, G=1), "f32", "bilinear"),
    ("s6", dict(B=2, L=4, D=32, N=16), "f32", "dirac"),
    ("ssd", dict(B=1, L=3, H=2, P=16, N=64, G=1), "bf16", "zoh_euler"),
    ("gla", dict(B=2, L=4, H=3, K=48, V=72), "bf16", "none"),
    ("gla", dict(B=1, L=1, H=2, K=128, V=128), "f32", "none"),
]


def make_inputs(kind, shape, io, seed):
    if kind == "rglru":
        return inputs.rglru(shape["B"], shape["L"], shape["D"], seed=seed, io=io)
    if kind == "rotlru":
        return inputs.rotlru(shape["B"], shape["L"], shape["D"], seed=seed, io=io)
    if kind == "s6":
        return inputs.s6(shape["B"], shape["L"], shape["D"], shape["N"], seed=seed, io=io)
    if kind == "ssd":
        return inputs.ssd(shape["B"], shape["L"], shape["H"], shape["P"], shape["N"], shape["G"], seed=seed,
                          io=io, with_z=True)
    return inputs.gla(shape["B"], shape["L"], shape["H"], shape["K"], shape["V"], seed=seed, io=io)


def oracle_run(kind, inp, disc, h0):
    """(y, final state) of the oracle from initial state h0 (the GPU's layout; None = zero)."""
    if kind == "rglru":
        return oracle.rglru_fwd(inp["a"], inp["b"], h0=h0, final=True)
    if kind == "rotlru":
        return oracle.rotlru_fwd(inp["b"], inp["g"], inp["mag"], inp["theta"], h0=h0, final=True)
    if kind == "s6":
        return oracle.s6_fwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp.get("Dskip"),
                             inp.get("z"), disc=disc, h0=h0, final=True)
    if kind == "ssd":  # the oracle's SSD state is [B, H, P, N]; lr_step's is [B, H, N, P]
        h0p = None if h0 is None else np.swapaxes(h0, 2, 3)
        y, hL = oracle.ssd_fwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp.get("Dskip"),
                               inp.get("z"), disc=disc, h0=h0p, final=True)
        return y, np.swapaxes(hL, 2, 3)
    return oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], h0=h0, final=True)


def api_inputs(kind, inp):
    return {k: v for k, v in inp.items() if k != "dy"}


def out_like(kind, g):
    return torch.empty_like(g["b" if kind in ("rglru", "rotlru") else ("v" if kind == "gla" else "x")])


@pytest.mark.parametrize("kind,shape,io,disc", CASES)
def test_step_parity(kind, shape, io, disc):
    inp = make_inputs(kind, shape, io, seed=7 + shape["L"])
    g = gpu_inputs(api_inputs(kind, inp))
    desc = lrscan.desc_for(kind, g, 1, disc)
    tol = TOL[torch.float32 if io == "f32" else torch.bfloat16]
    shp = lrscan.state_shape(desc)
    h0 = torch.randn(shp, dtype=torch.float32, generator=torch.Generator().manual_seed(3))
    for start in (h0, None):
        y = out_like(kind, g)
        s_out = torch.empty(shp, dtype=torch.float32, device="cuda")
        lrscan.step(desc, g, y, s_out, None if start is None else start.cuda())
        torch.cuda.synchronize()
        assert lrscan.last_dispatch() == kind + "_step"
        ry, rh = oracle_run(kind, api_inputs(kind, inp), disc, None if start is None else to64(start))
        assert_close("y", y, ry, tol)
        assert_close("state", s_out, rh, tol)


@pytest.mark.parametrize("kind", ["s6", "ssd"])
def test_step_softplus_front_end(kind):
    """lr_step with dt = softplus(delta + bias)."""
    shape = dict(B=2, L=5, D=32, N=16) if kind == "s6" else dict(B=2, L=5, H=4, P=16, N=32, G=2)
    inp = make_inputs(kind, shape, "f32", seed=13)
    gen = torch.Generator().manual_seed(8)
    inp["delta"] = torch.randn(inp["delta"].shape, generator=gen) - 1.0
    inp["delta_bias"] = 0.5 * torch.randn(shape["D"] if kind == "s6" else shape["H"], generator=gen)
    g = gpu_inputs(api_inputs(kind, inp))
    desc = lrscan.desc_for(kind, g, 1, "zoh", delta_softplus=True)
    shp = lrscan.state_shape(desc)
    y = out_like(kind, g)
    s_out = torch.empty(shp, dtype=torch.float32, device="cuda")
    lrscan.step(desc, g, y, s_out)
    torch.cuda.synchronize()
    ai = api_inputs(kind, inp)
    if kind == "s6":
        ry, rh = oracle.s6_fwd(ai["x"], ai["delta"], ai["A"], ai["Bm"], ai["Cm"], ai.get("Dskip"), ai.get("z"),
                               disc="zoh", final=True, delta_softplus=True, delta_bias=ai["delta_bias"])
    else:
        ry, rh = oracle.ssd_fwd(ai["x"], ai["delta"], ai["A"], ai["Bm"], ai["Cm"], ai.get("Dskip"), ai.get("z"),
                                disc="zoh", final=True, delta_softplus=True, delta_bias=ai["delta_bias"])
        rh = np.swapaxes(rh, 2, 3)
    assert_close("y", y, ry, TOL[torch.float32])
    assert_close("state", s_out, rh, TOL[torch.float32])


def test_step_rglru_gates():
    """lr_step with the RG-LRU gate front-end: parity with the oracle's gate composition from a
    random initial state, and the CUDA-graph decode loop equal to the one-call result bitwise."""
    inp = inputs.rglru_gated(2, 9, 40, seed=21)
    g = gpu_inputs(api_inputs("rglru", inp))
    desc = lrscan.desc_for("rglru", g, 1, gates=True)
    shp = lrscan.state_shape(desc)
    h0 = torch.randn(shp, dtype=torch.float32, generator=torch.Generator().manual_seed(5))
    y = torch.empty_like(g["b"])
    s_out = torch.empty(shp, dtype=torch.float32, device="cuda")
    lrscan.step(desc, g, y, s_out, h0.cuda())
    torch.cuda.synchronize()
    assert lrscan.last_dispatch() == "rglru_gated_step"
    ry, rh = oracle.rglru_gated_fwd(inp["a"], inp["b"], inp["x"], inp["A"], h0=to64(h0), final=True)
    assert_close("y", y, ry, TOL[torch.float32])
    assert_close("state", s_out, rh, TOL[torch.float32])
    toks = lrscan.TOKEN_INPUTS["rglru"]
    seq = {n: (v.transpose(0, 1).unsqueeze(2).contiguous() if n in toks else v) for n, v in g.items()}
    yg = torch.empty((9, 2, 1, 40), dtype=torch.float32, device="cuda")
    sg = h0.cuda()
    lrscan.DecodeGraph("rglru", seq, sg, yg, gates=True).replay()
    torch.cuda.synchronize()
    assert torch.equal(yg.squeeze(2).transpose(0, 1), y) and torch.equal(sg, s_out)


@pytest.mark.parametrize("kind,shape,io,disc", CASES[::2])
def test_step_modes_bitwise(kind, shape, io, disc):
    """One call of L steps == L one-step calls (state in place) == the CUDA-graph decode loop."""
    inp = make_inputs(kind, dict(shape, L=6), io, seed=11)
    g = gpu_inputs(api_inputs(kind, inp))
    desc = lrscan.desc_for(kind, g, 1, disc)
    shp = lrscan.state_shape(desc)
    h0 = torch.randn(shp, dtype=torch.float32, device="cuda")
    toks = lrscan.TOKEN_INPUTS[kind]
    y_all = out_like(kind, g)
    s_all = torch.empty_like(h0)
    lrscan.step(desc, g, y_all, s_all, h0)
    # one step at a time, in place
    s = h0.clone()
    ys = []
    for t in range(6):
        gt = {n: (v[:, t:t + 1].contiguous() if n in toks and v is not None else v) for n, v in g.items()}
        dt = lrscan.desc_for(kind, gt, 1, disc)
        yt = out_like(kind, gt)
        lrscan.step(dt, gt, yt, s, s)
        ys.append(yt)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys, dim=1), y_all) and torch.equal(s, s_all)
    # the same steps from a CUDA graph, time-major token buffers
    seq = {n: (v.transpose(0, 1).unsqueeze(2).contiguous() if n in toks and v is not None else v)
           for n, v in g.items()}
    yg = torch.empty((6,) + tuple(ys[0].shape), dtype=y_all.dtype, device="cuda")
    sg = h0.clone()
    graph = lrscan.DecodeGraph(kind, seq, sg, yg, disc)
    assert torch.equal(sg, h0)  # building the graph leaves the state alone
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg.squeeze(2).transpose(0, 1), y_all) and torch.equal(sg, s_all)


def test_ssd_decode_full_workload():
    """P7 at the SSD workload's size: decoding all 4096 tokens one at a time from a CUDA graph
    matches the chunked scan (outputs) and the oracle (outputs and final state, on 2 heads of
    one batch row; heads are independent given the shared B, C)."""
    inp = inputs.workload("ssd")
    w = inputs.WORKLOADS["ssd"]
    g = gpu_inputs(api_inputs("ssd", inp))
    plan = lrscan.plan_for("ssd", g, w["segment"], "zoh", w["chunk"])
    y_scan = torch.empty_like(g["x"])
    plan.fwd(g, y_scan)
    toks = lrscan.TOKEN_INPUTS["ssd"]
    seq = {n: (v.transpose(0, 1).unsqueeze(2).contiguous() if n in toks and v is not None else v)
           for n, v in g.items()}
    L = g["x"].shape[1]
    desc = lrscan.desc_for("ssd", g, 1, "zoh")
    state = torch.zeros(lrscan.state_shape(desc), dtype=torch.float32, device="cuda")
    yd = torch.empty((L,) + (g["x"].shape[0], 1) + tuple(g["x"].shape[2:]), dtype=g["x"].dtype, device="cuda")
    graph = lrscan.DecodeGraph("ssd", seq, state, yd, "zoh")
    graph.replay()
    torch.cuda.synchronize()
    y_dec = yd.squeeze(2).transpose(0, 1)
    tol = TOL[torch.bfloat16]
    assert_close("y (decode vs scan)", y_dec, to64(y_scan), tol)
    hs = slice(5, 7)
    sub = {"x": inp["x"][:1, :, hs], "delta": inp["delta"][:1, :, hs], "A": inp["A"][hs], "Bm": inp["Bm"][:1],
           "Cm": inp["Cm"][:1], "Dskip": inp["Dskip"][hs]}
    ry, rh = oracle.ssd_fwd(sub["x"], sub["delta"], sub["A"], sub["Bm"], sub["Cm"], sub["Dskip"], None,
                            disc="zoh", final=True)
    assert_close("y (decode vs oracle)", y_dec[:1, :, hs], ry, tol)
    assert_close("final state", state[:1, hs], np.swapaxes(rh, 2, 3), tol)
