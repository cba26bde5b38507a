"""GPU parity of the diagonal kinds (rglru_scan, rotlru_scan) against the fp64 oracle.

Cases span several tiles and ragged tails in time (L not a multiple of the segment) and in
channels (D not a multiple of the 32-channel tile), the degenerate L = 1 / S = 1 / L < S cases,
bf16 I/O, rows of up to 8 segment tiles (one thread-block cluster) and longer rows (the global
look-back), the rglru workload at full size and the long-sequence rotlru workload at full size on
sampled units.  Tolerance: max|err| <= 1e-5 max|ref| for fp32 I/O, 2e-2 for bf16, per tensor
(y, checkpoints and every gradient).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, assert_close, gpu_inputs, run_gpu, to64
from selective_state_space_09_b200 import inputs

pytestmark = pytest.mark.gpu

RGLRU_CASES = [
    # B, L, D, S, io
    (1, 1024, 256, 128, "f32"),     # the rglru workload itself
    (2, 1000, 96, 64, "f32"),       # ragged L, 3 channel blocks
    (3, 37, 40, 8, "f32"),          # ragged channels (40 = 32 + 8)
    (1, 1, 32, 1, "f32"),           # single step
    (2, 5, 64, 16, "f32"),          # L < S
    (1, 700, 64, 256, "f32"),       # maximum segment
    (2, 300, 128, 100, "bf16"),
    (1, 129, 8, 1, "f32"),          # S = 1: a checkpoint every step
    (2, 1024, 64, 128, "bf16"),     # rows of 8 tiles: the largest cluster
    (1, 1025, 64, 128, "f32"),      # rows of 9 tiles (ragged): the look-back, just past the clusters
]


@pytest.mark.parametrize("B,L,D,S,io", RGLRU_CASES)
def test_rglru_parity(B, L, D, S, io):
    inp = inputs.rglru(B, L, D, seed=B * 1000 + L, io=io)
    y, ck, gr, plan, disp = run_gpu("rglru", inp, S)
    tol = TOL[inp["a"].dtype]
    ry, rck = oracle.rglru_fwd(inp["a"], inp["b"], S=S)
    rg = oracle.rglru_bwd(inp["a"], inp["b"], inp["dy"])
    assert_close("y", y, ry, tol)
    assert_close("ckpt", ck, rck, max(tol, 1e-5))
    assert_close("da", gr["da"], rg["a"], tol)
    assert_close("db", gr["db"], rg["b"], tol)
    assert disp == ("diag_ws_zero+rglru_fwd_tile", "diag_ws_zero+rglru_bwd_tile")
    assert plan.device_error() == (0, 0)


GATED_CASES = [
    # B, L, D, S
    (1, 1024, 256, 128),    # the rglru workload's shapes
    (2, 1000, 96, 64),      # ragged L, 3 channel blocks
    (3, 37, 40, 8),         # ragged channels
    (1, 1, 32, 1),          # single step
    (1, 700, 64, 256),      # maximum segment
]


@pytest.mark.parametrize("B,L,D,S", GATED_CASES)
def test_rglru_gated_parity(B, L, D, S):
    """The RG-LRU gate front-end formed in the kernels (LR_RGLRU_GATES) against the oracle's gate
    composition: y, checkpoints, dr, di, dx and dLambda."""
    inp = inputs.rglru_gated(B, L, D, seed=B * 100 + L)
    y, ck, gr, plan, disp = run_gpu("rglru", inp, S, gates=True)
    tol = TOL[torch.float32]
    r, i, x, lam = inp["a"], inp["b"], inp["x"], inp["A"]
    ry, rck = oracle.rglru_gated_fwd(r, i, x, lam, S=S)
    rg = oracle.rglru_gated_bwd(r, i, x, lam, inp["dy"])
    assert_close("y", y, ry, tol)
    assert_close("ckpt", ck, rck, tol)
    assert_close("dr", gr["da"], rg["r"], tol)
    assert_close("di", gr["db"], rg["i"], tol)
    assert_close("dx", gr["dx"], rg["x"], tol)
    assert_close("dLambda", gr["dA"], rg["lam"], tol)
    assert disp == ("diag_ws_zero+rglru_gated_fwd_tile", "diag_ws_zero+rglru_gated_bwd_tile+rglru_param_reduce")
    assert plan.device_error() == (0, 0)


def test_rglru_gated_edge_gates():
    """Gates at the ends of their range: r near 0 (a -> 1, where sqrt(1 - a^2) is formed from
    expm1 to keep its relative precision) and near 1, i = 0 and 1 exactly, Lambda large."""
    B, L, D, S = 2, 200, 64, 32
    inp = inputs.rglru_gated(B, L, D, seed=77)
    gen = torch.Generator().manual_seed(4)
    u = torch.rand(B, L, D, generator=gen)
    inp["a"] = torch.where(u < 0.3, torch.full_like(u, 1e-3), torch.where(u > 0.7, torch.full_like(u, 0.999), inp["a"]))
    inp["b"] = torch.where(u < 0.1, torch.zeros_like(u), torch.where(u > 0.9, torch.ones_like(u), inp["b"]))
    inp["A"][: D // 2] = 9.0
    y, ck, gr, plan, _ = run_gpu("rglru", inp, S, gates=True)
    ry = oracle.rglru_gated_fwd(inp["a"], inp["b"], inp["x"], inp["A"])
    rg = oracle.rglru_gated_bwd(inp["a"], inp["b"], inp["x"], inp["A"], inp["dy"])
    tol = TOL[torch.float32]
    assert_close("y", y, ry, tol)
    for k, rk in (("da", "r"), ("db", "i"), ("dx", "x"), ("dA", "lam")):
        assert_close(k, gr[k], rg[rk], tol)


def test_rglru_gated_autograd_and_optional_dlambda():
    """lrscan.rglru_gated under torch autograd gives the ABI's gradients; a NULL dA skips the
    Lambda reduction and leaves the other gradients unchanged."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.rglru_gated(2, 300, 96, seed=9)
    y, ck, gr, plan, _ = run_gpu("rglru", inp, 64, gates=True)
    t = {k: v.cuda().requires_grad_(k != "dy") for k, v in inp.items()}
    yy = lrscan.rglru_gated(t["a"], t["b"], t["x"], t["A"], segment=64)
    yy.backward(t["dy"])
    assert torch.equal(yy.detach(), y)
    for k, gk in (("a", "da"), ("b", "db"), ("x", "dx"), ("A", "dA")):
        assert torch.equal(t[k].grad, gr[gk]), k
    g = gpu_inputs({k: v for k, v in inp.items() if k != "dy"})
    desc = lrscan.desc_for("rglru", g, 64, gates=True)
    p2 = lrscan.Plan(desc)
    y2, g2 = lrscan.alloc_outputs("rglru", g)
    p2.fwd(g, y2)
    del g2["dA"]
    p2.bwd(g, inp["dy"].cuda(), g2)
    torch.cuda.synchronize()
    assert lrscan.last_dispatch() == "diag_ws_zero+rglru_gated_bwd_tile"
    for k in ("da", "db", "dx"):
        assert torch.equal(g2[k], gr[k]), k


ROTLRU_CASES = [
    (2, 1000, 64, 64, "f32"),
    (1, 333, 40, 256, "f32"),       # 20 pairs: ragged pair block
    (3, 17, 8, 4, "f32"),
    (2, 600, 64, 128, "bf16"),
    (1, 1, 32, 1, "f32"),
]


@pytest.mark.parametrize("B,L,D,S,io", ROTLRU_CASES)
def test_rotlru_parity(B, L, D, S, io):
    inp = inputs.rotlru(B, L, D, seed=B * 1000 + L, io=io)
    y, ck, gr, plan, disp = run_gpu("rotlru", inp, S)
    tol = TOL[inp["b"].dtype]
    ry, rck = oracle.rotlru_fwd(inp["b"], inp["g"], inp["mag"], inp["theta"], S=S)
    rg = oracle.rotlru_bwd(inp["b"], inp["g"], inp["mag"], inp["theta"], inp["dy"])
    assert_close("y", y, ry, tol)
    assert_close("ckpt", ck, rck, max(tol, 1e-5))
    assert_close("db", gr["db"], rg["b"], tol)
    assert_close("dg", gr["dg"], rg["g"], tol)
    assert_close("dmag", gr["dmag"], rg["mag"], max(tol, 1e-5))
    assert_close("dtheta", gr["dtheta"], rg["theta"], max(tol, 1e-5))
    assert disp == ("diag_ws_zero+rotlru_fwd_tile", "diag_ws_zero+rotlru_bwd_tile+rotlru_param_reduce")
    assert plan.device_error() == (0, 0)


def test_diag_deterministic():
    """Two runs give bitwise-identical outputs (no order-dependent reductions, no races)."""
    inp = inputs.rotlru(2, 777, 96, seed=5)
    a = run_gpu("rotlru", inp, 64)
    b = run_gpu("rotlru", inp, 64)
    for k in ("db", "dg", "dmag", "dtheta"):
        assert torch.equal(a[2][k], b[2][k]), k
    assert torch.equal(a[0], b[0])


def test_withheld_carry_times_out_and_context_survives():
    """Failure path: tiles of the first segment withhold their carry; later tiles wait out
    their bound, record LR_ERR_TIMEOUT (status 6) and finish.  A normal call afterwards on the
    same context is correct."""
    from selective_state_space_09_b200 import lrscan
    inp = inputs.rglru(1, 256, 32, seed=3)
    y, ck, gr, plan, _ = run_gpu("rglru", inp, 64, flags=0x80000000)
    status, info = plan.device_error()
    assert status == 6 and info in (101, 201)
    y, ck, gr, plan, _ = run_gpu("rglru", inp, 64)
    assert plan.device_error() == (0, 0)
    assert_close("y", y, oracle.rglru_fwd(inp["a"], inp["b"]), 1e-5)


@pytest.mark.slow
def test_rotlru_full_size_sampled():
    """The long-sequence rotlru workload (B=16, D=4096, L=16384, S=256) on the GPU; the oracle
    recomputes sampled pairs (all batch rows of a pair, so the parameter gradients, which sum
    over batch and time, are checked too)."""
    w = inputs.WORKLOADS["rotlru"]
    inp = inputs.rotlru(w["B"], w["L"], w["D"], seed=0, device="cuda")
    y, ck, gr, plan, _ = run_gpu("rotlru", inp, w["segment"])
    assert plan.device_error() == (0, 0)
    rng = np.random.default_rng(0)
    pairs = sorted(set([0, w["D"] // 2 - 1] + list(rng.integers(0, w["D"] // 2, size=4))))
    oracle.set_threads(8)
    for k in pairs:
        sl = slice(2 * k, 2 * k + 2)
        b = to64(inp["b"][:, :, sl])
        g = to64(inp["g"][:, :, k:k + 1])
        mag, th = to64(inp["mag"][k:k + 1]), to64(inp["theta"][k:k + 1])
        dy = to64(inp["dy"][:, :, sl])
        ry, rck = oracle.rotlru_fwd(b, g, mag, th, S=w["segment"])
        rg = oracle.rotlru_bwd(b, g, mag, th, dy)
        assert_close("y[%d]" % k, y[:, :, sl], ry, 1e-5)
        assert_close("ckpt[%d]" % k, ck[:, :, sl], rck, 1e-5)
        assert_close("db[%d]" % k, gr["db"][:, :, sl], rg["b"], 1e-5)
        assert_close("dg[%d]" % k, gr["dg"][:, :, k:k + 1], rg["g"], 1e-5)
        assert_close("dmag[%d]" % k, gr["dmag"][k:k + 1], rg["mag"], 1e-5)
        assert_close("dtheta[%d]" % k, gr["dtheta"][k:k + 1], rg["theta"], 1e-5)


@pytest.mark.parametrize("kind,B,L,D,S,io", [("rglru", 2, 700, 96, 128, "f32"), ("rotlru", 2, 600, 64, 256, "f32"),
                                           ("rotlru", 1, 333, 64, 64, "bf16")])
def test_full_state_mode(kind, B, L, D, S, io):
    """LR_FULL_STATE: the checkpoint holds the state entering every step (the oracle's segment-1
    checkpoints) and the backward reads them.  Outputs equal the default mode's bitwise; the
    gradients agree to fp32 rounding (the default backward rebuilds each time group's entering
    state by folding group aggregates, while the full state stores the forward's sequential value
    of the same quantity) and match the oracle."""
    from selective_state_space_09_b200 import lrscan
    inp = (inputs.rglru if kind == "rglru" else inputs.rotlru)(B, L, D, seed=L, io=io)
    y0, _, g0, _, _ = run_gpu(kind, inp, S)
    y1, ck, g1, plan, disp = run_gpu(kind, inp, S, flags=lrscan.FULL_STATE)
    assert ck.shape[0] == L
    if kind == "rglru":
        _, rck = oracle.rglru_fwd(inp["a"], inp["b"], S=1)
    else:
        _, rck = oracle.rotlru_fwd(inp["b"], inp["g"], inp["mag"], inp["theta"], S=1)
    assert_close("full-state ckpt", ck, rck, max(TOL[inp["b"].dtype], 1e-5))
    assert torch.equal(y0, y1)
    tol = TOL[inp["b"].dtype]
    for k in g0:
        assert_close(k + " (full vs default)", g1[k], to64(g0[k]), 1e-6 if io == "f32" else tol)
    if kind == "rglru":
        rg = oracle.rglru_bwd(inp["a"], inp["b"], inp["dy"])
        pairs = (("da", "a"), ("db", "b"))
    else:
        rg = oracle.rotlru_bwd(inp["b"], inp["g"], inp["mag"], inp["theta"], inp["dy"])
        pairs = (("db", "b"), ("dg", "g"), ("dmag", "mag"), ("dtheta", "theta"))
    for k, r in pairs:
        assert_close(k, g1[k], rg[r], tol)
    assert plan.device_error() == (0, 0)


def test_entry_points_from_a_fresh_thread():
    """The entry points called from a thread that has made no CUDA call of its own (as a
    framework's backward worker may be): the tensor-map encoder, a driver call, needs the thread
    bound to the device's context, which the library does itself.  Results equal a call from the
    main thread bitwise."""
    import ctypes
    import threading
    from selective_state_space_09_b200 import lrscan
    inp = gpu_inputs(inputs.rglru(2, 300, 96, seed=5))
    dy = inp.pop("dy")
    desc = lrscan.desc_for("rglru", inp, 64)
    ref_plan = lrscan.Plan(desc)
    y_ref, g_ref = lrscan.alloc_outputs("rglru", inp)
    ref_plan.fwd(inp, y_ref)
    ref_plan.bwd(inp, dy, g_ref)
    torch.cuda.synchronize()
    plan = lrscan.Plan(desc)
    y, g = lrscan.alloc_outputs("rglru", inp)
    ii = lrscan.Inputs(*[lrscan._ptr(inp.get(n)) for n in lrscan._IN])
    gg = lrscan.Grads(*[lrscan._ptr(g.get(n)) for n in lrscan._GR])
    args = (ctypes.byref(desc), ctypes.byref(ii))
    status = []

    def work():  # the legacy default stream; no torch call on this thread
        status.append(lrscan.lib.lr_scan_fwd(*args, lrscan._ptr(y), lrscan._ptr(plan.ckpt), lrscan._ptr(plan.ws),
                                             plan.ws_bytes, None))
        status.append(lrscan.lib.lr_scan_bwd(*args, lrscan._ptr(dy), lrscan._ptr(plan.ckpt), ctypes.byref(gg),
                                             lrscan._ptr(plan.ws), plan.ws_bytes, None))

    th = threading.Thread(target=work)
    th.start()
    th.join()
    torch.cuda.synchronize()
    assert status == [0, 0]
    assert torch.equal(y, y_ref)
    for k in g_ref:
        assert torch.equal(g[k], g_ref[k]), k


@pytest.mark.parametrize("kind,B,L,D,S,io", [("rglru", 1, 1024, 256, 128, "f32"), ("rglru", 3, 37, 40, 8, "f32"),
                                           ("rotlru", 2, 600, 64, 256, "f32"), ("rotlru", 1, 333, 64, 64, "bf16")])
def test_cluster_exchange_equals_lookback(kind, B, L, D, S, io):
    """Rows of 2 .. 8 segment tiles run as one thread-block cluster and exchange their aggregates
    through distributed shared memory; forced onto the look-back over global-memory records
    (LR_TEST_LOOKBACK), the same problem gives bitwise the same outputs, checkpoints and gradients
    (both fold the same aggregates in the same order)."""
    from selective_state_space_09_b200 import lrscan
    inp = (inputs.rglru if kind == "rglru" else inputs.rotlru)(B, L, D, seed=L + 7, io=io)
    y0, c0, g0, p0, _ = run_gpu(kind, inp, S)
    y1, c1, g1, p1, _ = run_gpu(kind, inp, S, flags=lrscan.TEST_LOOKBACK)
    assert p0.device_error() == (0, 0) and p1.device_error() == (0, 0)
    assert torch.equal(y0, y1) and torch.equal(c0, c1)
    for k in g0:
        assert torch.equal(g0[k], g1[k]), k
