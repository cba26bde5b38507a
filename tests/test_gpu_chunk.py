"""GPU parity of the chunked-matmul kinds (SSD, GLA; tcgen05 tensor cores) against the fp64
oracle.  bf16 I/O, tolerance max|err| <= 2e-2 max|ref| per tensor.  Cases cover several chunks
chained through the look-back, a ragged last chunk (L not a multiple of 128), a single chunk,
several heads per group (SSD), and the workloads at full size on sampled heads."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, gpu_inputs, to64
from selective_state_space_09_b200 import inputs, lrscan

pytestmark = pytest.mark.gpu
TOL = 2e-2


def fwd_only(kind, inp, disc="none"):
    g = gpu_inputs(inp)
    g.pop("dy")
    g = {k: v for k, v in g.items() if v is not None}
    plan = lrscan.plan_for(kind, g, 128, disc, 128)
    y, _ = lrscan.alloc_outputs(kind, g)
    plan.fwd(g, y)
    disp = lrscan.last_dispatch()
    torch.cuda.synchronize()
    return y, plan.ckpt_view().clone(), plan, disp


SSD_CASES = [(1, 512, 4, 64, 1), (2, 300, 8, 64, 2), (1, 128, 2, 64, 1), (1, 77, 8, 64, 1)]


@pytest.mark.parametrize("B,L,H,P,G", SSD_CASES)
def test_ssd_forward(B, L, H, P, G):
    inp = inputs.ssd(B, L, H, P, 128, G=G, seed=B * 31 + L)
    y, ck, plan, disp = fwd_only("ssd", inp, "zoh")
    ry, rck = oracle.ssd_fwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"],
                             None, disc="zoh", S=128)
    assert_close("y", y, ry, TOL)
    assert_close("ckpt", ck.transpose(-1, -2), rck, TOL)   # kernel state [N, P], oracle [P, N]
    assert disp == "ssd_fwd_chunk"
    assert plan.device_error() == (0, 0)


GLA_CASES = [(1, 512, 2, 128), (2, 300, 3, 128), (1, 128, 1, 128), (2, 200, 2, 64)]


@pytest.mark.parametrize("B,L,H,V", GLA_CASES)
def test_gla_forward(B, L, H, V):
    inp = inputs.gla(B, L, H, 128, V, seed=B * 17 + L)
    y, ck, plan, disp = fwd_only("gla", inp)
    ry, rck = oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], S=128)
    assert_close("o", y, ry, TOL)
    assert_close("ckpt", ck, rck, TOL)
    assert disp == "gla_fwd_chunk"
    assert plan.device_error() == (0, 0)
