"""lrscan.StepGraph: one step's forward and backward calls captured in a CUDA graph and replayed
give bitwise the results of the same calls made eagerly, for every kind, and a replay after the
inputs change computes the step on the new inputs.  SSD's dB and dC sum the head blocks of a
group with reduction adds in arrival order, bitwise reproducible only with at most two blocks;
they are compared to 1e-5 of their scale."""
import pytest
import torch

from helpers import assert_close, gpu_inputs, to64
from selective_state_space_09_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = {  # case: (kind, input builder, segment, disc, chunk, gates)
    "rglru": ("rglru", lambda: inputs.rglru(2, 700, 96, seed=1), 128, "none", 0, False),
    "rglru_gated": ("rglru", lambda: inputs.rglru_gated(2, 300, 64, seed=2), 64, "none", 0, True),
    "rotlru": ("rotlru", lambda: inputs.rotlru(2, 600, 64, seed=3), 256, "none", 0, False),
    "s6": ("s6", lambda: inputs.s6(2, 200, 128, 16, seed=4), 64, "zoh", 0, False),
    "ssd": ("ssd", lambda: inputs.ssd(1, 512, 4, 64, 128, seed=5), 128, "zoh", 128, False),
    "gla": ("gla", lambda: inputs.gla(1, 384, 2, 128, 128, seed=6), 128, "none", 128, False),
}


def same(kind, k, a, b):
    if kind == "ssd" and k in ("dBm", "dCm"):
        assert_close(k, a, to64(b), 1e-5)
    else:
        assert torch.equal(a, b), k


@pytest.mark.parametrize("case", list(CASES))
def test_step_graph_replay_matches_eager(case):
    from selective_state_space_09_b200 import lrscan
    kind, build, seg, disc, chunk, gates = CASES[case]
    g = gpu_inputs(build())
    dy = g.pop("dy")
    plan = lrscan.plan_for(kind, g, seg, disc, chunk, gates=gates)
    y, grads = lrscan.alloc_outputs(kind, g)
    plan.fwd(g, y)
    plan.bwd(g, dy, grads)
    torch.cuda.synchronize()
    y_ref, g_ref = y.clone(), {k: v.clone() for k, v in grads.items()}
    sg = lrscan.StepGraph(plan, g, dy, y, grads)
    y.zero_()
    for v in grads.values():
        v.zero_()
    sg.replay()
    torch.cuda.synchronize()
    assert plan.device_error() == (0, 0)
    assert torch.equal(y, y_ref)
    for k in g_ref:
        same(kind, k, grads[k], g_ref[k])
    # new upstream gradient: the replay reads the buffer's current contents
    dy.mul_(-0.5)
    sg.replay()
    plan.bwd(g, dy, g_ref)
    torch.cuda.synchronize()
    for k in g_ref:
        same(kind, k, grads[k], g_ref[k])
