"""Shared test helpers: run the CUDA path through the C ABI and compare with the oracle."""
import numpy as np
import torch

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}


def to64(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def assert_close(name, got, ref, tol):
    """max |got - ref| <= tol * max |ref| (the tolerance rule of the parity bar)."""
    g, r = to64(got), np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (name, g.shape, r.shape)
    assert np.all(np.isfinite(g)), name + ": non-finite values"
    err = float(np.max(np.abs(g - r))) if r.size else 0.0
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    assert err <= tol * scale + 1e-30, "%s: max err %.3e > %.1e * max|ref| %.3e" % (name, err, tol, scale)
    return err / scale if scale else 0.0


def gpu_inputs(inp, device="cuda"):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in inp.items()}


def run_gpu(kind, inp, segment, disc="none", chunk=0, flags=0, gates=False):
    """Forward + backward through the C ABI on the current CUDA device.  Returns
    (y, ckpt view, grads dict, plan)."""
    from selective_state_space_09_b200 import lrscan
    g = gpu_inputs(inp)
    dy = g.pop("dy")
    desc = lrscan.desc_for(kind, g, segment, disc, chunk, gates=gates)
    desc.flags |= flags  # before the Plan sizes its buffers (LR_FULL_STATE changes the checkpoint)
    plan = lrscan.Plan(desc, "cuda")
    y, grads = lrscan.alloc_outputs(kind, g)
    plan.fwd(g, y)
    fwd_dispatch = lrscan.last_dispatch()
    plan.bwd(g, dy, grads)
    bwd_dispatch = lrscan.last_dispatch()
    torch.cuda.synchronize()
    return y, plan.ckpt_view().clone(), grads, plan, (fwd_dispatch, bwd_dispatch)
