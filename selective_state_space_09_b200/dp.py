"""Data-parallel plumbing of the scan: batch-row sharding and the sum of parameter gradients.

The scan's units (batch rows, channels, heads) are independent, so data parallelism needs no
exchange inside the scan.  Only the parameter gradients -- sums over batch and time of per-token
contributions -- must be summed across ranks (NCCL over NVLink on GPUs, gloo on CPU in tests).
"""
import torch
import torch.distributed as dist

# parameter gradients (names as in the C ABI's lr_grads) that sum over the batch
PARAM_GRADS = {"rglru": ("dA",), "rotlru": ("dmag", "dtheta"), "s6": ("dA", "dDskip", "ddelta_bias"),
               "ssd": ("dA", "dDskip", "ddelta_bias"), "gla": ()}
# per-token inputs (batch-major) of each kind; everything else is a parameter
TOKEN_INPUTS = {"rglru": ("a", "b", "x", "dy"), "rotlru": ("b", "g", "dy"),
                "s6": ("x", "delta", "Bm", "Cm", "z", "dy"), "ssd": ("x", "delta", "Bm", "Cm", "z", "dy"),
                "gla": ("q", "k", "v", "g", "dy")}


def shard(kind, inp, rank, world):
    """This rank's contiguous slice of the batch rows (parameters are replicated)."""
    out = {}
    for k, v in inp.items():
        if v is not None and k in TOKEN_INPUTS[kind]:
            B = v.shape[0]
            assert B % world == 0, "batch %d not divisible by %d ranks" % (B, world)
            n = B // world
            out[k] = v[rank * n:(rank + 1) * n]
        else:
            out[k] = v
    return out


def reduce_param_grads(kind, grads, group=None):
    """Sum this rank's parameter gradients over all ranks, in place."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return grads
    for name in PARAM_GRADS[kind]:
        t = grads.get(name)
        if t is not None:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return grads
