"""Data-parallel step through the CUDA path: two ranks (processes) each take half of the batch,
run the forward and backward pass through the C ABI, and sum their parameter gradients with
selective_state_space_09_b200.dp (gloo, on host copies).  The summed gradients must equal the
full batch's gradients from one CUDA call, and the per-token gradients must be the full batch's
rows.  Both ranks share one GPU here; their kernels never wait on each other (each call only
depends on its own stream), and the exchange runs on the host.  On several GPUs bench.py runs
the same step with NCCL, one rank per GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rotlru():
    from selective_state_space_09_b200 import inputs
    return inputs.rotlru(4, 300, 64, seed=3)


def _s6():
    from selective_state_space_09_b200 import inputs
    return inputs.s6(4, 128, 128, 16, seed=4)


def _ssd():
    from selective_state_space_09_b200 import inputs
    return inputs.ssd(2, 256, 8, 64, 128, seed=5)


CASES = {  # case: (kind, input builder, segment, disc, chunk)
    "rotlru": ("rotlru", _rotlru, 64, "none", 0),
    "s6": ("s6", _s6, 64, "zoh", 0),
    "ssd": ("ssd", _ssd, 128, "zoh", 128),
}


def _cuda_grads(case, inp):
    from selective_state_space_09_b200 import lrscan
    kind, _, seg, disc, chunk = CASES[case]
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    dy = g.pop("dy")
    plan = lrscan.plan_for(kind, g, seg, disc, chunk)
    y, grads = lrscan.alloc_outputs(kind, g)
    plan.fwd(g, y)
    plan.bwd(g, dy, grads)
    torch.cuda.synchronize()
    assert plan.device_error() == (0, 0)
    return grads


def _worker(rank, world, port, case, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from selective_state_space_09_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        kind = CASES[case][0]
        mine = dp.shard(kind, CASES[case][1](), rank, world)
        grads = {k: v.cpu() for k, v in _cuda_grads(case, mine).items()}
        dp.reduce_param_grads(kind, grads)
        q.put((rank, {k: v.float().numpy() for k, v in grads.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["rotlru", "s6", "ssd"])
def test_two_rank_cuda_gradients_sum_to_the_full_batch(case):
    from selective_state_space_09_b200 import dp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    kind = CASES[case][0]
    full = {k: v.float().cpu().numpy() for k, v in _cuda_grads(case, CASES[case][1]()).items()}
    for name in dp.PARAM_GRADS[kind]:
        if name not in full:
            continue
        scale = float(np.max(np.abs(full[name])))
        tol = 1e-5 if kind == "rotlru" else 2e-2
        for r in range(2):
            err = float(np.max(np.abs(res[r][name] - full[name])))
            assert err <= tol * scale, (name, r, err, scale)
    tok = "db" if kind == "rotlru" else "dx"
    both = np.concatenate([res[0][tok], res[1][tok]])
    assert np.max(np.abs(both - full[tok])) <= (1e-5 if kind == "rotlru" else 2e-2) * np.max(np.abs(full[tok]))
