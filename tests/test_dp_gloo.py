"""Two-rank data-parallel path on CPU (gloo): each rank takes its shard of the batch, computes its
gradients (here with the oracle; on GPUs the C ABI computes them), and the parameter gradients are
summed with selective_state_space_09_b200.dp.  The result must equal the full-batch gradients."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _grads(kind, inp):
    import oracle
    if kind == "rotlru":
        g = oracle.rotlru_bwd(inp["b"], inp["g"], inp["mag"], inp["theta"], inp["dy"])
        return {"dmag": g["mag"], "dtheta": g["theta"], "db": g["b"]}
    g = oracle.s6_bwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"],
                      inp["dy"], disc="zoh")
    return {"dA": g["A"], "dDskip": g["D"], "dx": g["x"]}


def _worker(rank, world, port, kind, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from selective_state_space_09_b200 import dp, inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = inputs.rotlru(4, 40, 16, seed=3) if kind == "rotlru" else inputs.s6(4, 24, 16, 16, seed=4)
        mine = dp.shard(kind, inp, rank, world)
        g = {k: torch.from_numpy(v) for k, v in _grads(kind, mine).items()}
        dp.reduce_param_grads(kind, g)
        q.put((rank, {k: v.numpy() for k, v in g.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["rotlru", "s6"])
def test_two_rank_gradient_sum_equals_full_batch(kind):
    from selective_state_space_09_b200 import dp, inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, kind, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = inputs.rotlru(4, 40, 16, seed=3) if kind == "rotlru" else inputs.s6(4, 24, 16, 16, seed=4)
    full = _grads(kind, inp)
    for name in dp.PARAM_GRADS[kind]:
        for r in range(2):
            np.testing.assert_allclose(res[r][name], full[name], rtol=1e-12, atol=1e-12)
    # per-token gradients stay per shard: rank r holds rows [2r, 2r+2)
    tok = "db" if kind == "rotlru" else "dx"
    np.testing.assert_allclose(np.concatenate([res[0][tok], res[1][tok]]), full[tok], rtol=1e-12)


def test_shard_slices_token_inputs_only():
    from selective_state_space_09_b200 import dp, inputs
    inp = inputs.s6(4, 8, 16, 16, seed=1)
    s = dp.shard("s6", inp, 1, 2)
    assert s["x"].shape[0] == 2 and torch.equal(s["x"], inp["x"][2:4])
    assert s["A"] is inp["A"] and s["Dskip"] is inp["Dskip"]
