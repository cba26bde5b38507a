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


# case -> (kind, inputs, gradients by the oracle named as in the C ABI's lr_grads)
def _case_inputs(case):
    from selective_state_space_09_b200 import inputs
    if case == "rotlru":
        return inputs.rotlru(4, 40, 16, seed=3)
    if case == "rglru_gated":
        return inputs.rglru_gated(4, 30, 8, seed=2)
    inp = inputs.s6(4, 24, 16, 16, seed=4)
    inp["delta_bias"] = torch.linspace(-0.5, 0.5, 16)
    return inp


KIND = {"rotlru": "rotlru", "s6": "s6", "rglru_gated": "rglru"}


def _grads(case, inp):
    import oracle
    if case == "rotlru":
        g = oracle.rotlru_bwd(inp["b"], inp["g"], inp["mag"], inp["theta"], inp["dy"])
        return {"dmag": g["mag"], "dtheta": g["theta"], "db": g["b"]}
    if case == "rglru_gated":
        g = oracle.rglru_gated_bwd(inp["a"], inp["b"], inp["x"], inp["A"], inp["dy"])
        return {"dA": g["lam"], "dx": g["x"]}
    g = oracle.s6_bwd(inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"],
                      inp["dy"], disc="zoh", delta_softplus=True, delta_bias=inp["delta_bias"])
    return {"dA": g["A"], "dDskip": g["D"], "ddelta_bias": g["delta_bias"], "dx": g["x"]}


def _worker(rank, world, port, case, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from selective_state_space_09_b200 import dp, inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kind = KIND[case]
        inp = _case_inputs(case)
        mine = dp.shard(kind, inp, rank, world)
        g = {k: torch.from_numpy(v) for k, v in _grads(case, mine).items()}
        dp.reduce_param_grads(kind, g)
        q.put((rank, {k: v.numpy() for k, v in g.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["rotlru", "s6", "rglru_gated"])
def test_two_rank_gradient_sum_equals_full_batch(case):
    """rotlru (dmag, dtheta), S6 with the softplus front-end (dA, dD, dbias) and rglru with its
    gates (dLambda): every parameter gradient summed over the ranks equals the full batch's."""
    from selective_state_space_09_b200 import dp, inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    kind = KIND[case]
    full = _grads(case, _case_inputs(case))
    for name in dp.PARAM_GRADS[kind]:
        for r in range(2):
            np.testing.assert_allclose(res[r][name], full[name], rtol=1e-12, atol=1e-12)
    # per-token gradients stay per shard: rank r holds rows [2r, 2r+2)
    tok = "db" if kind == "rotlru" else "dx"
    assert set(dp.PARAM_GRADS[kind]) <= set(full)
    np.testing.assert_allclose(np.concatenate([res[0][tok], res[1][tok]]), full[tok], rtol=1e-12)


def test_shard_slices_token_inputs_only():
    from selective_state_space_09_b200 import dp, inputs
    inp = inputs.s6(4, 8, 16, 16, seed=1)
    s = dp.shard("s6", inp, 1, 2)
    assert s["x"].shape[0] == 2 and torch.equal(s["x"], inp["x"][2:4])
    assert s["A"] is inp["A"] and s["Dskip"] is inp["Dskip"]
