"""Multi-rank host logic on CPU: two gloo ranks, world size 2.

Each rank draws its own images (the data-parallel shard) with the shared
theta, computes its d theta (here with the fp64 oracle, standing in for the
GPU kernels), and the ranks sum it with the path's one collective.  The sum
must equal d theta of the two shards as one batch: d theta is a sum over
images, so splitting the batch over ranks must not change it.  The job time is
the maximum over ranks.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from vision_transformer_windowed_b200 import dp

SHAPE = dict(B=1, H=16, W=16, heads=2, d=32)
M, S = 8, 4


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank: int, world: int, port: int, out: str):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], rank, "cpu")
        ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, S, dout=inp["dout"], nthreads=1)
        dth = torch.from_numpy(np.ascontiguousarray(ref["dtheta"]))
        dp.allreduce_dtheta(dth)
        t = dp.max_over_ranks(float(rank + 1) * 1.5, "cpu")
        if rank == 0:
            torch.save({"dtheta": dth, "t": t}, out)
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_dtheta_and_take_the_slowest_time(tmp_path):
    out = str(tmp_path / "rank0.pt")
    mp.spawn(_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    res = torch.load(out)
    a = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], 0, "cpu")
    b = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], 1, "cpu")
    assert not torch.equal(a["q"], b["q"]) and torch.equal(a["theta"], b["theta"])
    cat = {k: torch.cat([a[k], b[k]]) for k in ("q", "k", "v", "dout")}
    whole = oracle.full(cat["q"], cat["k"], cat["v"], a["theta"], M, S, dout=cat["dout"], nthreads=1)
    np.testing.assert_allclose(res["dtheta"].numpy(), whole["dtheta"], rtol=1e-10, atol=1e-12)
    assert res["t"] == 3.0


def test_single_process_helpers_are_identities():
    x = torch.arange(4.0)
    assert torch.equal(dp.allreduce_dtheta(x.clone()), x)
    assert dp.max_over_ranks(2.5, "cpu") == 2.5


def _bias_worker(rank: int, world: int, port: int, out: str):
    from vision_transformer_windowed_b200.inputs import make_bias
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], rank, "cpu")
        bias = make_bias(SHAPE["heads"], M)
        ref = oracle.full(inp["q"], inp["k"], inp["v"], inp["theta"], M, S, dout=inp["dout"], nthreads=1,
                          bias=(bias["u"], bias["w"]))
        grads = [torch.from_numpy(np.ascontiguousarray(ref[k])) for k in ("dtheta", "du", "dw")]
        dp.allreduce_param_grads(*grads)
        if rank == 0:
            torch.save(dict(zip(("dtheta", "du", "dw"), grads)), out)
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_the_bias_factor_gradients(tmp_path):
    """With the low-rank bias the factors U, W are shared by the batch like theta:
    the ranks' summed dU, dW equal those of the two shards as one batch."""
    from vision_transformer_windowed_b200.inputs import make_bias
    out = str(tmp_path / "rank0_bias.pt")
    mp.spawn(_bias_worker, args=(2, _free_port(), out), nprocs=2, join=True)
    res = torch.load(out)
    a = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], 0, "cpu")
    b = dp.rank_inputs(SHAPE["B"], SHAPE["H"], SHAPE["W"], SHAPE["heads"], SHAPE["d"], 1, "cpu")
    bias = make_bias(SHAPE["heads"], M)
    cat = {k: torch.cat([a[k], b[k]]) for k in ("q", "k", "v", "dout")}
    whole = oracle.full(cat["q"], cat["k"], cat["v"], a["theta"], M, S, dout=cat["dout"], nthreads=1,
                        bias=(bias["u"], bias["w"]))
    for key in ("dtheta", "du", "dw"):
        np.testing.assert_allclose(res[key].numpy(), whole[key], rtol=1e-10, atol=1e-12)
