"""The multi-process (N > 1) path on CPU: two gloo ranks, each with its own
token batch (seed = rank) and replicated weights.

Checks: (1) the summed weight gradients of the two ranks equal the oracle's
gradients of the concatenated batch (the data-parallel gradient all-reduce is
exact up to float64 rounding); (2) the reported step time is the maximum over
ranks; (3) each rank's inputs differ (weak scaling draws new tokens per rank).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_offsets_b200 import dist as mdist
from mixture_experts_layer_offsets_b200.inputs import CONFIGS, make_inputs, shrink
from oracle import moe_ref as ref

CFG = shrink(CONFIGS["tiny_f32"], name="gloo", T=24, d_model=16, E=4, top_k=2, d_ff=8,
             router_std=0.25)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _f64(t):
    return t.double().numpy()


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        weights = make_inputs(CFG, seed=0)          # replicated parameters
        mine = make_inputs(CFG, seed=mdist.rank_seed(0, rank))
        res = ref.layer_fwd_bwd(_f64(mine["x"]), _f64(weights["w_router"]), _f64(weights["w1"]),
                                _f64(weights["w2"]), _f64(mine["dout"]), CFG.top_k)
        grads = [torch.from_numpy(res[k].copy()) for k in ("dw1", "dw2", "dw_router")]
        mdist.allreduce_grads(grads)
        t = mdist.max_over_ranks(1.0 + rank)
        out[rank] = ([g.numpy() for g in grads], t, float(mine["x"][0, 0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_sum_gradients_and_take_max_time():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    weights = make_inputs(CFG, seed=0)
    shards = [make_inputs(CFG, seed=mdist.rank_seed(0, r)) for r in range(world)]
    x = np.concatenate([_f64(s["x"]) for s in shards])
    dout = np.concatenate([_f64(s["dout"]) for s in shards])
    full = ref.layer_fwd_bwd(x, _f64(weights["w_router"]), _f64(weights["w1"]), _f64(weights["w2"]),
                             dout, CFG.top_k)
    for r in range(world):
        grads, t, first = out[r]
        for g, key in zip(grads, ("dw1", "dw2", "dw_router")):
            np.testing.assert_allclose(g, full[key], rtol=1e-12, atol=1e-14, err_msg=key)
        assert t == 2.0
    assert out[0][2] != out[1][2]


def test_single_process_helpers_are_identities():
    assert mdist.max_over_ranks(3.5) == 3.5
    g = torch.ones(3)
    mdist.allreduce_grads([g])
    assert torch.equal(g, torch.ones(3))
