"""Expert parallelism across processes on CPU: two and four gloo ranks.

Each rank routes its own tokens (float64 oracle), the ranks gather every rank's expert
counts with an all-gather, each computes the exchange layout from them, and the token
rows travel to their experts' owners as point-to-point messages carrying (destination
row, row).  Owners run their experts (oracle) on the rows they received and send the
output rows back; sources combine them.  Checked: every owner's receive buffer equals
the oracle's expert-parallel layout and the single-device permutation of its experts'
rows, and every rank's output equals the single-device layer's on the concatenated
batch.  This is the data movement the CUDA kernels do through peer memory, with the
same layout rule, run with real process groups.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_offsets_b200.inputs import CONFIGS, make_inputs, shrink
from oracle import moe_ep_ref as ep
from oracle import moe_ref as ref

CFG = shrink(CONFIGS["tiny_f32"], name="ep_gloo", T=10, d_model=8, E=8, top_k=2, d_ff=8,
             router_std=0.4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange(rank, world, outgoing, width):
    """outgoing[o] = (rows [n], data [n, width]) for every rank o; returns what every rank
    sent here, as (rows, data) pairs in source order."""
    sizes = [torch.tensor([len(outgoing[o][0])], dtype=torch.int64) for o in range(world)]
    recv_sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    reqs = []
    for o in range(world):
        if o != rank:
            reqs.append(dist.isend(sizes[o], o))
            reqs.append(dist.irecv(recv_sizes[o], o))
    for r in reqs:
        r.wait()
    recv_sizes[rank] = sizes[rank]
    got = [None] * world
    reqs = []
    for o in range(world):
        if o == rank:
            got[o] = outgoing[o]
            continue
        rows, data = outgoing[o]
        reqs.append(dist.isend(torch.as_tensor(rows, dtype=torch.int64), o))
        reqs.append(dist.isend(torch.as_tensor(data, dtype=torch.float64).reshape(-1, width), o))
        n = int(recv_sizes[o])
        rr, rd = torch.zeros(n, dtype=torch.int64), torch.zeros(n, width, dtype=torch.float64)
        reqs.append(dist.irecv(rr, o))
        reqs.append(dist.irecv(rd, o))
        got[o] = (rr, rd)
    for r in reqs:
        r.wait()
    return [(np.asarray(r), np.asarray(d)) for r, d in got]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        E, El, k, d = CFG.E, CFG.E // world, CFG.top_k, CFG.d_model
        w = make_inputs(CFG, seed=100)
        mine = make_inputs(CFG, seed=rank)
        x = mine["x"].double().numpy()
        wr, w1, w2 = (w[key].double().numpy() for key in ("w_router", "w1", "w2"))
        r = ref.route(x, wr, k)
        counts = torch.from_numpy(r["counts"].astype(np.int64))
        gathered = [torch.zeros_like(counts) for _ in range(world)]
        dist.all_gather(gathered, counts)
        counts_all = torch.stack(gathered).numpy()
        rows = ep.ep_rows(r["idx"], counts_all, rank)
        own = ep.ep_owner(r["idx"], E, world)
        # dispatch: every selected row to its owner, with its row in the owner's buffer
        outgoing = []
        for o in range(world):
            sel = np.argwhere(own == o)
            outgoing.append((rows[sel[:, 0], sel[:, 1]], x[sel[:, 0]]))
        got = _exchange(rank, world, outgoing, d)
        roff = ep.ep_recv_offsets(counts_all, rank)
        x_recv = np.zeros((int(roff[-1]), d))
        for rr, data in got:
            x_recv[rr] = data
        # the owner's experts on its rows, then the output rows back to their sources
        _, _, _, y = ref.expert_ffn_fwd(x_recv, roff, w1[rank * El:(rank + 1) * El],
                                        w2[rank * El:(rank + 1) * El])
        back = []
        for s, (rr, _) in enumerate(got):
            back.append((rr, y[rr]))
        returned = _exchange(rank, world, back, d)
        ylocal = np.zeros((CFG.T * k, d))
        for o in range(world):
            sel = np.argwhere(own == o)
            # the owner returns this rank's rows in the order this rank sent them
            rr, data = returned[o]
            assert np.array_equal(rr, rows[sel[:, 0], sel[:, 1]])
            ylocal[sel[:, 0] * k + sel[:, 1]] = data
        slot = np.arange(CFG.T * k).reshape(CFG.T, k)
        out[rank] = (counts_all, x_recv, roff, ref.combine(ylocal, slot, r["gate"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_exchange_rows_by_the_expert_parallel_layout(world):
    res = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, _free_port(), res), nprocs=world, join=True,
                       start_method="spawn")
    w = make_inputs(CFG, seed=100)
    shards = [make_inputs(CFG, seed=s) for s in range(world)]
    xs = [s["x"].double().numpy() for s in shards]
    wr, w1, w2 = (w[key].double().numpy() for key in ("w_router", "w1", "w2"))
    full = ref.layer_fwd_bwd(np.concatenate(xs), wr, w1, w2,
                             np.concatenate([s["dout"].double().numpy() for s in shards]),
                             CFG.top_k)
    o = ep.ep_layer_fwd_bwd(xs, wr, w1, w2, [s["dout"].double().numpy() for s in shards],
                            CFG.top_k)
    El = CFG.E // world
    for r in range(world):
        counts_all, x_recv, roff, out = res[r]
        assert np.array_equal(counts_all, o["counts_all"])
        assert np.array_equal(roff, o["recv_offsets"][r])
        assert np.array_equal(x_recv, o["x_recv"][r])
        r0, r1 = full["offsets"][r * El], full["offsets"][(r + 1) * El]
        assert np.array_equal(x_recv, full["x_perm"][r0:r1])
        np.testing.assert_allclose(out, full["out"][r * CFG.T:(r + 1) * CFG.T], rtol=1e-12,
                                   atol=1e-14)
