"""Expert parallelism on one GPU: N ranks emulated in one process, each with its own
tokens and its own receive buffers, the "peer" pointers being the other emulated ranks'
buffers on the same device.  The phases run rank by rank with the device in program
order between them, so no kernel ever waits for another (the real multi-GPU run puts a
collective between the phases instead); the counts all-gather is a stack of the ranks'
count vectors, the router-gradient all-reduce a sum.

Checked against (a) the single-device layer (MoELayer) on the ranks' concatenated
batches, which the expert-parallel layout reproduces row for row: outputs, gate
gradients, the owners' expert outputs and their experts' weight gradients bit for bit,
input gradients and the summed router gradient within the bf16 tolerance; and (b) the
float64 expert-parallel oracle (oracle/moe_ep_ref.py), whose receive layout and row map
must match bit for bit.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import f64, i64, rel
from mixture_experts_layer_offsets_b200 import inputs
from mixture_experts_layer_offsets_b200.ep import EPLayer
from mixture_experts_layer_offsets_b200.layer import MoELayer
from oracle import moe_ep_ref as ep

pytestmark = pytest.mark.gpu

BASE = inputs.CONFIGS["bf16_e8"]
CASES = {
    "n2_e8": (inputs.shrink(BASE, name="n2_e8", T=300, d_model=256, E=8, top_k=4, d_ff=256), 2),
    # a logit bias that dominates the router: a few experts take every token, so some
    # owners receive nothing and some ranks send nothing to some owners
    "n4_e16_skew": (inputs.shrink(BASE, name="n4_e16_skew", T=200, d_model=256, E=16, top_k=2,
                                  d_ff=256, router_std=0.01, bias_std=4.0), 4),
    "n4_e128": (inputs.shrink(BASE, name="n4_e128", T=256, d_model=256, E=128, top_k=4,
                              d_ff=256), 4),
}


def _run_ep(cfg, N, ws_inp, shards):
    dev = "cuda"
    bufs = {}

    def shared_for(rank):
        # the n-th shared buffer of every rank, created on first use
        counter = {"i": 0}

        def shared(shape, dtype):
            i = counter["i"]
            counter["i"] += 1
            if i not in bufs:
                bufs[i] = [torch.zeros(*shape, dtype=dtype, device=dev) for _ in range(N)]
            return bufs[i][rank], [b.data_ptr() for b in bufs[i]]
        return shared

    layers = [EPLayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, dev, N, r,
                      shared_for(r)) for r in range(N)]
    El = cfg.E // N
    w1 = [ws_inp["w1"][r * El:(r + 1) * El].contiguous() for r in range(N)]
    w2 = [ws_inp["w2"][r * El:(r + 1) * El].contiguous() for r in range(N)]
    wr, bias = ws_inp["w_router"], ws_inp["bias"]
    for r, L in enumerate(layers):
        L.route(shards[r]["x"], wr, bias)
    counts_all = torch.stack([L.counts for L in layers])          # the all-gather
    for r, L in enumerate(layers):
        L.counts_all.copy_(counts_all)
        L.dispatch(shards[r]["x"])
    for r, L in enumerate(layers):
        L.expert_fwd(w1[r], w2[r])
    for r, L in enumerate(layers):
        L.combine_and_grad(shards[r]["dout"])
    for r, L in enumerate(layers):
        L.expert_bwd(w1[r], w2[r])
    for r, L in enumerate(layers):
        L.router_bwd(shards[r]["x"], wr)
    torch.cuda.synchronize()
    dwr = sum(L.dw_router for L in layers)                        # the all-reduce
    return layers, dwr


@pytest.mark.parametrize("name", list(CASES))
def test_expert_parallel_ranks_reproduce_the_single_device_layer(name):
    cfg, N = CASES[name]
    wcpu = inputs.make_inputs(cfg, device="cpu", seed=100)
    scpu = [inputs.make_inputs(cfg, device="cpu", seed=s) for s in range(N)]
    ws_inp = {k: (v.cuda() if v is not None else None) for k, v in wcpu.items()}
    shards = [{k: (v.cuda() if v is not None else None) for k, v in s.items()} for s in scpu]
    layers, dwr = _run_ep(cfg, N, ws_inp, shards)
    # single device, concatenated batch
    T, E, El = cfg.T, cfg.E, cfg.E // N
    x = torch.cat([s["x"] for s in shards])
    dout = torch.cat([s["dout"] for s in shards])
    S = MoELayer(T * N, cfg.d_model, E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda")
    S.step(x, ws_inp["w_router"], ws_inp["bias"], ws_inp["w1"], ws_inp["w2"], dout)
    torch.cuda.synchronize()
    assert S.device_status() == 0
    for r, L in enumerate(layers):
        sl = slice(r * T, (r + 1) * T)
        assert L.ws[:4].view(torch.int32).item() == 0
        assert torch.equal(L.topk_idx, S.topk_idx[sl])
        assert torch.equal(L.out, S.out[sl]), r
        assert torch.equal(L.dgate, S.dgate[sl]), r
        assert rel(f64(L.dx), f64(S.dx[sl])) <= 1e-2
        # the owner's rows and its experts' gradients
        e0, e1 = r * El, (r + 1) * El
        o0, o1 = int(S.offsets[e0]), int(S.offsets[e1])
        assert torch.equal(L.recv_offsets.long(), (S.offsets[e0:e1 + 1] - o0).long())
        n = o1 - o0
        assert torch.equal(L.x_recv[:n], S.x_perm[o0:o1])
        assert torch.equal(L.y_recv[:n], S.y_perm[o0:o1])
        assert torch.equal(L.dx_recv[:n], S.dx_perm[o0:o1])
        assert torch.equal(L.dw1, S.dw1[e0:e1]), r
        assert torch.equal(L.dw2, S.dw2[e0:e1]), r
    assert rel(f64(dwr), f64(S.dw_router)) <= 1e-2
    # the float64 oracle's layout and row map, on the device's own routing
    ca = np.stack([i64(L.counts) for L in layers])
    for r, L in enumerate(layers):
        assert np.array_equal(i64(L.counts_all), ca)
        assert np.array_equal(i64(L.recv_offsets), ep.ep_recv_offsets(ca, r))
        assert np.array_equal(i64(L.send_base), ep.ep_send_base(ca, r))
        assert np.array_equal(i64(L.ep_row), ep.ep_rows(i64(L.topk_idx), ca, r))
    if name == "n4_e16_skew":
        sent = np.stack([ca[:, o * El:(o + 1) * El].sum(axis=1) for o in range(N)], axis=1)
        assert (sent == 0).any(), "some rank must send nothing to some owner"


def test_expert_parallel_ranks_match_the_oracle():
    """Values against the float64 expert-parallel oracle (its routing taken on the
    device's logits)."""
    cfg, N = CASES["n2_e8"]
    wcpu = inputs.make_inputs(cfg, device="cpu", seed=100)
    scpu = [inputs.make_inputs(cfg, device="cpu", seed=s) for s in range(N)]
    ws_inp = {k: (v.cuda() if v is not None else None) for k, v in wcpu.items()}
    shards = [{k: (v.cuda() if v is not None else None) for k, v in s.items()} for s in scpu]
    layers, dwr = _run_ep(cfg, N, ws_inp, shards)
    o = ep.ep_layer_fwd_bwd([f64(s["x"]) for s in scpu], f64(wcpu["w_router"]), f64(wcpu["w1"]),
                            f64(wcpu["w2"]), [f64(s["dout"]) for s in scpu], cfg.top_k,
                            select_logits=[f64(L.logits) for L in layers])
    for r, L in enumerate(layers):
        assert np.array_equal(i64(L.topk_idx), o["idx"][r])
        for key, dev in (("out", L.out), ("dgate", L.dgate), ("dx", L.dx)):
            assert rel(f64(dev), o[key][r]) <= 1e-2, (r, key)
        assert rel(f64(L.dw1), o["dw1"][r]) <= 1e-2
        assert rel(f64(L.dw2), o["dw2"][r]) <= 1e-2
    assert rel(f64(dwr), o["dw_router"]) <= 1e-2
