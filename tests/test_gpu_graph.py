"""The whole layer step captures into a CUDA graph: no host synchronisation,
no allocation, no device-to-host copy inside the C-ABI calls (routing metadata
stays on the GPU).  A replay must reproduce the eager results bit for bit,
also after the inputs change in place (the graph reads device memory, not
values the host saw at capture time)."""

import pytest
import torch

from mixture_experts_layer_offsets_b200 import inputs
from mixture_experts_layer_offsets_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

OUTS = ("logits", "topk_idx", "topk_gate", "counts", "offsets", "slot_row", "x_perm", "act",
        "y_perm", "out", "dgate", "dy_perm", "dx_perm", "dw1", "dw2", "dx", "dw_router")


@pytest.mark.parametrize("name,capacity", [("bf16_e8", None), ("bf16_skew_e128", 60)])
def test_graph_replay_matches_eager(name, capacity):
    base = inputs.CONFIGS[name]
    cfg = inputs.shrink(base, T=1500, d_model=512, d_ff=256,
                        router_std=base.router_std if not base.bias_std else 512 ** -0.5)
    a = inputs.make_inputs(cfg, device="cuda", seed=4)
    b = inputs.make_inputs(cfg, device="cuda", seed=5)
    L = MoELayer(cfg.T, cfg.d_model, cfg.E, cfg.top_k, cfg.d_ff, cfg.dtype, "cuda",
                 capacity=capacity)
    live = {k: (v.clone() if v is not None else None) for k, v in a.items()}
    args = lambda: (live["x"], live["w_router"], live["bias"], live["w1"], live["w2"], live["dout"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        L.step(*args())
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        L.step(*args())

    for src in (a, b):  # replay on the capture inputs, then on new values in place
        for k, v in src.items():
            if v is not None:
                live[k].copy_(v)
        for k in OUTS:  # both runs start from the same buffers (rows a call does not
            getattr(L, k).fill_(0)  # write keep whatever they held)
        L.step(*args())
        torch.cuda.synchronize()
        eager = {k: getattr(L, k).clone() for k in OUTS}
        for k in OUTS:
            getattr(L, k).fill_(0)
        g.replay()
        torch.cuda.synchronize()
        for k in OUTS:
            assert torch.equal(getattr(L, k), eager[k]), k
    assert L.device_status() == 0
    del g
